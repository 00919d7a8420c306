// Explicit and ragged row types on the tensor-core path.
//
// The strided tensor-core path reads the rows of one type through a TMA view
// that needs every sequence to be a whole number of q positions long.  When
// the types are explicit, or the positions do not line up (agihunt.info
// digest, Transformer-mapping paragraph: a token's type comes from its
// absolute position, so any packing of sequences is legal), the rows are
// first sorted by type on the device into a caller workspace: a per-block
// histogram, one scan that also writes the tcgen05 kernel's tile table (a
// type's rows in tiles of 128), a scatter that records the permutation, and
// a wide gather that copies each row of X into its type's contiguous
// segment.  The tcgen05
// kernel then runs in segment mode and its epilogue writes every output row
// back to its original place.  No host synchronisation: the tile count stays
// on the device and tiles past it are empty.  The launches form one chain of
// programmatic dependent launches: each kernel lets the next one be launched
// as soon as it starts, and waits for its predecessor's results before it
// reads or writes anything, so the launch latencies overlap the work.
#include <utility>

#include "aal_internal.h"

namespace aal {
namespace seg {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = 4096;
constexpr int kMaxQ = 256;
constexpr int kPerThread = kRowsPerBlock / kThreads;  // rows of a histogram / scatter thread

struct Layout {
  size_t blk, counts, tiles, perm, xg, hg, total;
  long long G;  // row blocks of the histogram and scatter kernels
  int tmax;     // bound on the tile table's length
};

static size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

// Start of every kernel of the chain: release the next launch, then wait
// until the previous grid has finished and its writes are visible.
__device__ __forceinline__ void chain_enter() {
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <typename... Exp, typename... Act>
static cudaError_t launch_chained(void (*kernel)(Exp...), unsigned grid, unsigned block, cudaStream_t s,
                                  Act&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Act>(args)...);
}

// Workspace of a call over ``rows`` rows gathering w1 columns (and w2 more
// for a SwiGLU's hidden activation).
static Layout layout(int q, long long rows, long long w1, long long w2) {
  Layout L;
  L.G = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  L.tmax = (int)((rows + 127) / 128 + q);
  size_t off = 0;
  L.blk = off;
  off = up256(off + (size_t)L.G * q * 4);
  L.counts = off;
  off = up256(off + (size_t)(q + 4) * 4);
  L.tiles = off;
  off = up256(off + (size_t)L.tmax * 16);
  L.perm = off;
  off = up256(off + (size_t)rows * 4);
  L.xg = off;
  off = up256(off + (size_t)rows * w1 * 2);
  L.hg = off;
  off = up256(off + (size_t)rows * w2 * 2);
  L.total = off;
  return L;
}

// Warp-aggregated claim on the per-type counters c (shared memory): the
// lanes holding one type share a single atomic add.  Returns the lane's place
// among the claims (its old counter value plus its rank among those lanes),
// or -1 for t < 0.  All 32 lanes of the warp call it together.
__device__ __forceinline__ int claim(int* c, int t) {
  const unsigned peers = __match_any_sync(0xffffffffu, t);
  const int lane = threadIdx.x & 31, leader = __ffs(peers) - 1;
  int base = 0;
  if (t >= 0 && lane == leader) base = atomicAdd(&c[t], __popc(peers));
  base = __shfl_sync(0xffffffffu, base, leader);
  return t >= 0 ? base + __popc(peers & ((1u << lane) - 1u)) : -1;
}

// Types of rows r0 + u * kStride + threadIdx.x (u < N; -1 at and past row
// r0 + nr): every load is issued before any type is decoded and checked.
template <int N, int kStride>
__device__ __forceinline__ void load_types(const RowTypes& rt, long long r0, int nr, int (&ty)[N]) {
  long long raw[N];
#pragma unroll
  for (int u = 0; u < N; ++u) {
    const int i = u * kStride + (int)threadIdx.x;
    raw[u] = i < nr ? row_type_raw(rt, r0 + i) : 0;
  }
#pragma unroll
  for (int u = 0; u < N; ++u) {
    const int i = u * kStride + (int)threadIdx.x;
    ty[u] = i < nr ? row_type_decode(rt, r0 + i, raw[u]) : -1;
  }
}

// Segment starts seg[t] and tile-table starts tst[t] (exclusive prefix sums
// of the type counts cnt and of their 128-row tile counts), seg[q] and tst[q]
// the totals; the tile total also goes to counts[q] and the row total to
// counts[q + 1].  Run by warp 0: lane l
// takes a run of ceil(q / 32) types, and a shuffle scan joins the runs.
__device__ __forceinline__ void scan_starts(const int* cnt, int q, int* seg, int* tst, int* counts) {
  const int lane = threadIdx.x & 31, per = (q + 31) / 32, a = lane * per, b = a + per < q ? a + per : q;
  int sr = 0, nt = 0;
  for (int t = a; t < b; ++t) {
    sr += cnt[t];
    nt += (cnt[t] + 127) / 128;
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int s2 = __shfl_up_sync(0xffffffffu, sr, o), n2 = __shfl_up_sync(0xffffffffu, nt, o);
    if (lane >= o) {
      sr += s2;
      nt += n2;
    }
  }
  int s0 = __shfl_up_sync(0xffffffffu, sr, 1), n0 = __shfl_up_sync(0xffffffffu, nt, 1);
  if (lane == 0) s0 = n0 = 0;
  for (int t = a; t < b; ++t) {
    seg[t] = s0;
    tst[t] = n0;
    s0 += cnt[t];
    n0 += (cnt[t] + 127) / 128;
  }
  if (lane == 31) {
    seg[q] = sr;
    tst[q] = nt;
    counts[q] = nt;  // the tile count the tcgen05 kernel reads
    counts[q + 1] = sr;
  }
}

// 1. per-block histogram of the row types (rows with an invalid type are
//    left out; row_type records the bounds error)
__global__ void __launch_bounds__(kThreads) k_seg_hist(RowTypes rt, long long rows, int q, int* blk) {
  chain_enter();
  __shared__ int c[kMaxQ];
  for (int i = threadIdx.x; i < q; i += kThreads) c[i] = 0;
  __syncthreads();
  const long long r0 = (long long)blockIdx.x * kRowsPerBlock;
  const int nr = (int)(rows - r0 < kRowsPerBlock ? rows - r0 : kRowsPerBlock);
  int ty[kPerThread];
  load_types<kPerThread, kThreads>(rt, r0, nr, ty);
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) claim(c, ty[u]);
  __syncthreads();
  for (int i = threadIdx.x; i < q; i += kThreads) blk[(long long)blockIdx.x * q + i] = c[i];
}

// 2. one block: type totals, segment starts, per-(block, type) scatter
//    offsets (in place of the histogram), and the tile table
__global__ void __launch_bounds__(kThreads) k_seg_scan(long long G, int q, int* blk, int* counts,
                                                       int4* tiles) {
  chain_enter();
  __shared__ int tot[kMaxQ];
  __shared__ int seg[kMaxQ + 1];
  __shared__ int tst[kMaxQ + 1];
  for (int t = threadIdx.x; t < q; t += kThreads) {
    int s = 0;
    for (long long b = 0; b < G; ++b) s += blk[b * q + t];
    tot[t] = s;
  }
  __syncthreads();
  if (threadIdx.x < 32) scan_starts(tot, q, seg, tst, counts);
  __syncthreads();
  for (int t = threadIdx.x; t < q; t += kThreads) {
    int run = seg[t];
    for (long long b = 0; b < G; ++b) {
      const int c = blk[b * q + t];
      blk[b * q + t] = run;
      run += c;
    }
    counts[t] = tot[t];
    const int nt = (tot[t] + 127) / 128;
    for (int i = 0; i < nt; ++i) tiles[tst[t] + i] = make_int4(t, seg[t] + 128 * i, seg[t] + tot[t], 0);
  }
}

// 3. each row takes the next place of its type's segment; the permutation
//    records it
__global__ void __launch_bounds__(kThreads) k_seg_scatter(RowTypes rt, long long rows, int q, const int* blk,
                                                          int* perm) {
  chain_enter();
  __shared__ int cur[kMaxQ];
  for (int i = threadIdx.x; i < q; i += kThreads) cur[i] = blk[(long long)blockIdx.x * q + i];
  __syncthreads();
  const long long r0 = (long long)blockIdx.x * kRowsPerBlock;
  const int nr = (int)(rows - r0 < kRowsPerBlock ? rows - r0 : kRowsPerBlock);
  int ty[kPerThread];
  load_types<kPerThread, kThreads>(rt, r0, nr, ty);
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int d = claim(cur, ty[u]);
    if (d >= 0) perm[d] = (int)(r0 + u * kThreads + threadIdx.x);
  }
}

// 1-3 in one block, for calls whose rows all fit one block of the histogram:
// histogram, segment starts, tile table and permutation without leaving the
// CTA (one launch instead of three).  Each thread keeps its rows' types in
// registers between the two passes.
constexpr int kSmallThreads = 1024;
constexpr int kSmallPer = kRowsPerBlock / kSmallThreads;
__global__ void __launch_bounds__(kSmallThreads) k_seg_sort_small(RowTypes rt, long long rows, int q, int* counts,
                                                                  int4* tiles, int* perm) {
  chain_enter();
  __shared__ int c[kMaxQ];
  __shared__ int seg[kMaxQ + 1];
  __shared__ int tst[kMaxQ + 1];
  for (int i = threadIdx.x; i < q; i += kSmallThreads) c[i] = 0;
  __syncthreads();
  int ty[kSmallPer];
  load_types<kSmallPer, kSmallThreads>(rt, 0, (int)rows, ty);
#pragma unroll
  for (int u = 0; u < kSmallPer; ++u) claim(c, ty[u]);
  __syncthreads();
  if (threadIdx.x < 32) scan_starts(c, q, seg, tst, counts);
  __syncthreads();
  for (int t = threadIdx.x; t < q; t += kSmallThreads) {
    counts[t] = c[t];
    const int nt = (c[t] + 127) / 128;
    for (int i = 0; i < nt; ++i) tiles[tst[t] + i] = make_int4(t, seg[t] + 128 * i, seg[t] + c[t], 0);
    c[t] = seg[t];  // now the next free place of type t
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kSmallPer; ++u) {
    const int d = claim(c, ty[u]);
    if (d >= 0) perm[d] = (int)(threadIdx.x + u * kSmallThreads);
  }
}

// 4. the gathered copy: row d of Xg is row perm[d] of X (one warp per row,
//    16-byte vectors, kGatherBatch of them per lane loaded before any is
//    stored; rows past the sorted count are left alone)
constexpr int kGatherBatch = 8;
__global__ void __launch_bounds__(kThreads) k_seg_gather(const int* __restrict__ counts, int q,
                                                         const int* __restrict__ perm,
                                                         const __nv_bfloat16* __restrict__ X, long long ldx, int cols,
                                                         __nv_bfloat16* __restrict__ Xg, long long ldg, long long rows) {
  chain_enter();
  const int total = counts[q + 1];  // rows with a valid type
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nv = cols >> 3;
  for (long long d = (long long)blockIdx.x * (kThreads / 32) + warp; d < rows && d < total;
       d += (long long)gridDim.x * (kThreads / 32)) {
    const uint4* __restrict__ src = reinterpret_cast<const uint4*>(X + (long long)perm[d] * ldx);
    uint4* __restrict__ out = reinterpret_cast<uint4*>(Xg + d * ldg);
    for (int v0 = lane; v0 < nv; v0 += 32 * kGatherBatch) {
      uint4 r[kGatherBatch];
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u)
        if (v0 + 32 * u < nv) r[u] = src[v0 + 32 * u];
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u)
        if (v0 + 32 * u < nv) out[v0 + 32 * u] = r[u];
    }
  }
}

static bool rows16(const aal_mat& m) {
  return m.dtype == AAL_BF16 && ((uintptr_t)m.ptr % 16) == 0 && m.ld % 8 == 0;
}

}  // namespace seg

// Whether the rows of this rule need the sorted (segment) path: explicit
// types, or sequences / rows that are not whole multiples of q.
bool seg_needed(const RowTypes& rt, int q, long long rows) {
  return !(rt.kind == kTypesPosition && rt.seq_len % q == 0 && rows % q == 0);
}

int64_t seg_workspace_bytes(int q, long long rows, long long w1, long long w2) {
  return (int64_t)seg::layout(q, rows, w1, w2).total;
}

// Sorts the rows by type and gathers X into the workspace's segments.
static aal_status seg_prepare(int q, const RowTypes& rt, long long rows, const aal_mat& X, char* ws,
                              const seg::Layout& L, cudaStream_t s) {
  using namespace seg;
  int* blk = (int*)(ws + L.blk);
  int* counts = (int*)(ws + L.counts);
  int4* tiles = (int4*)(ws + L.tiles);
  int* perm = (int*)(ws + L.perm);
  __nv_bfloat16* Xg = (__nv_bfloat16*)(ws + L.xg);
  cudaError_t e;
  if (L.G == 1) {
    e = launch_chained(k_seg_sort_small, 1, kSmallThreads, s, rt, rows, q, counts, tiles, perm);
  } else {
    e = launch_chained(k_seg_hist, (unsigned)L.G, seg::kThreads, s, rt, rows, q, blk);
    if (e == cudaSuccess) e = launch_chained(k_seg_scan, 1, seg::kThreads, s, L.G, q, blk, counts, tiles);
    if (e == cudaSuccess) e = launch_chained(k_seg_scatter, (unsigned)L.G, seg::kThreads, s, rt, rows, q,
                                             (const int*)blk, perm);
  }
  const long long gb = (rows + seg::kThreads / 32 - 1) / (seg::kThreads / 32);
  if (e == cudaSuccess)
    e = launch_chained(k_seg_gather, (unsigned)(gb < 4096 ? gb : 4096), seg::kThreads, s, (const int*)counts, q,
                       (const int*)perm, (const __nv_bfloat16*)X.ptr, X.ld, (int)X.cols, Xg, (long long)X.cols,
                       rows);
  note_launch(L.G == 1 ? 2 : 4);
  return cuda_status(e);
}

// Common eligibility of the segment path (before anything is launched).
static bool seg_ok(int q, long long rows, const aal_mat& X, const aal_mat* const* mats, int nmats,
                   void* ws, uint64_t ws_bytes, long long w2) {
  if (q > seg::kMaxQ || rows <= 0 || rows > (1LL << 30) || !ws || ((uintptr_t)ws % 256) != 0) return false;
  if (!seg::rows16(X) || (X.cols % 16)) return false;
  for (int i = 0; i < nmats; ++i)
    if (!seg::rows16(*mats[i])) return false;
  return (uint64_t)seg_workspace_bytes(q, rows, X.cols, w2) <= ws_bytes;
}

aal_status seg_project_fwd(int law, int q, const RowTypes& rt, const aal_mat& X, const aal_mat& W,
                           const aal_mat& Y, void* ws, uint64_t ws_bytes, cudaStream_t s) {
  const aal_mat* mats[] = {&W, &Y};
  if (!seg_ok(q, X.rows, X, mats, 2, ws, ws_bytes, 0)) return AAL_ERR_UNSUPPORTED;
  if ((X.cols / q) % 16 || (W.cols / q) % 16) return AAL_ERR_UNSUPPORTED;
  const seg::Layout L = seg::layout(q, X.rows, X.cols, 0);
  char* w = (char*)ws;
  aal_status st = seg_prepare(q, rt, X.rows, X, w, L, s);
  if (st != AAL_OK) return st;
  aal_mat Xg = X;
  Xg.ptr = w + L.xg;
  Xg.ld = X.cols;
  return tc_project_seg(law, q, X.rows, Xg, W, nullptr, Y, (const int4*)(w + L.tiles),
                        (const int*)(w + L.counts) + q, (const int*)(w + L.perm), L.tmax, nullptr, s);
}

aal_status seg_swiglu_fwd(int law, int q, const RowTypes& rt, const aal_mat& X, const aal_mat& Wg,
                          const aal_mat& Wu, const aal_mat& Wd, const aal_mat& H, const aal_mat& Y, void* ws,
                          uint64_t ws_bytes, cudaStream_t s) {
  const aal_mat* mats[] = {&Wg, &Wu, &Wd, &H, &Y};
  const long long F = Wg.cols;
  if (!seg_ok(q, X.rows, X, mats, 5, ws, ws_bytes, F)) return AAL_ERR_UNSUPPORTED;
  if ((X.cols / q) % 16 || (F / q) % 16) return AAL_ERR_UNSUPPORTED;
  const seg::Layout L = seg::layout(q, X.rows, X.cols, F);
  char* w = (char*)ws;
  aal_status st = seg_prepare(q, rt, X.rows, X, w, L, s);
  if (st != AAL_OK) return st;
  aal_mat Xg = X, Hg = H;
  Xg.ptr = w + L.xg;
  Xg.ld = X.cols;
  Hg.ptr = w + L.hg;
  Hg.ld = F;
  const int4* tiles = (const int4*)(w + L.tiles);
  const int* count = (const int*)(w + L.counts) + q;
  const int* perm = (const int*)(w + L.perm);
  // gate/up with SiLU*mul: H in the caller's row order, and the gathered
  // copy the down projection reads
  st = tc_project_seg(law, q, X.rows, Xg, Wg, &Wu, H, tiles, count, perm, L.tmax, &Hg, s);
  if (st != AAL_OK) return st;
  return tc_project_seg(law, q, X.rows, Hg, Wd, nullptr, Y, tiles, count, perm, L.tmax, nullptr, s);
}

}  // namespace aal
