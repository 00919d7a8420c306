// One-launch decode step of a whole algebraic SwiGLU FFN:
//   h = silu(x * Wg) . (x * Wu),   y = h * Wd
// where every "*" evaluates only the new token's row of the multiplication
// table (agihunt.info digest: decoding computes the new position's row as a
// matrix-vector product with a kernel of its own; the FFN's gate, up and down
// projections share the row types).
//
// The launch holds two kinds of CTA.  A gate/up CTA owns 16 columns of h: it
// pulls those columns of Wg and Wu for every input row with TMA (boxes of
// 16 columns x 256 rows, 32-byte swizzle), stages the activations x in
// rounds, runs warp-level tensor-core MMAs (mma.sync m16n8k16: M = the 16
// columns, N = batch entries, K = input rows) with each entry's table row
// applied to its operand fragment, and writes silu(g) u in bf16.  A down CTA
// owns 16 columns of y: it pulls its columns of Wd at launch, while the
// gate/up CTAs run, then waits until every gate/up CTA has written its part
// of h and streams h the same way.  The two phases meet in a grid barrier in
// device memory; no CTA of the first phase ever waits on another CTA, so the
// launch progresses whenever fewer down CTAs than SMs exist, and the wait is
// bounded (it records AAL_ERR_DEVICE_TIMEOUT and returns).
//
// Every output column sums over all input rows inside one CTA, so there is no
// split-K reduction across CTAs.  Inside a CTA the K range is split over
// warps, each warp keeps up to four batch tiles and two accumulator chains
// per tile (alternate K steps) so that dependent MMAs overlap, and the
// partials meet in shared memory.
#include <atomic>
#include <type_traits>

#include "aal_internal.h"

namespace aal {
namespace ffn {

constexpr int kThreads = 256;
constexpr int kCols = 16;         // output columns per CTA (one 32-byte row piece of a weight)
constexpr int kBoxRows = 256;     // weight rows per TMA box
constexpr int kMaxB = 128;        // batch entries per launch
constexpr int kSlots = 64;        // barrier slots, taken round robin per launch
constexpr int kSmemMax = 220 * 1024;
constexpr unsigned long long kWaitNs = 2000000000ull;

// Grid barrier state of one launch: ``count`` arrivals so far (back to 0 once
// all have arrived), ``gen`` bumped by the last arrival.  Each slot sits in
// its own 128-byte line.
struct __align__(128) Bar {
  unsigned count;
  unsigned gen;
  unsigned pad[30];
};
__device__ Bar g_ffn_bar[kSlots];

struct Params {
  CUtensorMap map_w[3];  // Wg, Wu, Wd seen as [rows][cols]: box {16 columns, 256 rows}, 32-byte swizzle
  CUtensorMap map_a[2];  // x and h of this launch's entries: box {64 columns, Bp rows}, 128-byte swizzle
  int law, q;
  int B, Bp;           // entries, entries rounded up to 8
  int D, F;
  int p1, p2;          // gate/up CTAs (F / 16) and down CTAs (D / 16)
  int kr1, kr2;        // activation rows staged per round in each phase
  int ng, ks;          // warps: ng groups of batch tiles x ks slices of K
  tc::FastDiv div_bi[2];  // input group size of the gate/up (D / q) and down (F / q) projections
  int slot;
  const int64_t* pos;
  __nv_bfloat16* h;
  long long ldh;
  __nv_bfloat16* y;
  long long ldy;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  // src_bytes 0 fills the 16 bytes with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// One arrival with acquire-release semantics at GPU scope: released are this
// thread's writes and, through the __syncthreads before it, its CTA's.  The
// last of ``total`` resets the count and bumps the generation.
__device__ __forceinline__ void bar_arrive(Bar* b, unsigned total) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(&b->count) : "memory");
  if (old == total - 1) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(&b->count), "r"(0u) : "memory");
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&b->gen) : "memory");
  }
}
// Waits (bounded) until the generation differs from ``g0``.
__device__ __noinline__ bool bar_wait(const Bar* b, unsigned g0) {
  const unsigned long long t0 = global_ns();
  for (unsigned i = 0;; ++i) {
    if (ld_acquire(&b->gen) != g0) return true;
    if ((i & 63u) == 63u && global_ns() - t0 > kWaitNs) {
      flag_device_error(kDevTimeout);
      return false;
    }
    __nanosleep(32);
  }
}
__device__ __forceinline__ void mbar_init1(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(bar)));
}
__device__ __forceinline__ void mbar_expect(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
// Bounded wait for the phase of ``bar`` with the given parity: false (and the
// timeout recorded) if it does not complete in kWaitNs.
__device__ __noinline__ bool mbar_wait0(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  for (unsigned i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((i & 63u) == 63u && global_ns() - t0 > kWaitNs) {
      flag_device_error(kDevTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load2(const CUtensorMap* map, uint32_t dst, uint64_t* bar, int c0,
                                          int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"((unsigned long long)map), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Shared-memory byte offset of row r, 16-byte column half c of a staged
// weight slice (rows of 32 bytes, 32-byte swizzle: the half flips on rows
// 4..7 of every 8).
__device__ __forceinline__ uint32_t wrow(int r, int c) {
  return (uint32_t)r * 32u + ((uint32_t)(c ^ ((r >> 2) & 1)) << 4);
}
// Byte offset of entry n, 16-byte chunk c (8 inputs) of a staged activation
// box (rows of 128 bytes, 128-byte swizzle: the chunk index is XORed with the
// row's index within its 8-row group).
__device__ __forceinline__ uint32_t arow(int n, int c) {
  return (uint32_t)n * 128u + ((uint32_t)(c ^ (n & 7)) << 4);
}

// NTW: batch tiles (8 entries) per warp; NCH = 8 / NTW independent
// accumulator chains per tile (consecutive K steps of a warp's slice go to
// different chains, so up to eight dependent-free MMAs are in flight).
template <int NTW>
__global__ void __launch_bounds__(kThreads, 1) k_ffn_decode(const __grid_constant__ Params p) {
  constexpr int NCH = 8 / NTW;
  extern __shared__ uint8_t dsm[];
  __shared__ int s_type[kMaxB];
  __shared__ unsigned s_pres[kThreads / 32][2];
  __shared__ unsigned char s_used[64];
  __shared__ int s_go;
  __shared__ __align__(8) uint64_t s_wbar;     // weight slice landed
  __shared__ __align__(8) uint64_t s_abar[2];  // activation buffer landed

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the position of entry tid is in flight while the copies are issued
  long long my_pos = -1;
  if (tid < p.B) my_pos = p.pos[tid];

  const bool up = (int)blockIdx.x < p.p1;  // gate/up CTA, else down CTA
  const int nops = up ? 2 : 1;
  const int K = up ? p.D : p.F;              // input rows of this CTA's projection
  const int bo = (up ? p.F : p.D) / p.q;     // output group size
  const int c0 = (up ? (int)blockIdx.x : (int)blockIdx.x - p.p1) * kCols;
  const int k = c0 / bo;                     // output group of the CTA's columns
  const int kr = up ? p.kr1 : p.kr2;         // activation columns per round (multiple of 64)
  const int nrounds = (K + kr - 1) / kr;
  const int nbox = (K + kBoxRows - 1) / kBoxRows;
  const int wrows = nbox * kBoxRows;         // staged rows per operand (the last box may run past K)
  const CUtensorMap* amap = &p.map_a[up ? 0 : 1];
  // dynamic shared memory (1024-byte aligned for the swizzles): weights,
  // two activation buffers of kr / 64 boxes each, partial sums
  const uint32_t base = (smem_addr(dsm) + 1023u) & ~1023u;
  uint8_t* sbase = dsm + (base - smem_addr(dsm));
  const uint32_t ws = base;
  const uint32_t abuf_bytes = (uint32_t)(kr / 64) * (uint32_t)p.Bp * 128u;
  const uint32_t as0 = ws + (uint32_t)(nops * wrows * 32);
  float* red = reinterpret_cast<float*>(sbase + (size_t)nops * wrows * 32 + 2 * (size_t)abuf_bytes);
  Bar* bar = &g_ffn_bar[p.slot];
  const unsigned total = (unsigned)(p.p1 + p.p2);

  if (tid == 0) {
    mbar_init1(&s_wbar);
    mbar_init1(&s_abar[0]);
    mbar_init1(&s_abar[1]);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    // A down CTA reads the generation, then arrives: the release needs this
    // arrival, so the CTA cannot miss the bump it waits for.
    if (!up) {
      const unsigned g = ld_acquire(&bar->gen);
      s_go = (int)g;
      bar_arrive(bar, total);
    }
  }
  __syncthreads();
  const unsigned g0 = (unsigned)s_go;

  // Round rd of the activations into buffer rd & 1: boxes of 64 inputs x
  // Bp entries (rows past the batch read as zeros), issued by warp 0's lanes.
  auto stage = [&](int rd) {
    const int r0 = rd * kr, cols = min(kr, K - r0), nb = (cols + 63) / 64;
    uint64_t* ab = &s_abar[rd & 1];
    if (lane == 0) mbar_expect(ab, (uint32_t)nb * (uint32_t)p.Bp * 128u);
    __syncwarp();
    const uint32_t dst = as0 + (uint32_t)(rd & 1) * abuf_bytes;
    for (int b = lane; b < nb; b += 32)
      tma_load2(amap, dst + (uint32_t)b * (uint32_t)p.Bp * 128u, ab, r0 + 64 * b, 0);
  };

  // 1. this CTA's columns of the weights for every input row, and the first
  //    round of x (no dependence on the positions, so the copies start at once)
  if (warp == 0) {
    if (lane == 0) {
      mbar_expect(&s_wbar, (uint32_t)(nops * nbox * kBoxRows * 32));
      for (int o = 0; o < nops; ++o)
        for (int bx = 0; bx < nbox; ++bx)
          tma_load2(&p.map_w[up ? o : 2], ws + (uint32_t)((o * wrows + bx * kBoxRows) * 32), &s_wbar, c0,
                    bx * kBoxRows);
    }
    if (up) stage(0);
  }

  // 2. row types (-1 for padding and negative positions) and the input
  //    groups some present type uses with output group k
  int t = -1;
  if (tid < p.B) {
    if (my_pos < 0) {
      if (blockIdx.x == 0) flag_device_error(kDevBounds);
    } else {
      t = (int)(my_pos % p.q);
    }
  }
  if (tid < p.Bp) s_type[tid] = t;
  const unsigned lo = __reduce_or_sync(0xffffffffu, (t >= 0 && t < 32) ? 1u << t : 0u);
  const unsigned hi = __reduce_or_sync(0xffffffffu, t >= 32 ? 1u << (t - 32) : 0u);
  if (lane == 0) { s_pres[warp][0] = lo; s_pres[warp][1] = hi; }
  __syncthreads();
  if (tid < p.q) {
    unsigned long long pres = 0ull;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w)
      pres |= (unsigned long long)s_pres[w][0] | ((unsigned long long)s_pres[w][1] << 32);
    bool u = false;
    for (int tt = 0; tt < p.q && !u; ++tt)
      if ((pres >> tt) & 1ull) u = in_table(p.law, tt, k, tid);
    s_used[tid] = u ? 1 : 0;
  }
  __syncthreads();  // s_used is read by every thread below

  if (!up) {
    // 3. down CTA: wait until every gate/up CTA has written its part of h,
    //    then read h through the async proxy
    if (tid == 0) s_go = bar_wait(bar, g0) ? 1 : 0;
    __syncthreads();
    if (!s_go) {
      mbar_wait0(&s_wbar, 0);  // the weight copies land before the CTA leaves
      return;
    }
    if (warp == 0) {
      // h was written through the generic proxy; the copies read it through
      // the async proxy
      asm volatile("fence.proxy.async;" ::: "memory");
      stage(0);
    }
  }
  bool ok = mbar_wait0(&s_wbar, 0);  // every thread sees the weight slice
  unsigned long long used = 0ull;     // bit a: some present type uses input group a
  for (int a = 0; a < p.q; ++a) used |= (unsigned long long)(s_used[a] != 0) << a;
  const tc::FastDiv dbi = p.div_bi[up ? 0 : 1];

  // 4. MMAs.  Warp (g, s): batch tiles g, g + NG, ... (up to NTW) and the
  //    s-th contiguous slice of each round's K steps.
  const int NT = p.Bp >> 3, NG = p.ng, KS = p.ks;
  const int wg = warp % NG, wk = warp / NG;
  float acc[2][NTW][NCH][4];
#pragma unroll
  for (int o = 0; o < 2; ++o)
#pragma unroll
    for (int j = 0; j < NTW; ++j)
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[o][j][c][e] = 0.f;
  int my_t[NTW];  // row type of the entry whose B fragment this lane holds
#pragma unroll
  for (int j = 0; j < NTW; ++j) {
    const int nt = wg + NG * j;
    my_t[j] = nt < NT ? s_type[nt * 8 + (lane >> 2)] : -1;
  }
  const int lrow = (lane & 7) + ((lane >> 4) << 3), lcol = (lane >> 3) & 1;
  for (int rd = 0; rd < nrounds && ok; ++rd) {
    const int r0 = rd * kr, rows = min(kr, K - r0);
    if (rd + 1 < nrounds && warp == 0) {
      // the buffer was last read in round rd - 1, which every warp has left
      if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      stage(rd + 1);
    }
    ok = mbar_wait0(&s_abar[rd & 1], (uint32_t)((rd >> 1) & 1));
    if (!ok) break;
    const uint32_t ab = as0 + (uint32_t)(rd & 1) * abuf_bytes;
    const int steps = rows >> 4, per = (steps + KS - 1) / KS;
    const int s_beg = wk * per, s_end = min(steps, s_beg + per);
    for (int s0 = s_beg; s0 < s_end; s0 += NCH) {
      // straight-line loads for NCH steps (a step past the slice reloads its
      // last step and is not multiplied), then the MMAs of the active steps
      uint32_t af[NCH][2][4];
      uint32_t bf[NCH][NTW][2];
      unsigned actm = 0u;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int st = min(s0 + c, s_end - 1);
        const int r = r0 + st * 16, a = (int)tc::fdiv((uint32_t)r, dbi);
        if (s0 + c < s_end && ((used >> a) & 1ull)) actm |= 1u << c;
        ldsm_x4_trans(ws + wrow(r + lrow, lcol), af[c][0]);
        if (up) ldsm_x4_trans(ws + (uint32_t)wrows * 32u + wrow(r + lrow, lcol), af[c][1]);
        const int kk = st * 16, bx = kk >> 6, ch = ((kk & 63) >> 3) + lcol;
#pragma unroll
        for (int j = 0; j < NTW; ++j) {
          const int nt = min(wg + NG * j, NT - 1);
          ldsm_x2(ab + (uint32_t)bx * (uint32_t)p.Bp * 128u + arow(nt * 8 + (lane & 7), ch), bf[c][j]);
          if (!(my_t[j] >= 0 && in_table(p.law, my_t[j], k, a))) { bf[c][j][0] = 0u; bf[c][j][1] = 0u; }
        }
      }
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        if (!((actm >> c) & 1u)) continue;
#pragma unroll
        for (int j = 0; j < NTW; ++j) {
          if (wg + NG * j >= NT) continue;
          mma16816(acc[0][j][c], af[c][0], bf[c][j]);
          if (up) mma16816(acc[1][j][c], af[c][1], bf[c][j]);
        }
      }
    }
    __syncthreads();  // this round's buffer is refilled in the next round
  }
  if (!ok) {
    // a copy never arrived (timeout recorded): write nothing; as a gate/up
    // CTA still arrive, so that the barrier slot is left balanced
    __syncthreads();
    if (up && tid == 0) bar_arrive(bar, total);
    return;
  }

  // 5. partials [ks][op][entry][16 columns] meet in shared memory
#pragma unroll
  for (int j = 0; j < NTW; ++j) {
    const int nt = wg + NG * j;
    if (nt >= NT) continue;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = nt * 8 + 2 * (lane & 3) + e, m = lane >> 2;
#pragma unroll
      for (int o = 0; o < 2; ++o) {
        if (o >= nops) break;
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) { v0 += acc[o][j][c][e]; v1 += acc[o][j][c][2 + e]; }
        float* dst = red + ((size_t)(wk * nops + o) * p.Bp + n) * kCols;
        dst[m] = v0;
        dst[m + 8] = v1;
      }
    }
  }
  __syncthreads();
  // one thread per (entry, column): sum the slices, apply the activation
  __nv_bfloat16* out = up ? p.h : p.y;
  const long long ldo = up ? p.ldh : p.ldy;
  for (int i = tid; i < p.B * kCols; i += kThreads) {
    const int n = i >> 4, m = i & 15;
    if (s_type[n] < 0) continue;
    float v = 0.f, u = 0.f;
    for (int sl = 0; sl < KS; ++sl) {
      v += red[((size_t)(sl * nops) * p.Bp + n) * kCols + m];
      if (up) u += red[((size_t)(sl * nops + 1) * p.Bp + n) * kCols + m];
    }
    if (up) v = __fdividef(v, 1.0f + __expf(-v)) * u;  // silu(g) * u = g / (1 + e^-g) * u
    out[(long long)n * ldo + c0 + m] = __float2bfloat16_rn(v);
  }
  if (up) {
    // 6. gate/up CTA: its part of h is written; arrive
    __syncthreads();
    if (tid == 0) bar_arrive(bar, total);
  }
}

static std::atomic<unsigned> g_next_slot{0};

static int num_sms_cached() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      n = v;
    else
      return 148;
  }
  return n;
}

// Warp split for Bp entries: (batch tiles per warp, tile groups, K slices).
static void warp_split(int Bp, int* ntw, int* ng, int* ks) {
  const int nt = Bp / 8;
  if (nt <= 1) { *ntw = 1; *ng = 1; *ks = 8; }
  else if (nt <= 2) { *ntw = 2; *ng = 1; *ks = 8; }
  else if (nt <= 4) { *ntw = 4; *ng = 1; *ks = 8; }
  else if (nt <= 8) { *ntw = 4; *ng = 2; *ks = 4; }
  else { *ntw = 4; *ng = 4; *ks = 2; }
}

static size_t phase_smem(int nops, int K, int Bp, int kr) {
  int ntw, ng, ks;
  warp_split(Bp, &ntw, &ng, &ks);
  const int wrows = (K + kBoxRows - 1) / kBoxRows * kBoxRows;
  return 1024 + (size_t)nops * wrows * 32 + (size_t)2 * (kr / 64) * Bp * 128 +
         (size_t)ks * nops * Bp * kCols * 4;
}

// Largest round (multiple of 64 inputs, at most K rounded up to 64) that fits.
static int pick_round(int nops, int K, int Bp) {
  for (int kr = (K + 63) / 64 * 64; kr >= 64; kr -= 64)
    if (phase_smem(nops, K, Bp, kr) <= (size_t)kSmemMax) return kr;
  return 0;
}

static bool rows16(const aal_mat& m) { return ((uintptr_t)m.ptr % 16) == 0 && m.ld % 8 == 0; }

// A weight [rows, cols] seen by TMA as a 2-D tensor: box {16 columns, 256 rows}.
static bool weight_map(CUtensorMap* m, const aal_mat& w) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)w.cols, (cuuint64_t)w.rows};
  cuuint64_t strides[1] = {(cuuint64_t)(w.ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)kCols, (cuuint32_t)kBoxRows};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.ptr, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The activations [entries, cols] of one launch: box {64 columns, Bp rows}
// (rows past ``rows`` read as zeros).
static bool act_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld, int Bp) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)Bp};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The one-launch kernel is opt-in (AAL_FFN_DECODE_FUSED=1 in the
// environment): on B200 the two tuned decode launches chained by a
// programmatic dependent launch measured faster at batch 1 to 64.
static bool fused_disabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("AAL_FFN_DECODE_FUSED");
    v = (e && e[0] == '1') ? 0 : 1;
  }
  return v == 1;
}

}  // namespace ffn

// Whether the one-launch kernel serves this FFN decode call.
bool ffn_decode_fused_ok(int law, int q, const aal_mat& x, const aal_mat& Wg, const aal_mat& Wu,
                         const aal_mat& Wd, const aal_mat& h, const aal_mat& y) {
  using namespace ffn;
  if (fused_disabled()) return false;
  const long long D = x.cols, F = Wg.cols;
  if (x.dtype != AAL_BF16 || q > 64 || D <= 0 || F <= 0 || D > (1 << 20) || F > (1 << 20)) return false;
  if ((D / q) % 16 || (F / q) % 16) return false;
  if (!rows16(x) || !rows16(Wg) || !rows16(Wu) || !rows16(Wd) || !rows16(h) || !rows16(y)) return false;
  const int sms = num_sms_cached();
  const long long p1 = F / kCols, p2 = D / kCols;
  if (p2 >= sms || p1 + p2 > 2LL * sms) return false;
  if (pick_round(2, (int)D, kMaxB) == 0 || pick_round(1, (int)F, kMaxB) == 0) return false;
  return true;
}

aal_status ffn_decode_fused(int law, int q, const int64_t* positions, const aal_mat& x,
                            const aal_mat& Wg, const aal_mat& Wu, const aal_mat& Wd, const aal_mat& h,
                            const aal_mat& y, cudaStream_t s) {
  using namespace ffn;
  static unsigned long long attr_done = 0;  // per device (bit dev % 64)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AAL_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done & bit)) {
    if (cudaFuncSetAttribute(k_ffn_decode<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) !=
            cudaSuccess ||
        cudaFuncSetAttribute(k_ffn_decode<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) !=
            cudaSuccess ||
        cudaFuncSetAttribute(k_ffn_decode<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) !=
            cudaSuccess)
      return AAL_ERR_CUDA;
    attr_done |= bit;
  }
  ffn::Params p;
  memset(&p, 0, sizeof(p));
  if (!weight_map(&p.map_w[0], Wg) || !weight_map(&p.map_w[1], Wu) || !weight_map(&p.map_w[2], Wd))
    return AAL_ERR_UNSUPPORTED;
  const long long B = x.rows;
  for (long long b0 = 0; b0 < B; b0 += kMaxB) {
    const int nb = (int)(B - b0 < kMaxB ? B - b0 : kMaxB);
    p.law = law;
    p.q = q;
    p.B = nb;
    p.Bp = (nb + 7) & ~7;
    p.D = (int)x.cols;
    p.F = (int)Wg.cols;
    p.p1 = p.F / kCols;
    p.p2 = p.D / kCols;
    p.kr1 = pick_round(2, p.D, p.Bp);
    p.kr2 = pick_round(1, p.F, p.Bp);
    int ntw = 1;
    warp_split(p.Bp, &ntw, &p.ng, &p.ks);
    p.div_bi[0] = tc::make_fastdiv((uint32_t)(p.D / q));
    p.div_bi[1] = tc::make_fastdiv((uint32_t)(p.F / q));
    p.slot = (int)(g_next_slot.fetch_add(1u) % kSlots);
    p.pos = positions + b0;
    p.h = (__nv_bfloat16*)h.ptr + b0 * h.ld;
    p.ldh = h.ld;
    if (!act_map(&p.map_a[0], (const __nv_bfloat16*)x.ptr + b0 * x.ld, nb, x.cols, x.ld, p.Bp) ||
        !act_map(&p.map_a[1], p.h, nb, h.cols, h.ld, p.Bp))
      return AAL_ERR_UNSUPPORTED;
    p.y = (__nv_bfloat16*)y.ptr + b0 * y.ld;
    p.ldy = y.ld;
    const size_t s1 = phase_smem(2, p.D, p.Bp, p.kr1), s2 = phase_smem(1, p.F, p.Bp, p.kr2);
    const size_t smem = s1 > s2 ? s1 : s2;
    const dim3 grid((unsigned)(p.p1 + p.p2));
    if (ntw == 1) k_ffn_decode<1><<<grid, ffn::kThreads, smem, s>>>(p);
    else if (ntw == 2) k_ffn_decode<2><<<grid, ffn::kThreads, smem, s>>>(p);
    else k_ffn_decode<4><<<grid, ffn::kThreads, smem, s>>>(p);
    note_launch();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return AAL_ERR_CUDA;
  }
  return AAL_OK;
}

}  // namespace aal
