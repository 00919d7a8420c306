// Tensor-core path: one persistent, warp-specialised tcgen05 kernel for every
// block product of the algebra.
//
// What it computes.  Every call is a set of output tiles; a tile is a
// 128 x N fp32 accumulator in tensor memory (TMEM) that sums, over the
// members a of a table entry S(t, k), the block products X_a W_ak (agihunt.info
// digest, multiplication-table paragraph).  The K range of a tile is a list of
// up to six "segments" (one per table member, or a merged contiguous range),
// walked in 64-element chunks; each chunk is one TMA load of an A tile and a B
// tile into shared memory and up to four tcgen05.mma instructions (K = 16
// each) accumulating into TMEM.  Because the |S| products of a tile land in
// the same accumulator, the sum over the table never round-trips through HBM.
//
// Row typing without a gather pass.  A token of type t sits at rows
// r = j*q + c with c = (t - offset) mod q when sequences are multiples of q
// long (agihunt.info digest: the type comes from the absolute position).  A
// row-major [M, d] matrix is therefore described to TMA as a 3-D tensor
// [M/q][q][d]; a box with extent 1 in the middle dimension pulls the rows of
// one type class straight out of HBM.  No index buffer, no copy.
//
// Roles (448 threads): warps 0 and 10..12 issue TMA loads (chunk i goes to
// producer warp i mod 4), warp 1 owns TMEM and issues the MMAs (one thread),
// warps 2..9 drain TMEM to registers and write bf16 results (optionally
// applying SiLU(g)*u or adding into the destination; two epilogue warps share
// each 32-lane quarter of TMEM and split its columns), and warp 13 decodes
// the tiles into a shared-memory ring the other roles read.
// Schedules: up to 1024 tiles of unequal cost are assigned on the host
// longest first to the least loaded CTA; launches with many tiles a CTA hand
// them out through a counter in device memory (CTAs that run faster take
// more); the rest stride through the tile list.
// Sharing the term common to several outputs (Q_q): on the swapped layout a
// tile holds 2-4 row types and their diagonal term is one MMA (class groups);
// on the unswapped projection, the fused gate/up and the square product a
// tile holds two output groups and the type's (row block's) own term spans
// both (output-group pairs); with at most 64 rows a type two types share an
// unswapped tile (class pairs).  Each such mode is compiled only into the
// instantiations that use it (the MODE template parameter, compile-time flags).
// The backward's few very long tiles can run as split-K pieces added by a
// reduction kernel (with a caller workspace).
// Every launch is a programmatic dependent launch: a CTA sets up while the
// previous grid finishes and waits (griddepcontrol.wait) before its first
// global access; the tile decoder, which reads only parameters, starts early.
// Shared-memory stages and the two TMEM accumulator buffers are handed over
// with mbarriers; every wait is bounded (2 s of global time) and on expiry the
// kernel records AAL_ERR_DEVICE_TIMEOUT in the status word, lets in-flight
// copies and MMAs land, frees TMEM and returns.
#include <cuda.h>

#include <algorithm>
#include <queue>
#include <atomic>
#include <vector>
#include <limits.h>
#include <stdlib.h>

#include "aal_internal.h"

namespace aal {
namespace tc {

constexpr int kEpiWarps = 8;
// TMA producer warps: warp 0 and the warps after the epilogue.  One warp's
// bulk-tensor copies are issued one after another at several hundred cycles
// each whatever the box size, so consecutive K chunks go to different warps.
constexpr int kProdWarps = 4;
// One more warp decodes each tile once (index -> table segments and
// coordinates) into a ring in shared memory that every role reads.
constexpr int kSchedWarp = 2 + kEpiWarps + kProdWarps - 1;
constexpr int kThreads = 32 * (kSchedWarp + 1);
constexpr int kTileRing = 8;
// Tile schedules up to this many slots are balanced on the host (longest
// processing time first onto the least loaded CTA) and passed with the launch.
constexpr int kMaxOrder = 1024;
constexpr int kMaxPairs = 256;
constexpr int kMaxSegs = 6;  // K segments of one tile
constexpr int kMaxStages = 8;
constexpr int kSmemBudget = 224 * 1024;  // + 1 KB alignment slack, under the 227 KB per-CTA limit
constexpr int kEpiSmem = kEpiWarps * 2048;  // TMA-store staging
constexpr unsigned long long kWaitNs = 2000000000ull;
// Limit of the test stall (see Params::test_stall).
constexpr unsigned long long kStallNs = 50000000ull;

enum Op : int { OP_FWD = 0, OP_SWIGLU = 1, OP_DX = 2, OP_DW = 3, OP_SQUARE = 4 };

// Exact unsigned division by a runtime constant (x < 2^31): q = (hi(x*m) + x) >> s.
struct FastDiv {
  uint32_t d, m, s;
};
__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.s = 0;
  while ((1u << f.s) < d) ++f.s;
  f.m = (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << f.s) - d)) / d + 1);
  return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t x, const FastDiv& f) {
  return (uint32_t)(((uint64_t)__umulhi(x, f.m) + x) >> f.s);
}

struct Seg {
  int k0;   // first K index of the segment (feature column, or token within the class)
  int len;  // K extent
  int cls;  // row class used for coordinate 1 of gathered operands
  int map;  // which of the two maps of a gathered operand (dW: 1 = contiguous rows)
};

struct Params {
  CUtensorMap mapA[2];
  CUtensorMap mapB[2];
  CUtensorMap mapOut;  // output seen as [rows/qv][qv][cols]: box {16, 1, 32} (SW32)
                       // or, when swapped, {32, 1, 16} (no swizzle)
  int op, law, q, off;
  int bi, bo;          // block sizes of the two grouped dimensions (op specific)
  int n_mma;           // MMA N (the MMA M is always 128)
  int a_aw, b_aw;      // atom width (elements) of MN-major A / B tiles: 64 or 16
  int a_rows, b_rows;  // MN extent of the A tile (128) and of the B tile (n_mma)
  int swap;            // 1: TMEM lanes run along the column side of the output
  int n1, n2, n3;      // tile index = ((i0*n1 + i1)*n2 + i2)*n3 + i3
  int ntiles;
  long long Mq;        // rows per class of gathered operands
  long long Mall;      // all rows (dW over a contiguous map)
  int qv;              // classes in the gathered view
  int xr;              // token rows per tile
  int wn;              // output columns per tile on the weight side
  uint32_t idesc;      // tcgen05 instruction descriptor (kind::f16, bf16 x bf16 -> f32)
  uint32_t idesc2;     // same with N = 2 * n_mma (gate and up tiles read as one operand)
  int fuse_b;          // DUAL == 1: issue one MMA over both B tiles
  int stages;
  uint32_t stage_bytes, a_bytes, b_bytes;
  int acc_cols;        // TMEM columns of one accumulator set
  uint32_t tmem_cols;  // TMEM allocation (power of two)
  int swiglu;          // epilogue: silu(acc0) * acc1
  int accumulate;      // epilogue: out += acc (register path, no TMA store)
  int swiglu_bwd;      // epilogue: acc is dH; with G, U at the same place write
                       // dG = dH u silu'(g) to out and dU = dH silu(g) to out2
  const __nv_bfloat16* g_in;
  const __nv_bfloat16* u_in;
  __nv_bfloat16* out2;
  int tma_store;       // epilogue: stage in shared memory and store with TMA
  __nv_bfloat16* out;
  long long ldo;
  // Tile order: pair rank -> (p0, p1).  For q <= 16 the host stores the pairs
  // sorted by cost (p0 << 8 | p1); otherwise the law is Q_q and the diagonal
  // pairs go first (diag_first) or last.
  int npairs_list;
  int diag_first;
  uint16_t pairs[kMaxPairs];
  FastDiv div_n1, div_n3, div_qm1;
  int a_merged, b_merged;  // MN-major operand loaded as one box spanning all its atoms
  // Schedule: CTA c runs the tiles order[c], order[c + grid], ... up to the
  // first 0xFFFF (use_order), else tiles c, c + grid, ... below ntiles.
  int use_order;
  int nslots;
  // Test hook: 1 makes the MMA thread first wait on a barrier nothing ever
  // arrives on, so the bounded wait runs out (after kStallNs), the kernel
  // records AAL_ERR_DEVICE_TIMEOUT and takes its abort path.
  int test_stall;
  int map_mask;        // tensor maps in use: bits 0-1 mapA, 2-3 mapB, 4 mapOut
  // Split K of the heavy Q_q tiles (dW diagonal blocks a == k, whose K runs
  // over every token, and dX tiles a == t, whose K runs over every output
  // group).  Heavy tile dg = (i0 * n1 + i1) * n3 + i3 is cut into ksplit
  // pieces of split_len K positions: piece 0 is the tile's own slot, pieces
  // 1.. are the extra tiles split_base + dg * (ksplit - 1) + piece - 1.  Each
  // piece writes its fp32 accumulator to split_ws[dg * ksplit + piece][128][n_mma]
  // (TMEM lane, column) and a reduction kernel adds the pieces.
  int ksplit, split_len, split_base;
  float* split_ws;
  // Class-group mode (swapped forward under Q_q): a tile covers grp classes
  // of grp_n token rows each; its diagonal segment is one MMA over all of them
  // (N = grp * grp_n, idesc), its per-class segments MMAs of N = grp_n
  // (idesc_one) into the class's TMEM columns.  box_bytes: one class's B box.
  int grp, grp_n;
  uint32_t idesc_one, box_bytes;
  // Output-group pairs (unswapped projection under Q_q, the k_tc<0,1,0,0,true>
  // instantiation): a tile covers output groups k0 = 2 kp and k0 + 1 of one
  // class; its first segment is X_c[., t] W(t, [k0, k0 + 2)) as one MMA of
  // N = 2 rg_n, then X_c[., g] W(g, g) for each g != t of the pair as an MMA
  // of N = rg_n (idesc_one) into group g's TMEM columns.
  int rg_n;
  // Dynamic schedule (>= 0): CTA c runs tile c first, then the tiles handed
  // out by the counter pair g_tile_ctr[dyn_slot] (next, CTAs done), so SMs
  // that run faster take more tiles; the last CTA to finish resets the pair.
  int dyn_slot;
  // Segment mode (forward ops with explicit or ragged row types): the rows
  // were gathered type by type into contiguous segments; tile j of the device
  // table seg_tiles (j < *seg_count) is {type, first row, end of its type's
  // segment, 0}; tile index = (j * q + k) * n3 + i3.  Output row x of the
  // gathered order is row seg_perm[x] of the caller's output; with seg_copy
  // the tile is also written, in the gathered order, to seg_copy.
  // Ragged mode (forward projection whose blocks are not multiples of 16,
  // e.g. 20 x 100): a segment is one input group a of gbi features.  Its A
  // box holds ka features from the 16-byte aligned start below a * gbi (the
  // group sits at offset (a * gbi) mod 8); its B boxes come from W seen as
  // [groups][gbi rows][cols], started at row -offset, so every K position
  // outside the group reads as zero and the neighbours' features in A are
  // multiplied by zeros.  A tile spans N columns from the 16-column aligned
  // start below k * gbo; the epilogue writes the group's gbo columns only.
  int ragged;
  int gbi, gbo, ka;
  uint32_t tx_bytes;   // bytes one stage's copies deliver
  uint32_t b_lbo;      // MN-major B: bytes between 16-column atoms (ragged mode)
  int seg_mode;
  const int4* seg_tiles;
  const int* seg_count;
  const int* seg_perm;
  __nv_bfloat16* seg_copy;
  long long ld_copy;
  FastDiv div_qn3;
  uint16_t order[kMaxOrder];
};

static_assert(sizeof(Params) <= 4096, "kernel parameters stay within the classic 4 KB limit");

struct TileDesc {
  Seg seg[kMaxSegs];
  int nseg;
  int a_f, b_f;    // fixed coordinate of A / B (row start of K-major, column start of MN-major)
  int a_c1, b_c1;  // 1: coordinate 1 is the segment's class
  long long rbase;
  int rstride, roff;
  long long rlimit;
  long long cbase;
  int vlo, vhi;    // tile columns the epilogue writes (ragged mode)
  int split;       // >= 0: a piece of a split heavy tile (partial-sum slot), else -1
};

// Tile counters of the dynamic schedule, one pair per launch slot (launches
// take slots round-robin, so consecutive launches, which may overlap under
// programmatic dependent launch, never share one).  Zero between launches.
constexpr int kDynSlots = 64;
__device__ unsigned int g_tile_ctr[kDynSlots][2];

// ------------------------------------------------------------------ PTX glue
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long gtime() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok;
}
// Bounded wait by one thread.  Returns false if the kernel was aborted or the
// wait ran out (which records the timeout and aborts the kernel).
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                       unsigned long long limit_ns = kWaitNs) {
  const unsigned long long t0 = gtime();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u) {
      if (*abort) return false;
      if (gtime() - t0 > limit_ns) {
        flag_device_error(kDevTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}
// Bounded wait used during teardown: never aborts early, gives up after the limit.
__device__ __noinline__ void mbar_wait_teardown(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = gtime();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return;
    if ((i & 255u) == 255u && gtime() - t0 > kWaitNs) {
      flag_device_error(kDevTimeout);
      return;
    }
  }
}
// The whole warp waits on lane 0's bounded wait (first probe inline).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const int lane = threadIdx.x & 31;
  uint32_t ok = 0;
  if (lane == 0) ok = (mbar_try_wait(bar, parity) || mbar_wait(bar, parity, abort)) ? 1u : 0u;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

__device__ __forceinline__ void tma_load(const CUtensorMap* map, uint32_t dst, uint64_t* bar,
                                         int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"((unsigned long long)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_store(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                          int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          (unsigned long long)map),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- CTA-pair (cta_group::2) helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory object in CTA ``rank`` of the cluster.
__device__ __forceinline__ uint32_t mapa_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// TMA load whose completion counts on an mbarrier that may sit in the peer CTA.
__device__ __forceinline__ void tma_load_pair(const CUtensorMap* map, uint32_t dst, uint32_t bar,
                                              int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"((unsigned long long)map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrives on the barrier at this offset in both CTAs of the pair once the
// pair's previously issued MMAs have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"((unsigned short)3)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ void tma_load4(const CUtensorMap* map, uint32_t dst, uint64_t* bar,
                                          int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"((unsigned long long)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_load4_pair(const CUtensorMap* map, uint32_t dst, uint32_t bar,
                                               int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"((unsigned long long)map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 "version 1").  Field units are
// 16 bytes.  K-major tiles: rows of 128 B (64 bf16 of K) in 8-row, 1024 B
// swizzle atoms; SBO = 1024 B between 8-row groups, LBO unused; a K step of 16
// elements moves the start address by 32 B.  MN-major tiles: per atom, rows of
// (atom width x 2) B, one row per K index; LBO = distance between atoms along
// MN, SBO = distance between 8-row K groups.
__device__ __forceinline__ uint64_t make_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for tcgen05
  d |= (uint64_t)layout << 61;
  return d;
}
constexpr uint32_t kLayoutSW128 = 2, kLayoutSW64 = 4, kLayoutSW32 = 6;

// Descriptor of an operand tile at shared address ``tile`` (K step 0) and the
// amount a K step of 16 adds to it (the start-address field is in 16-byte
// units, so advancing the address is a plain 64-bit add).
template <bool MN>
__device__ __forceinline__ uint64_t operand_desc0(uint32_t tile, int aw) {
  if (!MN) return make_desc(tile, 16, 1024, kLayoutSW128);
  if (aw == 64) return make_desc(tile, 64 * 128, 1024, kLayoutSW128);
  return make_desc(tile, 64 * 32, 8 * 32, kLayoutSW32);
}
template <bool MN>
__device__ __forceinline__ uint64_t operand_kstep(int aw) {
  if (!MN) return 32 >> 4;
  return aw == 64 ? (16 * 128) >> 4 : (16 * 32) >> 4;
}


// ------------------------------------------------------------- tile layout
// A tile description lives in registers: every access to its segment array
// uses a constant index (a runtime index would put it in local memory, and
// every role decodes every tile it visits).
__device__ __forceinline__ void add_seg(TileDesc& d, int k0, int len, int cls, int map) {
  // merge with the previous segment when the K ranges touch (same class/map)
  bool merged = false;
#pragma unroll
  for (int j = 0; j < kMaxSegs; ++j) {
    Seg& s = d.seg[j];
    if (j == d.nseg - 1 && s.cls == cls && s.map == map && s.k0 + s.len == k0) {
      s.len += len;
      merged = true;
    }
  }
  if (merged) return;
#pragma unroll
  for (int j = 0; j < kMaxSegs; ++j) {
    if (j == d.nseg) {
      d.seg[j].k0 = k0;
      d.seg[j].len = len;
      d.seg[j].cls = cls;
      d.seg[j].map = map;
    }
  }
  ++d.nseg;
}
__device__ __forceinline__ Seg seg_at(const TileDesc& d, int s) {
  Seg r = d.seg[0];
  if (s == 1) r = d.seg[1];
  if (s == 2) r = d.seg[2];
  if (s == 3) r = d.seg[3];
  if (s == 4) r = d.seg[4];
  if (s == 5) r = d.seg[5];
  return r;
}
// The members a of S(t, k) in ascending order, each added as a K segment of
// width ``w`` starting at a * w (class ``cls``).
__device__ __forceinline__ void add_members(const Params& p, TileDesc& d, int t, int k, int w, int cls) {
  if (p.law == AAL_LAW_Q) {
    if (t == k) {
      add_seg(d, t * w, w, cls, 0);
    } else {
      add_seg(d, min(t, k) * w, w, cls, 0);
      add_seg(d, max(t, k) * w, w, cls, 0);
    }
  } else {
#pragma unroll
    for (int g = 0; g < 4; ++g)
      if (in_table(p.law, t, k, g)) add_seg(d, g * w, w, cls, 0);
  }
}

// The p1 that makes pair (p0, p1) diagonal: the row type of class p0 for the
// row-typed ops, p0 itself for the square product and dW.
__device__ __forceinline__ int type_of_class(const Params& p, int c) {
  const int t = c + p.off;  // c, off < q
  return t >= p.q ? t - p.q : t;
}
__device__ __forceinline__ int diag_partner(const Params& p, int p0) {
  return (p.op == OP_SQUARE || p.op == OP_DW) ? p0 : type_of_class(p, p0);
}

__device__ __forceinline__ void pair_of(const Params& p, int pr, int& p0, int& p1) {
  if (p.npairs_list) {
    const int v = p.pairs[pr];
    p0 = v >> 8;
    p1 = v & 255;
    return;
  }
  const int q = p.q, nd = q * (q - 1);
  int r = pr;
  if (p.diag_first) {
    if (r < q) { p0 = r; p1 = diag_partner(p, r); return; }
    r -= q;
  } else if (r >= nd) {
    p0 = r - nd;
    p1 = diag_partner(p, p0);
    return;
  }
  p0 = (int)fdiv((uint32_t)r, p.div_qm1);
  const int j = r - p0 * (q - 1), dg = diag_partner(p, p0);
  p1 = j < dg ? j : j + 1;
}

// Segment mode: tile = (j * q + k) * n3 + i3 over the device tile table.
__device__ __forceinline__ void describe_seg(const Params& p, int tile, TileDesc& d) {
  d.vlo = 0;
  d.vhi = INT_MAX;
  const int j = (int)fdiv((uint32_t)tile, p.div_qn3);
  const int rem = tile - j * p.q * p.n3;
  const int k = (int)fdiv((uint32_t)rem, p.div_n3);
  const int i3 = rem - k * p.n3;
  d.nseg = 0;
  d.rstride = 1;
  d.roff = 0;
  d.a_c1 = 0;
  d.b_c1 = 0;
  d.b_f = k * p.bo + i3 * p.wn;
  d.cbase = d.b_f;
  if (j >= *(volatile const int*)p.seg_count) {  // past the table: an empty tile
    d.a_f = 0;
    d.rbase = 0;
    d.rlimit = 0;
    return;
  }
  const int4 e = p.seg_tiles[j];
  add_members(p, d, e.x, k, p.bi, 0);
  d.a_f = e.y;
  d.rbase = e.y;
  d.rlimit = e.z;
}

// tile = (pair_rank * n1 + i1) * n3 + i3; the pair is (i0, i2) of the op.
// Segment markers of output-group-pair tiles (Seg::map): the type's own
// segment spans both groups' columns; a diagonal segment only group j's.
constexpr int kRgWide = 0x40, kRgNarrow = 0x20;

// Output-group-pair tile (c, i1, kp): class c's 128-row block i1, output
// groups k0 = 2 kp and k0 + 1.  Under Q_q, y_g = x_t W(t, g) + [g != t] x_g W(g, g).
// For the square product the class is row block i (Z_ig = X_ii W_ig + [g != i]
// X_ig W_gg) and its rows are plain rows of X and Z.
__device__ __forceinline__ void describe_rg(const Params& p, int tile, TileDesc& d) {
  const int npair = p.q >> 1;
  if (p.seg_mode) {
    // segment mode: entry j of the tile table (type t, gathered rows
    // [e.y, e.z)) and output groups 2 kp, 2 kp + 1
    const int j = tile / npair, k0 = 2 * (tile - j * npair);
    d.nseg = 0;
    d.a_c1 = 0;
    d.b_f = k0 * p.bo;
    d.b_c1 = 0;
    d.rstride = 1;
    d.roff = 0;
    d.cbase = d.b_f;
    d.vlo = 0;
    d.vhi = INT_MAX;
    if (j >= *(volatile const int*)p.seg_count) {  // past the table: an empty tile
      d.a_f = 0;
      d.rbase = 0;
      d.rlimit = 0;
      return;
    }
    const int4 e = p.seg_tiles[j];
    add_seg(d, e.x * p.bi, p.bi, 0, kRgWide);
    for (int g = 0; g < 2; ++g)
      if (k0 + g != e.x) add_seg(d, (k0 + g) * p.bi, p.bi, 0, kRgNarrow | g);
    d.a_f = e.y;
    d.rbase = e.y;
    d.rlimit = e.z;
    return;
  }
  const int kp = tile % npair, r = tile / npair, i1 = r % p.n1, c = r / p.n1;
  const bool sq = p.op == OP_SQUARE;
  const int k0 = 2 * kp, t = sq ? c : type_of_class(p, c);
  const int cls = sq ? 0 : c;
  d.nseg = 0;
  add_seg(d, t * p.bi, p.bi, cls, kRgWide);
  for (int j = 0; j < 2; ++j)
    if (k0 + j != t) add_seg(d, (k0 + j) * p.bi, p.bi, cls, kRgNarrow | j);
  d.a_f = sq ? c * p.bi + i1 * 128 : i1 * 128;
  d.a_c1 = sq ? 0 : 1;
  d.b_f = k0 * p.bo;
  d.b_c1 = 0;
  d.rbase = d.a_f;
  d.rstride = sq ? 1 : p.qv;
  d.roff = sq ? 0 : c;
  d.rlimit = sq ? LLONG_MAX : p.Mq;
  d.cbase = d.b_f;
  d.vlo = 0;
  d.vhi = INT_MAX;
}

// Class-pair tile (cp, k, i3) of the unswapped projection (at most 64 rows a
// type): the 128 A rows are classes c0 = 2 cp and c0 + 1, 64 rows each.  The
// diagonal term X_c[., k] W(k, k) is one MMA over both; X_c[., t] W(t, k)
// (t = type of c != k) loads class c's rows and zeros in the other half.
constexpr int kCpBoth = 0x50, kCpOne = 0x60;
__device__ __forceinline__ void describe_cp(const Params& p, int tile, TileDesc& d) {
  const int i3 = tile % p.n3, r = tile / p.n3, k = r % p.q, cp = r / p.q;
  const int c0 = 2 * cp;
  d.nseg = 0;
  add_seg(d, k * p.bi, p.bi, c0, kCpBoth);
  for (int j = 0; j < 2; ++j) {
    const int t = type_of_class(p, c0 + j);
    if (t != k) add_seg(d, t * p.bi, p.bi, c0 + j, kCpOne | j);
  }
  d.a_f = 0;
  d.a_c1 = 1;
  d.b_f = k * p.bo + i3 * p.wn;
  d.b_c1 = 0;
  d.rbase = 0;
  d.rstride = p.qv;
  d.roff = c0;
  d.rlimit = p.Mq;
  d.cbase = d.b_f;
  d.vlo = 0;
  d.vhi = INT_MAX;
}

// Class-group tile (cg, k, i3): classes c0 = cg * grp ... c0 + grp - 1, output
// group k, 128-column block i3 of it.  Under Q_q every class's rows add
// X_c[., k] W(k, k) (the diagonal term, one segment over all grp classes: B
// is their boxes side by side) and, for type t(c) != k, X_c[., t] W(t, k)
// (one segment per class, into that class's TMEM columns).
__device__ __forceinline__ void describe_grp(const Params& p, int tile, TileDesc& d) {
  const int i3 = tile % p.n3, r = tile / p.n3, k = r % p.q, cg = r / p.q;
  const int c0 = cg * p.grp, wcol0 = k * p.bo + i3 * p.wn;
  d.nseg = 0;
  add_seg(d, k * p.bi, p.bi, c0, p.grp);
  for (int j = 0; j < p.grp; ++j) {
    const int c = c0 + j, t = type_of_class(p, c);
    if (t != k) add_seg(d, t * p.bi, p.bi, c, 1);
  }
  d.a_f = wcol0;
  d.a_c1 = 0;
  d.b_f = 0;
  d.b_c1 = 1;
  d.rbase = 0;
  d.rstride = p.qv;
  d.roff = c0;
  d.rlimit = p.Mq;
  d.cbase = wcol0;
  d.vlo = 0;
  d.vhi = INT_MAX;
}

template <bool kGrp, bool kSplit, bool kRg, bool kCp>
__device__ __forceinline__ void describe(const Params& p, int tile, TileDesc& d) {
  d.split = -1;
  if (kRg) {
    describe_rg(p, tile, d);
    return;
  }
  if (kCp) {
    describe_cp(p, tile, d);
    return;
  }
  if (kGrp && p.grp) {
    describe_grp(p, tile, d);
    return;
  }
  if (p.seg_mode) {
    describe_seg(p, tile, d);
    return;
  }
  int i0, i1, i2, i3, piece = 0;
  if (kSplit && p.ksplit > 1 && tile >= p.split_base) {
    // an extra piece of heavy tile dg
    const int j = tile - p.split_base, dg = j / (p.ksplit - 1);
    piece = 1 + (j - dg * (p.ksplit - 1));
    i3 = dg % p.n3;
    i1 = (dg / p.n3) % p.n1;
    i0 = dg / (p.n3 * p.n1);
    i2 = p.op == OP_DW ? i0 : type_of_class(p, i0);
  } else {
    const int t3 = (int)fdiv((uint32_t)tile, p.div_n3);
    i3 = tile - t3 * p.n3;
    const int pr = (int)fdiv((uint32_t)t3, p.div_n1);
    i1 = t3 - pr * p.n1;
    pair_of(p, pr, i0, i2);
  }
  d.nseg = 0;
  d.rstride = 1;
  d.roff = 0;
  d.rlimit = LLONG_MAX;
  d.vlo = 0;
  d.vhi = INT_MAX;
  if (p.ragged) {  // OP_FWD, not swapped: i0 class, i1 token block, i2 output group k
    // law Q_q: S(t, t) = {t}, S(t, k) = {t, k}; a segment's k0 is the group
    const int c = i0, k = i2, t = type_of_class(p, c);
    d.seg[0].k0 = t < k ? t : k;
    d.seg[1].k0 = t < k ? k : t;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      d.seg[j].len = p.ka;
      d.seg[j].cls = c;
      d.seg[j].map = 0;
    }
    d.nseg = t == k ? 1 : 2;
    const int col0 = k * p.gbo, x0 = col0 & ~15;
    d.a_f = i1 * p.xr;
    d.a_c1 = 1;
    d.b_f = x0;
    d.b_c1 = 0;
    d.rbase = d.a_f;
    d.rstride = p.qv;
    d.roff = c;
    d.rlimit = p.Mq;
    d.cbase = x0;
    d.vlo = col0 - x0;
    d.vhi = d.vlo + p.gbo;
    return;
  }
  switch (p.op) {
    case OP_FWD:
    case OP_SWIGLU: {  // i0 class, i1 token block, i2 output group k, i3 column block
      const int c = i0, k = i2, t = type_of_class(p, c);
      add_members(p, d, t, k, p.bi, c);
      const int xrow0 = i1 * p.xr, wcol0 = k * p.bo + i3 * p.wn;
      if (!p.swap) { d.a_f = xrow0; d.a_c1 = 1; d.b_f = wcol0; d.b_c1 = 0; }
      else { d.a_f = wcol0; d.a_c1 = 0; d.b_f = xrow0; d.b_c1 = 1; }
      d.rbase = xrow0; d.rstride = p.qv; d.roff = c; d.rlimit = p.Mq; d.cbase = wcol0;
      break;
    }
    case OP_SQUARE: {  // i0 row block i, i1 128-row slab, i2 column block k, i3 column slab
      const int i = i0, k = i2;
      add_members(p, d, i, k, p.bi, 0);
      d.a_f = i * p.bi + i1 * 128; d.a_c1 = 0;
      d.b_f = k * p.bo + i3 * p.wn; d.b_c1 = 0;
      d.rbase = d.a_f; d.cbase = d.b_f;
      break;
    }
    case OP_DX: {  // i0 class, i1 token block, i2 input group a, i3 column block of group a
      const int c = i0, a = i2, t = type_of_class(p, c);
      if (p.law == AAL_LAW_Q) {
        // a in S(t, k) for Q_q: a == t (every k: one run over all groups) or k == a
        if (kSplit && a == t && p.ksplit > 1) {
          const int k0 = piece * p.split_len;
          add_seg(d, k0, min(p.split_len, p.q * p.bo - k0), c, 0);
          d.split = ((c * p.n1 + i1) * p.n3 + i3) * p.ksplit + piece;
        } else if (a == t) {
          add_seg(d, 0, p.q * p.bo, c, 0);
        } else {
          add_seg(d, a * p.bo, p.bo, c, 0);
        }
      } else {
        for (int k = 0; k < p.q; ++k)
          if (in_table(p.law, t, k, a)) add_seg(d, k * p.bo, p.bo, c, 0);
      }
      d.a_f = i1 * 128; d.a_c1 = 1;
      d.b_f = a * p.bi + i3 * p.wn; d.b_c1 = 0;
      d.rbase = i1 * 128; d.rstride = p.qv; d.roff = c; d.rlimit = p.Mq;
      d.cbase = d.b_f;
      break;
    }
    case OP_DW: {  // i0 group a, i2 group k; (i1, i3) = (row slab, column block) or swapped
      const int a = i0, k = i2;
      const int mb = p.swap ? i3 : i1, nb = p.swap ? i1 : i3;
      if (kSplit && p.law == AAL_LAW_Q && a == k && p.ksplit > 1) {
        const int k0 = piece * p.split_len;
        add_seg(d, k0, (int)min((long long)p.split_len, p.Mall - k0), 0, 1);
        d.split = ((a * p.n1 + i1) * p.n3 + i3) * p.ksplit + piece;
      } else if (p.law == AAL_LAW_Q && a == k) {
        add_seg(d, 0, (int)p.Mall, 0, 1);  // every type uses the diagonal block
      } else if (p.law == AAL_LAW_Q) {
        // a != k: a in S(t, k) only for t == a, the class whose type is a
        const int c = (a - p.off + p.q) % p.q;
        if (c < p.qv) add_seg(d, 0, (int)p.Mq, c, 0);
      } else {
        for (int c = 0; c < p.qv; ++c)
          if (in_table(p.law, type_of_class(p, c), k, a)) add_seg(d, 0, (int)p.Mq, c, 0);
      }
      const int xf = a * p.bi + (p.swap ? nb * p.wn : mb * 128);
      const int yf = k * p.bo + (p.swap ? mb * 128 : nb * p.wn);
      if (!p.swap) { d.a_f = xf; d.b_f = yf; } else { d.a_f = yf; d.b_f = xf; }
      d.a_c1 = 1; d.b_c1 = 1;
      d.rbase = xf; d.cbase = yf;
      break;
    }
  }
}

__device__ __forceinline__ int seg_chunks(const Seg& s) { return (s.len + 63) >> 6; }

// Tile of schedule slot ``slot`` (slot = CTA + round * grid), or -1 when this
// CTA has no more tiles.
__device__ __forceinline__ int tile_at(const Params& p, int slot) {
  if (!p.use_order) return slot < p.ntiles ? slot : -1;
  if (slot >= p.nslots) return -1;
  const int t = p.order[slot];
  return t == 0xFFFF ? -1 : t;
}

// Copies the description of this role's i-th tile out of the ring and frees
// the slot (WARP: the whole warp reads it and lane 0 arrives).
template <bool WARP>
__device__ __forceinline__ bool take_tile(const TileDesc* ring, uint64_t* full, uint64_t* empty,
                                          uint32_t i, TileDesc& d, volatile int* abort) {
  const uint32_t slot = i % kTileRing, ph = (i / kTileRing) & 1u;
  if (WARP) {
    if (!warp_wait(&full[slot], ph, abort)) return false;
  } else if (!(mbar_try_wait(&full[slot], ph) || mbar_wait(&full[slot], ph, abort))) {
    return false;
  }
  d = ring[slot];
  if (WARP) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[slot]);
  } else {
    mbar_arrive(&empty[slot]);
  }
  return true;
}

// --------------------------------------------------------------- the kernel
// A_MN / B_MN: operand tiles stored MN-major (else K-major).
// DUAL: 0 one MMA per K step; 1 two B operands (gate/up); 2 two A operands;
// 3 two (A, B) pairs summed into one accumulator (the SwiGLU backward's
// dX = dG Wg^T + dU Wu^T).
// PAIR: the tile is computed by a CTA pair with tcgen05 cta_group::2 (M = 256);
// each CTA loads its half of A's rows and of B's columns (for DUAL == 1, CTA r
// loads B operand r), only the pair's first CTA issues MMAs and counts the
// transaction bytes, and each CTA drains its own 128 TMEM lanes.
// MODE: 0 plain; 1 output-group pairs; 2 class pairs (unswapped projection)
template <bool A_MN, bool B_MN, int DUAL, bool PAIR, int MODE = 0>
__global__ void __launch_bounds__(kThreads, 1) k_tc(const __grid_constant__ Params p) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[kMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ __align__(8) uint64_t tile_full[kTileRing];
  __shared__ __align__(8) uint64_t tile_empty[kTileRing];
  __shared__ TileDesc s_tile[kTileRing];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_last_chunk[kMaxStages];  // last K chunk issued into each stage (-1: none)
  __shared__ __align__(8) uint64_t stall_bar;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t smem0 = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int S = p.stages;
  // The optional modes exist only in the instantiations that can meet them:
  // class groups on the swapped forward, split K on dX and dW.  The other
  // instantiations compile without their code.
  constexpr bool kGrp = A_MN && !B_MN && !PAIR && (DUAL == 0 || DUAL == 2);
  constexpr bool kSplit = !PAIR && ((!A_MN && !B_MN && (DUAL == 0 || DUAL == 3)) || (A_MN && B_MN && DUAL == 0));
  constexpr bool kRg = MODE == 1 && !A_MN && B_MN && (DUAL == 0 || DUAL == 1) && !PAIR;  // output-group pairs
  constexpr bool kCp = MODE == 2 && !A_MN && B_MN && DUAL == 0 && !PAIR;  // class pairs
  const bool grp = kGrp && p.grp;
  // Programmatic dependent launch: the next kernel of the stream may start
  // its own set-up on SMs this grid has left; it reads nothing of ours before
  // its griddepcontrol.wait, which returns once this grid has completed.
  asm volatile("griddepcontrol.launch_dependents;");
  // start fetching the tensor maps in use while the barriers are set up
  if (warp == kSchedWarp && lane < 5 && ((p.map_mask >> lane) & 1)) {
    const CUtensorMap* m = lane < 2 ? &p.mapA[lane] : (lane < 4 ? &p.mapB[lane - 2] : &p.mapOut);
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<unsigned long long>(m)) : "memory");
  }
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool issuer = !PAIR || rank == 0;
  const int tile0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tstep = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int nprod = S < kProdWarps ? S : kProdWarps;  // producer warps in use

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], (PAIR ? 2 : 1) * kEpiWarps);
    }
    mbar_init(&done_bar, 1);
    mbar_init(&stall_bar, 1);
    for (int s = 0; s < kMaxStages; ++s) s_last_chunk[s] = -1;
    // a ring slot is free again once every consuming warp has copied it: the
    // producer warps in use, the MMA thread (where this CTA issues) and the
    // epilogue warps
    for (int r = 0; r < kTileRing; ++r) {
      mbar_init(&tile_full[r], 1);
      mbar_init(&tile_empty[r], nprod + (issuer ? 1 : 0) + kEpiWarps);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    if (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&s_tmem)),
                   "r"(p.tmem_cols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&s_tmem)),
                   "r"(p.tmem_cols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // Everything above touches only this CTA's shared memory, TMEM and its
  // parameters; global memory (inputs a previous kernel of the stream writes,
  // outputs it may still read) is used only after the previous grid is done.
  // The tile decoder reads only parameters and shared memory (outside segment
  // mode, whose tables are device data), so it describes the first tiles
  // while a previous grid may still run.
  if (warp != kSchedWarp || p.seg_mode) asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0 || (warp >= 2 + kEpiWarps && warp < kSchedWarp)) {
    // ------------------------------------------------------ TMA producers
    // Every producer warp walks the same chunk sequence and issues the chunks
    // i with i mod nprod == its index.  With nprod <= S a warp waiting for
    // stage i mod S to empty cannot mistake an older phase for the one it
    // needs: its previous chunk i - nprod already saw chunk i - nprod - S
    // released, and the MMAs release stages in order.
    const int pw = warp == 0 ? 0 : warp - (1 + kEpiWarps);
    uint32_t it = 0, st = 0, ph = 0, ti = 0;
    bool ok = pw < nprod;
    for (; ok; ++ti) {
      TileDesc d;
      if (!take_tile<true>(s_tile, tile_full, tile_empty, ti, d, &s_abort)) break;
      if (d.nseg < 0) break;  // the decoder's end mark
      for (int s = 0; s < d.nseg && ok; ++s) {
        const Seg sg = seg_at(d, s);
        const int nch = seg_chunks(sg);
        for (int kc = 0; kc < nch; ++kc) {
          const bool mine = (int)(it % (uint32_t)nprod) == pw;
          if (mine && !warp_wait(&empty_bar[st], ph ^ 1u, &s_abort)) { ok = false; break; }
          if (mine) {
            // The boxes of a stage are issued by separate lanes: one thread
            // issuing them back to back serialises the TMA requests.
            const uint32_t base = smem0 + st * p.stage_bytes;
            const int kofs = sg.k0 + kc * 64;
            const uint32_t fb = PAIR ? mapa_rank(smem_u32(&full_bar[st]), 0) : smem_u32(&full_bar[st]);
            if (lane == 0 && issuer) {
              // class-group mode: the segment's classes' B boxes (sg.map of them)
              const uint32_t tx =
                  grp ? (uint32_t)(DUAL >= 2 ? 2 : 1) * p.a_bytes + (uint32_t)sg.map * p.box_bytes
                      : kRg ? p.a_bytes + (uint32_t)(sg.map == kRgWide ? 2 : 1) * (uint32_t)p.rg_n * 128u *
                                            (DUAL == 1 ? 2u : 1u)
                            : (PAIR ? 2u : 1u) * p.tx_bytes;
              mbar_expect_tx(&full_bar[st], tx);
            }
            if (lane == 0) atomicMax(&s_last_chunk[st], (int)it);
            if (!A_MN && B_MN && DUAL == 0 && !PAIR && p.ragged) {
              // lane 0: the A box; lane 1: the B box (all atoms, ka rows from -oa)
              const int a = sg.k0, oa = (a * p.gbi) & 7;
              if (lane == 0)
                tma_load(&p.mapA[0], base, &full_bar[st], a * p.gbi - oa, d.a_c1 ? sg.cls : 0, d.a_f);
              else if (lane == 1)
                tma_load4(&p.mapB[0], base + p.a_bytes, &full_bar[st], 0, -oa, a, d.b_f >> 4);
            } else {
            const int na = DUAL >= 2 ? 2 : 1;
            const int nb = ((DUAL == 1 && !PAIR) || DUAL == 3) ? 2 : 1;
            const int nA = kCp ? 2 : (A_MN && !p.a_merged) ? p.a_rows / p.a_aw : 1;  // boxes per A operand
            const int nB = grp ? sg.map
                           : kRg ? (sg.map == kRgWide ? 2 * p.rg_n : p.rg_n) / p.b_aw
                                 : ((B_MN && !p.b_merged) ? p.b_rows / p.b_aw : 1);  // boxes per B operand
            const int arow = PAIR ? (int)rank * 128 : 0;  // this CTA's half of the A tile
            const int bsh = (PAIR && DUAL != 1) ? (int)rank * p.b_rows : 0;
            for (int bx = lane; bx < na * nA + nb * nB; bx += 32) {
              if (bx < na * nA) {
                const int o = bx / nA, at = bx - o * nA;
                // (sg.map counts the classes of a class-group segment, not a map)
                const CUtensorMap* m = &p.mapA[DUAL >= 2 ? o : ((grp || kRg || kCp) ? 0 : sg.map)];
                // class pairs: box at = class c0 + at's 64 rows; a one-class segment
                // reads rows past the end (zeros) for the other class
                const bool cp_zero = kCp && sg.map != kCpBoth && at != (sg.map & 1);
                const int c1 = kCp ? d.roff + at : (d.a_c1 ? sg.cls : 0);
                const uint32_t dst = base + o * p.a_bytes + (A_MN ? at * (p.a_aw * 2 * 64) : 0) +
                                     (kCp ? at * 64 * 128 : 0);
                if (A_MN && p.a_merged) {
                  // all atoms at once: coordinates (col in atom, class, K row, atom)
                  const int x3 = (d.a_f + arow) / p.a_aw;
                  if (PAIR) tma_load4_pair(m, dst, fb, 0, c1, kofs, x3);
                  else tma_load4(m, dst, &full_bar[st], 0, c1, kofs, x3);
                } else {
                  const int x0 = A_MN ? d.a_f + arow + at * p.a_aw : kofs;
                  const int x2 = A_MN ? kofs : (cp_zero ? 64 : d.a_f + arow);
                  if (PAIR) tma_load_pair(m, dst, fb, x0, c1, x2);
                  else tma_load(m, dst, &full_bar[st], x0, c1, x2);
                }
              } else {
                // B: for a pair, CTA r holds columns [r*b_rows, (r+1)*b_rows) of
                // the MMA's B, or, with two B operands, all of operand r
                const int jb = bx - na * nA, o = jb / nB, at = jb - o * nB;
                const int mop = DUAL == 1 ? (PAIR ? (int)rank : o) : (DUAL == 3 ? o : ((grp || kRg || kCp) ? 0 : sg.map));
                const CUtensorMap* m = &p.mapB[mop];
                const int c1 = (d.b_c1 ? sg.cls : 0) + (grp ? at : 0);
                const uint32_t dst = base + na * p.a_bytes + o * p.b_bytes +
                                     (B_MN ? at * (p.b_aw * 2 * 64) : 0) + (grp ? at * p.box_bytes : 0);
                if (B_MN && p.b_merged) {
                  const int x3 = (d.b_f + bsh) / p.b_aw;
                  if (PAIR) tma_load4_pair(m, dst, fb, 0, c1, kofs, x3);
                  else tma_load4(m, dst, &full_bar[st], 0, c1, kofs, x3);
                } else {
                  // output-group pairs: a diagonal segment's columns are group j's
                  const int rgo = (kRg && sg.map != kRgWide) ? (sg.map & 1) * p.rg_n : 0;
                  const int x0 = B_MN ? d.b_f + bsh + at * p.b_aw + rgo : kofs;
                  const int x2 = B_MN ? kofs : d.b_f + bsh;
                  if (PAIR) tma_load_pair(m, dst, fb, x0, c1, x2);
                  else tma_load(m, dst, &full_bar[st], x0, c1, x2);
                }
              }
            }
            }
          }
          __syncwarp();
          ++it;
          if (++st == (uint32_t)S) { st = 0; ph ^= 1u; }
        }
      }
    }
    // Let every copy this CTA issued land before the CTA can exit (for a pair
    // the pair's first CTA sees both halves on its own barriers).  The chunks
    // issued into a stage always form a prefix of that stage's phases: chunk
    // i + S can only be issued after chunk i was consumed, so on the abort
    // path a chunk that was never issued stops its stage for good.  Waiting
    // for the phase of the last chunk actually issued into each stage (across
    // the four producer warps) therefore covers every copy in flight, on the
    // normal path and after an abort alike.
    __syncwarp();
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kProdWarps) : "memory");
    if (warp == 0 && lane == 0 && issuer) {
      for (int st = 0; st < S; ++st) {
        const int last = s_last_chunk[st];
        if (last >= 0) mbar_wait_teardown(&full_bar[st], ((uint32_t)last / (uint32_t)S) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (issuer && lane == 0) {
      // One thread issues; a running stage index and phase bit replace
      // divisions, so the next MMAs follow the previous ones closely.
      uint32_t st = 0, ph = 0, tl = 0;
      bool ok = true;
      const int na = DUAL >= 2 ? 2 : 1;
      // Descriptors of stage 0 and their per-stage and per-K-step increments,
      // built once: the issue loop below only adds.
      const bool rg = !A_MN && B_MN && DUAL == 0 && !PAIR && p.ragged;
      const uint64_t dA0 = rg ? make_desc(smem0, 16, 16u * p.ka, p.ka == 32 ? kLayoutSW64 : kLayoutSW128)
                              : operand_desc0<A_MN>(smem0, p.a_aw);
      const uint64_t dA1 = operand_desc0<A_MN>(smem0 + p.a_bytes, p.a_aw);
      const uint64_t dB0 = rg ? make_desc(smem0 + p.a_bytes, p.b_lbo, 8 * 32, kLayoutSW32)
                              : operand_desc0<B_MN>(smem0 + na * p.a_bytes, p.b_aw);
      const uint64_t dB1 = operand_desc0<B_MN>(smem0 + na * p.a_bytes + p.b_bytes, p.b_aw);
      const uint64_t dstage = p.stage_bytes >> 4;
      const uint64_t kA = operand_kstep<A_MN>(p.a_aw), kB = operand_kstep<B_MN>(p.b_aw);
      const uint32_t idesc = (PAIR ? (DUAL == 1 ? p.idesc2 : p.idesc)
                                   : ((DUAL == 1 && p.fuse_b) ? p.idesc2 : p.idesc));
      const bool single = PAIR || DUAL == 0 || (DUAL == 1 && p.fuse_b);
      uint64_t so = 0;  // dstage * st
      // test hook: a wait nothing ends, bounded by kStallNs; it records the
      // timeout and aborts the kernel before the first MMA
      if (p.test_stall && !mbar_wait(&stall_bar, 0, &s_abort, kStallNs)) ok = false;
      for (; ok; ++tl) {
        TileDesc d;
        if (!take_tile<false>(s_tile, tile_full, tile_empty, tl, d, &s_abort)) break;
        if (d.nseg < 0) break;
        const uint32_t buf = tl & 1u, use = tl >> 1;
        if (!(mbar_try_wait(&tempty_bar[buf], (use & 1u) ^ 1u) ||
              mbar_wait(&tempty_bar[buf], (use & 1u) ^ 1u, &s_abort))) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc0 = tmem + buf * p.acc_cols;
        const uint32_t acc1 = acc0 + p.n_mma;
        uint32_t accumulate = 0;
        for (int s = 0; s < d.nseg && ok; ++s) {
          const Seg sgm = seg_at(d, s);
          const int len = sgm.len;
          // class-group mode: a one-class segment writes its class's TMEM
          // columns with an N = grp_n MMA; the diagonal segment spans them all
          uint32_t aoff = 0, id0 = idesc, id1 = p.idesc;
          if (grp && sgm.map == 1) {
            aoff = (uint32_t)(sgm.cls - d.roff) * (uint32_t)p.grp_n;
            id0 = id1 = p.idesc_one;
          }
          if (kRg && sgm.map != kRgWide) {
            aoff = (uint32_t)(sgm.map & 1) * (uint32_t)p.rg_n;
            id0 = id1 = p.idesc_one;
          }
          const uint32_t accA = acc0 + aoff, accB = acc1 + aoff;
          for (int rem = len; rem > 0; rem -= 64) {
            if (!(mbar_try_wait(&full_bar[st], ph) || mbar_wait(&full_bar[st], ph, &s_abort))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t a0 = dA0 + so, b0 = dB0 + so;
            const uint64_t a1 = dA1 + so, b1 = dB1 + so;
            if (rem >= 64) {
              // the common full chunk: four K steps, unrolled
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                if (PAIR) {
                  tc_mma_pair(acc0, a0 + ks * kA, b0 + ks * kB, idesc, accumulate);
                } else if (single) {
                  tc_mma(accA, a0 + ks * kA, b0 + ks * kB, id0, accumulate);
                } else {
                  tc_mma(accA, a0 + ks * kA, b0 + ks * kB, id1, accumulate);
                  if (DUAL == 1) tc_mma(accB, a0 + ks * kA, b1 + ks * kB, id1, accumulate);
                  if (DUAL == 2) tc_mma(accB, a1 + ks * kA, b0 + ks * kB, id1, accumulate);
                  if (DUAL == 3) tc_mma(accA, a1 + ks * kA, b1 + ks * kB, id1, 1u);
                }
                accumulate = 1;
              }
            } else {
              const int ksteps = (rem + 15) >> 4;
              for (int ks = 0; ks < ksteps; ++ks) {
                const uint64_t da = a0 + ks * kA, db = b0 + ks * kB;
                if (PAIR) {
                  tc_mma_pair(acc0, da, db, idesc, accumulate);
                } else if (single) {
                  tc_mma(accA, da, db, id0, accumulate);
                } else {
                  tc_mma(accA, da, db, id1, accumulate);
                  if (DUAL == 1) tc_mma(accB, da, b1 + ks * kB, id1, accumulate);
                  if (DUAL == 2) tc_mma(accB, a1 + ks * kA, db, id1, accumulate);
                  if (DUAL == 3) tc_mma(accA, a1 + ks * kA, b1 + ks * kB, id1, 1u);
                }
                accumulate = 1;
              }
            }
            // frees the stage (in both CTAs of a pair) once these MMAs have read it
            if (PAIR) tc_commit_pair_mc(&empty_bar[st]);
            else tc_commit(&empty_bar[st]);
            if (++st == (uint32_t)S) { st = 0; ph ^= 1u; so = 0; }
            else so += dstage;
          }
        }
        if (!ok) break;
        if (PAIR) tc_commit_pair_mc(&tfull_bar[buf]);
        else tc_commit(&tfull_bar[buf]);
      }
      // wait for every MMA this CTA issued before TMEM is released
      if (PAIR) tc_commit_pair_mc(&done_bar);
      else tc_commit(&done_bar);
      mbar_wait_teardown(&done_bar, 0);
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------ epilogue
    const int quarter = warp & 3;             // TMEM lanes this warp may read
    const int half = (warp - 2) / 4;          // which of the 16-column chunks it drains
    const int row_in_tile = quarter * 32 + lane;
    // two 1 KB TMA-store staging buffers per epilogue warp, after the pipeline stages
    const uint32_t stage_buf = smem0 + S * p.stage_bytes + (warp - 2) * 2048;
    uint32_t nstore = 0;
    uint32_t tl = 0;
    const int erow = PAIR ? (int)rank * 128 : 0;  // this CTA's 128 rows of the pair's tile
    for (;; ++tl) {
      TileDesc d;
      if (!take_tile<true>(s_tile, tile_full, tile_empty, tl, d, &s_abort)) break;
      if (d.nseg < 0) break;
      d.rbase += erow;
      const uint32_t buf = tl & 1u, use = tl >> 1;
      if (!warp_wait(&tfull_bar[buf], use & 1u, &s_abort)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * p.acc_cols;
      // segment mode: the caller's row of this thread's TMEM lane, looked up
      // once per tile (its load overlaps the first TMEM read)
      int seg_row = 0;
      if (p.seg_mode && !p.swap && d.rbase + row_in_tile < d.rlimit) seg_row = p.seg_perm[d.rbase + row_in_tile];
      const uint32_t tempty_addr =
          PAIR ? mapa_rank(smem_u32(&tempty_bar[buf]), 0) : smem_u32(&tempty_bar[buf]);
      const int nch = (p.n_mma / 16 + 1 - half) / 2;  // chunks c0 = half*16 + 32*i
      for (int ci = 0; ci < nch; ++ci) {
        const int c0 = half * 16 + 32 * ci;
        float v[16];
        tmem_ld16(tbase + c0, v);
        if (p.swiglu) {
          float u[16];
          tmem_ld16(tbase + p.n_mma + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            // silu(g) * u = g / (1 + e^-g) * u with the fast exponential and
            // division intrinsics (a correctly rounded reciprocal costs a
            // multi-instruction sequence per element); for g below about -88
            // e^-g is inf and the quotient is 0
            v[j] = __fdividef(v[j], 1.0f + __expf(-v[j])) * u[j];
          }
        } else {
          tmem_wait_ld();
        }
        if (ci == nch - 1) {
          // the accumulator is in registers: hand the TMEM buffer back early
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (PAIR) mbar_arrive_remote(tempty_addr);
            else mbar_arrive(&tempty_bar[buf]);
          }
        }
        if (kSplit && p.ksplit > 1 && d.split >= 0) {
          // a piece of a split tile: its fp32 partial, TMEM lane by column
          float4* dst = reinterpret_cast<float4*>(
              p.split_ws + ((size_t)d.split * 128 + row_in_tile) * p.n_mma + c0);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          continue;
        }
        if (p.tma_store && (c0 < d.vlo || c0 + 16 > d.vhi)) {
          // ragged mode: a chunk at or past the edge of the group's columns;
          // its columns inside the group go out as 8-byte stores (4 columns,
          // when the edges fall on multiples of 4) or one by one
          const long long x = d.rbase + row_in_tile;
          if (!p.swap && x < d.rlimit && c0 + 16 > d.vlo && c0 < d.vhi) {
            __nv_bfloat16* dst = p.out + (x * d.rstride + d.roff) * p.ldo + d.cbase + c0;
            if (((d.vlo | d.vhi) & 3) == 0) {
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                if (c0 + 4 * g >= d.vlo && c0 + 4 * g + 4 <= d.vhi) {
                  uint2 w;
                  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&w);
                  h[0] = __floats2bfloat162_rn(v[4 * g], v[4 * g + 1]);
                  h[1] = __floats2bfloat162_rn(v[4 * g + 2], v[4 * g + 3]);
                  *reinterpret_cast<uint2*>(dst + 4 * g) = w;
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (c0 + j >= d.vlo && c0 + j < d.vhi) dst[j] = __float2bfloat16_rn(v[j]);
            }
          }
        } else if (p.tma_store) {
          const uint32_t sb = stage_buf + (nstore & 1u) * 1024;
          if (nstore >= 2) {
            if (lane == 0) bulk_wait_read1();  // the buffer's previous store has read it
            __syncwarp();
          }
          if (!p.swap) {
            // 32 rows x 16 columns, 32-byte rows, 32-byte swizzle
            uint4 w[2];
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(w);
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            const uint32_t row = sb + lane * 32;
            const uint32_t flip = (lane >> 2) & 1u;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((0u ^ flip) << 4)),
                         "r"(w[0].x), "r"(w[0].y), "r"(w[0].z), "r"(w[0].w));
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((1u ^ flip) << 4)),
                         "r"(w[1].x), "r"(w[1].y), "r"(w[1].z), "r"(w[1].w));
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              // class pairs: TMEM lanes 0-63 are class roff's rows, 64-127 the next class's
              if (kCp)
                tma_store(&p.mapOut, sb, (int)(d.cbase + c0), d.roff + (quarter >> 1),
                          (int)(d.rbase + (quarter & 1) * 32));
              else
                tma_store(&p.mapOut, sb, (int)(d.cbase + c0), d.roff,
                          (int)(d.rbase + quarter * 32));
              bulk_commit();
            }
          } else {
            // 16 rows x 32 columns (this warp's 32 TMEM lanes), 64-byte rows
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const __nv_bfloat16 hv = __float2bfloat16_rn(v[j]);
              asm volatile("st.shared.b16 [%0], %1;" ::"r"(sb + j * 64 + lane * 2),
                           "h"(*reinterpret_cast<const unsigned short*>(&hv)));
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              // class-group mode: TMEM columns run class by class, grp_n each
              const int gj = grp ? c0 / p.grp_n : 0, gt = grp ? c0 - gj * p.grp_n : c0;
              tma_store(&p.mapOut, sb, (int)(d.cbase + quarter * 32), d.roff + gj,
                        (int)(d.rbase + gt));
              bulk_commit();
            }
          }
          ++nstore;
        } else if (!p.swap) {
          const long long x = d.rbase + row_in_tile;
          // the SiLU' chain exists only in the dX instantiation (K-major A and B, one B)
          constexpr bool kDxKernel = !A_MN && !B_MN && DUAL == 0 && !PAIR;
          if (kDxKernel && x < d.rlimit && p.swiglu_bwd) {
            // SiLU' chain of the SwiGLU backward on the dH tile in registers
            const long long off = (x * d.rstride + d.roff) * p.ldo + d.cbase + c0;
            const uint4 g0 = reinterpret_cast<const uint4*>(p.g_in + off)[0];
            const uint4 g1 = reinterpret_cast<const uint4*>(p.g_in + off)[1];
            const uint4 u0 = reinterpret_cast<const uint4*>(p.u_in + off)[0];
            const uint4 u1 = reinterpret_cast<const uint4*>(p.u_in + off)[1];
            const __nv_bfloat16* gb0 = reinterpret_cast<const __nv_bfloat16*>(&g0);
            const __nv_bfloat16* gb1 = reinterpret_cast<const __nv_bfloat16*>(&g1);
            const __nv_bfloat16* ub0 = reinterpret_cast<const __nv_bfloat16*>(&u0);
            const __nv_bfloat16* ub1 = reinterpret_cast<const __nv_bfloat16*>(&u1);
            float du[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g = __bfloat162float(j < 8 ? gb0[j] : gb1[j - 8]);
              const float u = __bfloat162float(j < 8 ? ub0[j] : ub1[j - 8]);
              const float sg = __fdividef(1.0f, 1.0f + __expf(-g));  // sigmoid(g)
              du[j] = v[j] * g * sg;                                  // dH silu(g)
              v[j] = v[j] * u * sg * (1.0f + g * (1.0f - sg));        // dH u silu'(g)
            }
            uint4 w[2];
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(w);
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            reinterpret_cast<uint4*>(p.out + off)[0] = w[0];
            reinterpret_cast<uint4*>(p.out + off)[1] = w[1];
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = __floats2bfloat162_rn(du[2 * j], du[2 * j + 1]);
            reinterpret_cast<uint4*>(p.out2 + off)[0] = w[0];
            reinterpret_cast<uint4*>(p.out2 + off)[1] = w[1];
          } else if (x < d.rlimit) {
            const long long xo = p.seg_mode ? (long long)seg_row : x * d.rstride + d.roff;
            __nv_bfloat16* dst = p.out + xo * p.ldo + d.cbase + c0;
            if (p.accumulate) {
              uint4 o0 = reinterpret_cast<const uint4*>(dst)[0];
              uint4 o1 = reinterpret_cast<const uint4*>(dst)[1];
              const __nv_bfloat16* ob0 = reinterpret_cast<const __nv_bfloat16*>(&o0);
              const __nv_bfloat16* ob1 = reinterpret_cast<const __nv_bfloat16*>(&o1);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                v[j] += __bfloat162float(ob0[j]);
                v[8 + j] += __bfloat162float(ob1[j]);
              }
            }
            uint4 w[2];
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(w);
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            reinterpret_cast<uint4*>(dst)[0] = w[0];
            reinterpret_cast<uint4*>(dst)[1] = w[1];
            if (p.seg_copy) {
              uint4* cp = reinterpret_cast<uint4*>(p.seg_copy + x * p.ld_copy + d.cbase + c0);
              cp[0] = w[0];
              cp[1] = w[1];
            }
          }
        } else {
          const long long col = d.cbase + row_in_tile;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const long long x = d.rbase + c0 + j;
            if (x < d.rlimit) {
              __nv_bfloat16* dst = p.out + (x * d.rstride + d.roff) * p.ldo + col;
              float val = v[j];
              if (p.accumulate) val += __bfloat162float(*dst);
              *dst = __float2bfloat16_rn(val);
            }
          }
        }
      }
      if (nch == 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_remote(tempty_addr);
          else mbar_arrive(&tempty_bar[buf]);
        }
      }
    }
    // every TMA store of this warp must have finished before the CTA exits
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else if (warp == kSchedWarp) {
    // ------------------------------------------------------ tile decoder
    // The only role that walks the schedule: the others take descriptions
    // from the ring until the end mark (nseg = -1) that follows the last tile.
    if (lane == 0) {
      uint32_t i = 0;
      for (int ss = tile0; ; ss += tstep, ++i) {
        int tile;
        if (p.dyn_slot >= 0) {
          // the first tile is this CTA's own; later ones come from the counter
          const unsigned int t =
              i == 0 ? (unsigned)tile0 : gridDim.x + atomicAdd(&g_tile_ctr[p.dyn_slot][0], 1u);
          tile = t < (unsigned)p.ntiles ? (int)t : -1;
        } else {
          tile = tile_at(p, ss);
        }
        const uint32_t slot = i % kTileRing, ph = (i / kTileRing) & 1u;
        if (!(mbar_try_wait(&tile_empty[slot], ph ^ 1u) ||
              mbar_wait(&tile_empty[slot], ph ^ 1u, &s_abort)))
          break;
        TileDesc d;
        if (tile >= 0) describe<kGrp, kSplit, kRg, kCp>(p, tile, d);
        else d.nseg = -1;
        s_tile[slot] = d;
        mbar_arrive(&tile_full[slot]);  // release: the copy above is visible first
        if (tile < 0) break;
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // a pair stays resident until the peer is done with its shared memory and TMEM
  if (PAIR) cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    if (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(p.tmem_cols));
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(p.tmem_cols));
  }
  if (p.dyn_slot >= 0 && threadIdx.x == 0) {
    // every CTA has stopped taking tiles once it gets here: the last one to
    // arrive leaves the pair at zero for the slot's next launch
    if (atomicAdd(&g_tile_ctr[p.dyn_slot][1], 1u) == gridDim.x - 1) {
      atomicExch(&g_tile_ctr[p.dyn_slot][0], 0u);
      atomicExch(&g_tile_ctr[p.dyn_slot][1], 0u);
    }
  }
}

// ------------------------------------------------------------ host planning
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

// A row-major bf16 matrix [rows, cols] (leading dimension ld) seen as
// [rows/qv][qv][cols]; box {box0 elements, 1, box2 rows}.
static bool make_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld,
                     int qv, int box0, int box2, int swizzle_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rows % qv) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)qv, (cuuint64_t)(rows / qv)};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(ld * 2 * qv)};
  cuuint32_t box[3] = {(cuuint32_t)box0, 1u, (cuuint32_t)box2};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// K-major operand tile: box {64 K elements, 1, rows}.
static bool map_kmajor(CUtensorMap* m, const aal_mat& t, int qv, int rows_box) {
  return make_map(m, t.ptr, t.rows, t.cols, t.ld, qv, 64, rows_box, 128);
}
// MN-major operand tile: box {atom width, 1, 64 K rows}.
static bool map_mnmajor(CUtensorMap* m, const aal_mat& t, int qv, int aw) {
  return make_map(m, t.ptr, t.rows, t.cols, t.ld, qv, aw, 64, aw == 64 ? 128 : 32);
}
// MN-major operand tile in one box: the matrix seen as
// [cols/aw][rows/qv][qv][aw] (atom index outermost), box {aw, 1, 64, natoms};
// shared memory then holds the atoms one after another, as the MMA reads them.
static bool map_mnmajor_merged(CUtensorMap* m, const aal_mat& t, int qv, int aw, int natoms) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || t.rows % qv || t.cols % aw || natoms < 1 || natoms > 256) return false;
  cuuint64_t dims[4] = {(cuuint64_t)aw, (cuuint64_t)qv, (cuuint64_t)(t.rows / qv),
                        (cuuint64_t)(t.cols / aw)};
  cuuint64_t strides[3] = {(cuuint64_t)(t.ld * 2), (cuuint64_t)(t.ld * 2 * qv),
                           (cuuint64_t)(aw * 2)};
  cuuint32_t box[4] = {(cuuint32_t)aw, 1u, 64u, (cuuint32_t)natoms};
  cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  const CUresult r =
      enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.ptr), dims, strides, box, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, aw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
// Builds the one-box map when the encoder accepts it, else the per-atom map.
static bool map_mn(CUtensorMap* m, const aal_mat& t, int qv, int aw, int extent, int* merged) {
  if (map_mnmajor_merged(m, t, qv, aw, extent / aw)) { *merged = 1; return true; }
  *merged = 0;
  return map_mnmajor(m, t, qv, aw);
}

// Ragged mode: W [din, dout] seen as [dout / 16 atoms][din / gbi groups]
// [gbi rows][16 columns]; one box {16 columns, ka rows, 1 group, natoms}
// lands in shared memory as the MN-major atoms the MMA reads (ka rows of 32
// bytes each, 32-byte swizzle).  ka exceeds gbi: rows past the group, and
// rows before it when the box starts at a negative row, read as zeros.
static bool map_ragged_w(CUtensorMap* m, const aal_mat& w, int gbi, int ka, int natoms) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || w.rows % gbi || w.cols % 16) return false;
  cuuint64_t dims[4] = {16u, (cuuint64_t)gbi, (cuuint64_t)(w.rows / gbi), (cuuint64_t)(w.cols / 16)};
  cuuint64_t strides[3] = {(cuuint64_t)(w.ld * 2), (cuuint64_t)(w.ld * 2 * gbi), 32u};
  cuuint32_t box[4] = {16u, (cuuint32_t)ka, 1u, (cuuint32_t)natoms};
  cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, w.ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map for the TMA-store epilogue: 32 rows x 16 columns per store
// (32-byte swizzle), or 16 rows x 32 columns when TMEM lanes are columns.
static bool out_map(Params& p, const aal_mat& out, int qv) {
  p.tma_store = (p.accumulate || p.swiglu_bwd || p.seg_mode) ? 0 : 1;
  if (!p.tma_store) return true;
  if (p.swap) return make_map(&p.mapOut, out.ptr, out.rows, out.cols, out.ld, qv, 32, 16, 0);
  return make_map(&p.mapOut, out.ptr, out.rows, out.cols, out.ld, qv, 16, 32, 32);
}

static bool tc_aligned(const aal_mat& m) {
  return m.dtype == AAL_BF16 && ((uintptr_t)m.ptr % 16) == 0 && (m.ld % 8) == 0;
}

// Largest N <= cap with ext % N == 0 and N % 16 == 0, preferring multiples of 64.
static int pick_n(long long ext, int cap) {
  int best = 0;
  for (int n = cap; n >= 16; n -= 16) {
    if (ext % n) continue;
    if (n % 64 == 0) return n;
    if (!best) best = n;
  }
  return best;
}

static uint32_t make_idesc(int m, int n, bool a_mn, bool b_mn) {
  uint32_t d = 0;
  d |= 1u << 4;   // D format: f32
  d |= 1u << 7;   // A format: bf16
  d |= 1u << 10;  // B format: bf16
  d |= (a_mn ? 1u : 0u) << 15;
  d |= (b_mn ? 1u : 0u) << 16;
  d |= (uint32_t)(n >> 3) << 17;
  d |= (uint32_t)(m >> 4) << 24;
  return d;
}

// SM share of the launches this thread makes while it is set (0: all SMs):
// two launches that run side by side on two streams take half of the GPU each.
static thread_local int t_sm_share = 0;

static int all_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

static int num_sms() {
  const int n = all_sms();
  return (t_sm_share > 0 && t_sm_share < n) ? t_sm_share : n;
}

static bool is_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10;
}

// Fills the pipeline sizes and TMEM allocation; false if they do not fit.
static bool finish_plan(Params& p, int dual, bool pair = false) {
  const int na = dual >= 2 ? 2 : 1, nb = ((dual == 1 && !pair) || dual == 3) ? 2 : 1;
  p.a_bytes = (uint32_t)p.a_rows * 128u;
  p.b_bytes = (uint32_t)p.b_rows * 128u;
  p.stage_bytes = na * p.a_bytes + nb * p.b_bytes;
  if (p.ragged) {
    // A: 128 rows of ka features; B: the atoms of 16 columns x ka rows.  The
    // stride between stages stays a multiple of 1 KB (swizzle alignment).
    p.a_bytes = 128u * (uint32_t)p.ka * 2u;
    p.b_lbo = (uint32_t)p.ka * 32u;
    p.b_bytes = (uint32_t)(p.n_mma / 16) * p.b_lbo;
    p.tx_bytes = p.a_bytes + p.b_bytes;
    p.stage_bytes = (p.tx_bytes + 1023u) & ~1023u;
  } else {
    p.tx_bytes = p.stage_bytes;
  }
  p.stages = (kSmemBudget - kEpiSmem) / (int)p.stage_bytes;
  if (p.stages > kMaxStages) p.stages = kMaxStages;
  if (p.stages < 2) return false;
  p.acc_cols = p.n_mma * ((dual == 1 || dual == 2) ? 2 : 1);
  const int need = 2 * p.acc_cols;
  if (need > 512) return false;
  uint32_t cols = 32;
  while ((int)cols < need) cols <<= 1;
  p.tmem_cols = cols;
  p.ntiles = 0;
  return true;
}

// Block products behind the tile pair (p0, p1) of the op: the table-entry size
// for the forward ops, the number of k (dX) or classes (dW) that use a block.
static int pair_cost(const Params& p, int p0, int p1) {
  int mem[4];
  switch (p.op) {
    case OP_FWD:
    case OP_SWIGLU: return table_members(p.law, p.q, (p0 + p.off) % p.q, p1, mem);
    case OP_SQUARE: return table_members(p.law, p.q, p0, p1, mem);
    case OP_DX: {
      int n = 0;
      for (int k = 0; k < p.q; ++k) n += in_table(p.law, (p0 + p.off) % p.q, k, p1) ? 1 : 0;
      return n;
    }
    default: {
      if (p.law == AAL_LAW_Q && p0 == p1) return p.q;
      int n = 0;
      for (int c = 0; c < p.qv; ++c) n += in_table(p.law, (c + p.off) % p.q, p1, p0) ? 1 : 0;
      return n;
    }
  }
}

// Orders the q*q tile pairs longest first.
static void order_pairs(Params& p) {
  const int q = p.q;
  if (q * q <= kMaxPairs && q <= 256) {
    int n = 0;
    for (int cost = 4 * q; cost >= 0; --cost)
      for (int p0 = 0; p0 < q; ++p0)
        for (int p1 = 0; p1 < q; ++p1)
          if (pair_cost(p, p0, p1) == cost) p.pairs[n++] = (uint16_t)(p0 << 8 | p1);
    p.npairs_list = n;
  } else {
    p.npairs_list = 0;
    p.diag_first = (p.op == OP_DX || p.op == OP_DW) ? 1 : 0;
  }
}

// Host copy of pair_of (the pair of tile-pair rank ``pr``).
static void host_pair_of(const Params& p, int pr, int& p0, int& p1) {
  if (p.npairs_list) {
    p0 = p.pairs[pr] >> 8;
    p1 = p.pairs[pr] & 255;
    return;
  }
  const int q = p.q, nd = q * (q - 1);
  auto diag = [&](int a) {
    if (p.op == OP_SQUARE || p.op == OP_DW) return a;
    const int t = a + p.off;
    return t >= q ? t - q : t;
  };
  int r = pr;
  if (p.diag_first) {
    if (r < q) { p0 = r; p1 = diag(r); return; }
    r -= q;
  } else if (r >= nd) {
    p0 = r - nd;
    p1 = diag(p0);
    return;
  }
  p0 = r / (q - 1);
  const int j = r % (q - 1), dg = diag(p0);
  p1 = j < dg ? j : j + 1;
}

// Balances the tiles over ``grid`` CTAs: tiles by decreasing cost (the number
// of K segments of their table entry; every segment of an op has the same
// length), each onto the CTA with the least work so far.  Leaves the stride
// order when the schedule would not fit.
static void schedule_tiles(Params& p, int grid) {
  p.use_order = 0;
  const int nt = p.ntiles;
  if (grid <= 0 || nt <= grid || nt > kMaxOrder) return;
  std::vector<int> cost(nt), idx(nt);
  const int per_pair = p.n1 * p.n3;
  const bool split = p.ksplit > 1;
  const int piece_cost = split ? (p.q + p.ksplit - 1) / p.ksplit : 0;
  for (int t = 0; t < nt; ++t) {
    idx[t] = t;
    if (split && t >= p.split_base) {  // an extra piece of a split heavy tile
      cost[t] = piece_cost;
      continue;
    }
    int p0, p1;
    host_pair_of(p, t / per_pair, p0, p1);
    cost[t] = pair_cost(p, p0, p1);
    if (split && cost[t] == p.q) cost[t] = piece_cost;  // the heavy tile's own piece
  }
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<std::vector<int>> lists(grid);
  // (load, cta) min-heap
  std::priority_queue<std::pair<long long, int>, std::vector<std::pair<long long, int>>,
                      std::greater<std::pair<long long, int>>> heap;
  for (int c = 0; c < grid; ++c) heap.push({0, c});
  for (int t : idx) {
    auto top = heap.top();
    heap.pop();
    lists[top.second].push_back(t);
    heap.push({top.first + cost[t], top.second});
  }
  size_t rounds = 0;
  for (auto& l : lists) rounds = l.size() > rounds ? l.size() : rounds;
  if ((long long)rounds * grid > kMaxOrder) return;
  for (size_t r = 0; r < rounds; ++r)
    for (int c = 0; c < grid; ++c)
      p.order[r * grid + c] = r < lists[c].size() ? (uint16_t)lists[c][r] : (uint16_t)0xFFFF;
  p.nslots = (int)(rounds * grid);
  p.use_order = 1;
}

// ------------------------------------------------ split-K of the heavy tiles
struct SplitReduce {
  const float* ws;
  __nv_bfloat16* out;
  long long ldo, Mq;
  int op, ksplit, n, nheavy, n1, n3, bi, bo, wn, swap, accumulate, q, off, qv;
};

// Adds the ksplit fp32 partials of every heavy tile and writes the bf16 result
// (added to the output when accumulating): one thread per 4 columns of a TMEM
// lane of a heavy tile.
__global__ void __launch_bounds__(256) k_split_reduce(const SplitReduce r) {
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int nq = r.n >> 2;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)r.nheavy * 128 * nq) return;
  const int cq = (int)(gid % nq);
  const long long rest = gid / nq;
  const int lane = (int)(rest % 128);
  const int dg = (int)(rest / 128);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < r.ksplit; ++s) {
    const float4 v =
        reinterpret_cast<const float4*>(r.ws + ((size_t)(dg * r.ksplit + s) * 128 + lane) * r.n)[cq];
    acc[0] += v.x;
    acc[1] += v.y;
    acc[2] += v.z;
    acc[3] += v.w;
  }
  const int i3 = dg % r.n3, i1 = (dg / r.n3) % r.n1, i0 = dg / (r.n3 * r.n1);
  const int col = 4 * cq;
  if (r.op == OP_DW) {
    // block (a, a): TMEM lanes are rows of dW (columns when swapped)
    const int a = i0, mb = r.swap ? i3 : i1, nb = r.swap ? i1 : i3;
    const long long xf = (long long)a * r.bi + (r.swap ? (long long)nb * r.wn : (long long)mb * 128);
    const long long yf = (long long)a * r.bo + (r.swap ? (long long)mb * 128 : (long long)nb * r.wn);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long rr = r.swap ? xf + col + j : xf + lane;
      const long long cc = r.swap ? yf + lane : yf + col + j;
      __nv_bfloat16* o = r.out + rr * r.ldo + cc;
      const float v = r.accumulate ? acc[j] + __bfloat162float(*o) : acc[j];
      *o = __float2bfloat16_rn(v);
    }
  } else {
    // dX tile (class c, group a = type of c): TMEM lanes are the class's rows
    const int c = i0;
    int t = c + r.off;
    if (t >= r.q) t -= r.q;
    const long long x = (long long)i1 * 128 + lane;
    if (x >= r.Mq) return;
    __nv_bfloat16* o = r.out + (x * r.qv + c) * r.ldo + (long long)t * r.bi + (long long)i3 * r.wn + col;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float v = r.accumulate ? acc[j] + __bfloat162float(o[j]) : acc[j];
      o[j] = __float2bfloat16_rn(v);
    }
  }
}

// Split factor of the heavy tiles: pieces of about the average load of a CTA
// (counted in 64-wide K chunks), no smaller than a light tile.  The pieces'
// partial sums go through the caller's workspace and a reduction kernel.
static void plan_split(Params& p, long long heavy_k, long long light_k, long long nheavy,
                       long long nlight) {
  p.ksplit = 0;
  if (nheavy <= 0 || heavy_k <= 64) return;
  const long long ch = (heavy_k + 63) / 64, cl = (light_k + 63) / 64;
  const long long grid = std::min<long long>(nheavy + nlight, num_sms());
  const long long total = nheavy * ch + nlight * cl;
  const long long target = std::max(cl, (total + grid - 1) / grid);
  // the reduction costs about as much as 16 chunks of a heavy tile: split only
  // tiles that run at least that much longer than a CTA's average load
  if (ch - target < 16) return;
  long long S = std::min<long long>((ch + target - 1) / target, 16);
  if (S < 2) return;
  const long long len = ((heavy_k + S - 1) / S + 63) / 64 * 64;
  S = (heavy_k + len - 1) / len;
  if (S < 2 || len > INT_MAX) return;
  p.ksplit = (int)S;
  p.split_len = (int)len;
}

// AAL_TEST_STALL=1 in the environment turns on Params::test_stall for the
// tcgen05 launches made while it is set (a test hook for the timeout path;
// read at every launch so that a test can switch it off again).
static int test_stall_enabled() {
  const char* e = getenv("AAL_TEST_STALL");
  return (e && e[0] == '1') ? 1 : 0;
}

template <bool A_MN, bool B_MN, int DUAL, bool PAIR = false, int MODE = 0>
static aal_status launch(Params& p, long long ntiles, cudaStream_t s) {
  if (ntiles <= 0) return AAL_OK;
  if (ntiles > INT_MAX) return AAL_ERR_UNSUPPORTED;
  p.ntiles = (int)ntiles;
  p.test_stall = test_stall_enabled();
  p.map_mask = 0;
  const CUtensorMap* maps[5] = {&p.mapA[0], &p.mapA[1], &p.mapB[0], &p.mapB[1], &p.mapOut};
  for (int i = 0; i < 5; ++i) {
    const unsigned char* b = reinterpret_cast<const unsigned char*>(maps[i]);
    bool used = false;
    for (size_t j = 0; j < sizeof(CUtensorMap) && !used; ++j) used = b[j] != 0;
    if (used) p.map_mask |= 1 << i;
  }
  if (!p.seg_mode) order_pairs(p);
  p.div_n1 = make_fastdiv((uint32_t)p.n1);
  p.div_n3 = make_fastdiv((uint32_t)p.n3);
  p.div_qm1 = make_fastdiv((uint32_t)(p.q > 1 ? p.q - 1 : 1));
  p.div_qn3 = make_fastdiv((uint32_t)(p.q * p.n3));
  const size_t smem = (size_t)p.stages * p.stage_bytes + kEpiSmem + 1024;
  static unsigned long long attr_set = 0;  // one bit per device ordinal
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AAL_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    if (cudaFuncSetAttribute(k_tc<A_MN, B_MN, DUAL, PAIR, MODE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBudget + 1024) != cudaSuccess)
      return AAL_ERR_CUDA;
    attr_set |= bit;
  }
  const int sms = num_sms();
  // every launch may overlap its set-up with the previous kernel's last CTAs
  // (programmatic stream serialization; the kernel waits before any global access)
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  p.dyn_slot = -1;
  if (!PAIR) {
    const int grid = (int)(ntiles < sms ? ntiles : sms);
    if (!p.seg_mode && !p.grp && MODE == 0) schedule_tiles(p, grid);
    else p.use_order = 0;
    // Many tiles and no cost-balanced order: hand the tiles out as CTAs free
    // up (SMs do not all run at the same speed; on the square product the
    // last CTA of a static stride schedule ended 25 % after the first).  The
    // tile decoder reserves up to kTileRing tiles ahead, so with few tiles a
    // CTA the fixed stride is as good.
    if (!p.use_order && !p.seg_mode && ntiles >= 32LL * grid) {
      static std::atomic<unsigned int> next_slot{0};
      p.dyn_slot = (int)(next_slot.fetch_add(1) % kDynSlots);
    }
    cfg.gridDim = dim3((unsigned)grid);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k_tc<A_MN, B_MN, DUAL, false, MODE>, p);
    note_launch();
    return cuda_status(e);
  }
  const int pairs = (int)(ntiles < sms / 2 ? ntiles : sms / 2);
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_tc<A_MN, B_MN, DUAL, true>, p);
  note_launch();
  return cuda_status(e);
}

// Launches the op with its heavy tiles split (when plan_split chose to and the
// caller's workspace holds the partial sums) and the reduction of the pieces.
template <bool A_MN, bool B_MN, int DUAL>
static aal_status launch_split(Params& p, long long base_tiles, long long nheavy, cudaStream_t s) {
  uint64_t have = 0;
  float* ws = static_cast<float*>(current_workspace(&have));
  const size_t bytes = p.ksplit > 1 ? (size_t)nheavy * p.ksplit * 128 * p.n_mma * sizeof(float) : 0;
  if (p.ksplit < 2 || !ws || have < bytes) {
    p.ksplit = 0;
    return launch<A_MN, B_MN, DUAL>(p, base_tiles, s);
  }
  p.split_ws = ws;
  p.split_base = (int)base_tiles;
  aal_status st = launch<A_MN, B_MN, DUAL>(p, base_tiles + nheavy * (p.ksplit - 1), s);
  if (st == AAL_OK) {
    SplitReduce r;
    r.ws = ws;
    r.out = p.out;
    r.ldo = p.ldo;
    r.Mq = p.Mq;
    r.op = p.op;
    r.ksplit = p.ksplit;
    r.n = p.n_mma;
    r.nheavy = (int)nheavy;
    r.n1 = p.n1;
    r.n3 = p.n3;
    r.bi = p.bi;
    r.bo = p.bo;
    r.wn = p.wn;
    r.swap = p.swap;
    r.accumulate = p.accumulate;
    r.q = p.q;
    r.off = p.off;
    r.qv = p.qv;
    const long long threads = nheavy * 128 * (p.n_mma / 4);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((threads + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    st = cuda_status(cudaLaunchKernelEx(&cfg, k_split_reduce, r));
    note_launch();
  }
  return st;
}

// Heavy-tile geometry of the dX and dW launches (kept in step with their planners).
struct SplitGeom {
  long long nheavy = 0, nlight = 0, heavy_k = 0, light_k = 0;
  int n = 0;
};
static SplitGeom geom_dx(int q, long long rows, long long bi, long long bo) {
  SplitGeom g;
  g.n = pick_n(bi, 256);
  if (!g.n) return g;
  const long long n1 = (rows / q + 127) / 128, n3 = bi / g.n;
  g.nheavy = (long long)q * n1 * n3;
  g.nlight = (long long)q * n1 * q * n3 - g.nheavy;
  g.heavy_k = (long long)q * bo;
  g.light_k = bo;
  return g;
}
static SplitGeom geom_dw(int q, long long rows, long long bi, long long bo) {
  SplitGeom g;
  const bool swap = bi % 128 != 0;
  if (swap && bo % 128 != 0) return g;
  g.n = pick_n(swap ? bi : bo, 256);
  if (!g.n) return g;
  const long long n1 = swap ? bi / g.n : bi / 128, n3 = swap ? bo / 128 : bo / g.n;
  g.nheavy = (long long)q * n1 * n3;
  g.nlight = (long long)q * n1 * q * n3 - g.nheavy;
  g.heavy_k = rows;
  g.light_k = rows / q;
  return g;
}
static int64_t split_bytes(const SplitGeom& g) {
  if (!g.n || g.nheavy <= 0) return 0;
  Params p;
  memset(&p, 0, sizeof(p));
  plan_split(p, g.heavy_k, g.light_k, g.nheavy, g.nlight);
  return p.ksplit > 1 ? (int64_t)g.nheavy * p.ksplit * 128 * g.n * (int64_t)sizeof(float) : 0;
}


// AAL_TC_PAIR=1 in the environment turns the CTA-pair mode on.  It is off by
// default: on B200 the single-CTA kernel with four producer warps and the
// tile decoder is as fast or faster on every shape measured (the fused
// gate/up of the 110M FFN: 73 us single, 78 us paired).
static bool pair_disabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("AAL_TC_PAIR");
    v = (e && e[0] == '1') ? 0 : 1;
  }
  return v == 1;
}

// Most classes a class-group tile may hold on the swapped forward path:
// AAL_TC_CLASS_GROUPS = 0 (one class per tile), 2 or 4 (the default); read once.
static int grp_max() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("AAL_TC_CLASS_GROUPS");
    v = 4;
    if (e && (e[0] == '0' || e[0] == '1')) v = 0;
    if (e && e[0] == '2') v = 2;
  }
  return v;
}

// AAL_TC_CLASS_PAIRS=0 keeps one row type per tile on the unswapped
// projection when a type has at most 64 rows (read once).
static bool cp_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("AAL_TC_CLASS_PAIRS");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

// AAL_TC_GROUP_PAIRS=0 keeps one output group per tile on the unswapped
// projection (read once).
static bool rg_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("AAL_TC_GROUP_PAIRS");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

static bool position_rule_ok(const RowTypes& rt, int q, long long rows) {
  return rt.kind == kTypesPosition && rt.seq_len % q == 0 && rows % q == 0 && rows > 0;
}

static void base_params(Params& p, int law, int q, const RowTypes& rt, long long rows) {
  memset(&p, 0, sizeof(p));
  p.law = law;
  p.q = q;
  p.off = (int)(rt.pos_offset % q);
  p.qv = q;
  p.Mq = rows / q;
  p.Mall = rows;
}

}  // namespace tc

using namespace tc;

void set_sm_share(int n) { t_sm_share = n; }
int device_sms() { return all_sms(); }

// Projection and fused gate/up share the planning; ``Wu`` null -> projection.
static aal_status tc_project_impl(int law, int q, const RowTypes& rt, long long rows,
                                  const aal_mat& X, const aal_mat& Wg, const aal_mat* Wu,
                                  const aal_mat& Y, cudaStream_t s) {
  if (!is_sm100() || !position_rule_ok(rt, q, rows)) return AAL_ERR_UNSUPPORTED;
  if (!tc_aligned(X) || !tc_aligned(Wg) || !tc_aligned(Y) || (Wu && !tc_aligned(*Wu)))
    return AAL_ERR_UNSUPPORTED;
  const long long bi = X.cols / q, bo = Wg.cols / q;
  if (bi > INT_MAX || bo > INT_MAX) return AAL_ERR_UNSUPPORTED;
  const bool dual = Wu != nullptr;
  if (bi % 16 || bo % 16) {
    // Ragged mode (a forward projection with groups that are not multiples
    // of 16): the A box spans ka >= offset + gbi features, the tile N >=
    // column offset + gbo columns, over every group a and k.
    if (dual || bi < 16 || law != AAL_LAW_Q) return AAL_ERR_UNSUPPORTED;
    int oa = 0, oc = 0;
    for (long long g = 0; g < q; ++g) {
      oa = std::max(oa, (int)((g * bi) & 7));
      oc = std::max(oc, (int)((g * bo) & 15));
    }
    const int ka = (int)((oa + bi + 15) / 16 * 16), n = (int)((oc + bo + 15) / 16 * 16);
    if ((ka != 32 && ka != 64) || n > 256) return AAL_ERR_UNSUPPORTED;
    Params p;
    base_params(p, law, q, rt, rows);
    p.op = OP_FWD;
    p.ragged = 1;
    p.gbi = (int)bi;
    p.gbo = (int)bo;
    p.ka = ka;
    p.bi = (int)bi;
    p.bo = (int)bo;
    p.out = (__nv_bfloat16*)Y.ptr;
    p.ldo = Y.ld;
    p.swap = 0;
    p.xr = 128;
    p.wn = n;
    p.n_mma = n;
    p.a_rows = 128;
    p.b_rows = n;
    p.b_aw = 16;
    p.idesc = make_idesc(128, n, false, true);
    if (!finish_plan(p, 0)) return AAL_ERR_UNSUPPORTED;
    if (!make_map(&p.mapA[0], X.ptr, X.rows, X.cols, X.ld, q, ka, 128, ka * 2)) return AAL_ERR_UNSUPPORTED;
    if (!map_ragged_w(&p.mapB[0], Wg, (int)bi, ka, n / 16)) return AAL_ERR_UNSUPPORTED;
    if (!out_map(p, Y, q)) return AAL_ERR_UNSUPPORTED;
    p.n1 = (int)((p.Mq + 127) / 128);
    p.n2 = q;
    p.n3 = 1;
    return launch<false, true, 0>(p, (long long)q * p.n1 * p.n2, s);
  }
  Params p;
  base_params(p, law, q, rt, rows);
  p.op = dual ? OP_SWIGLU : OP_FWD;
  p.bi = (int)bi;
  p.bo = (int)bo;
  p.swiglu = dual;
  p.out = (__nv_bfloat16*)Y.ptr;
  p.ldo = Y.ld;
  const bool swap = p.Mq < 128 && bo % 128 == 0;
  long long ntiles;
  // CTA pair (M = 256): enough rows per class, and each CTA's half of B a
  // whole number of 16-column atoms
  const int npair = pick_n(bo, dual ? 128 : 256);
  const bool pair = !swap && p.Mq >= 256 && npair && (dual ? npair == 128 : (npair / 2) % 16 == 0) &&
                    !pair_disabled();
  if (pair) {
    const int n = npair;
    p.swap = 0;
    p.xr = 256;
    p.wn = n;
    p.n_mma = n;  // per-operand width; the MMA spans 2n with two operands
    p.a_rows = 128;
    p.b_rows = dual ? n : n / 2;
    p.b_aw = p.b_rows % 64 == 0 ? 64 : 16;
    p.fuse_b = dual;
    p.idesc = make_idesc(256, n, false, true);
    p.idesc2 = dual ? make_idesc(256, 2 * n, false, true) : 0;
    if (!finish_plan(p, dual ? 1 : 0, true)) return AAL_ERR_UNSUPPORTED;
    if (!map_kmajor(&p.mapA[0], X, q, 128)) return AAL_ERR_UNSUPPORTED;
    int mg1 = 1;
    if (!map_mn(&p.mapB[0], Wg, 1, p.b_aw, p.b_rows, &p.b_merged)) return AAL_ERR_UNSUPPORTED;
    if (dual && !map_mn(&p.mapB[1], *Wu, 1, p.b_aw, p.b_rows, &mg1)) return AAL_ERR_UNSUPPORTED;
    if (!mg1 && p.b_merged) {  // both operands must use the same form
      p.b_merged = 0;
      if (!map_mnmajor(&p.mapB[0], Wg, 1, p.b_aw)) return AAL_ERR_UNSUPPORTED;
    }
    if (!out_map(p, Y, q)) return AAL_ERR_UNSUPPORTED;
    p.n1 = (int)((p.Mq + 255) / 256);
    p.n2 = q;
    p.n3 = (int)(bo / n);
    ntiles = (long long)q * p.n1 * p.n2 * p.n3;
    return dual ? launch<false, true, 1, true>(p, ntiles, s) : launch<false, true, 0, true>(p, ntiles, s);
  }
  if (!swap && !dual && law == AAL_LAW_Q && q % 2 == 0 && p.Mq <= 64 && cp_enabled()) {
    // Class pairs: at most 64 rows a type fill half of a 128-row tile; two
    // types share the tile, the diagonal term as one MMA over both
    const int n = pick_n(bo, 256);
    if (!n) return AAL_ERR_UNSUPPORTED;
    p.swap = 0;
    p.xr = 128;
    p.wn = n;
    p.n_mma = n;
    p.a_rows = 128;
    p.b_rows = n;
    p.b_aw = n % 64 == 0 ? 64 : 16;
    p.idesc = make_idesc(128, n, false, true);
    if (!finish_plan(p, 0)) return AAL_ERR_UNSUPPORTED;
    if (!map_kmajor(&p.mapA[0], X, q, 64)) return AAL_ERR_UNSUPPORTED;
    if (!map_mn(&p.mapB[0], Wg, 1, p.b_aw, p.b_rows, &p.b_merged)) return AAL_ERR_UNSUPPORTED;
    if (!out_map(p, Y, q)) return AAL_ERR_UNSUPPORTED;
    p.n1 = 1;
    p.n2 = q;
    p.n3 = (int)(bo / n);
    ntiles = (long long)(q / 2) * q * p.n3;
    return launch<false, true, 0, false, 2>(p, ntiles, s);
  }
  if (!swap && law == AAL_LAW_Q && q % 2 == 0 && 2 * bo <= (dual ? 128 : 256) && rg_enabled()) {
    // Output-group pairs: the type's own segment x_t W(t, [k0, k0 + 2)) as
    // one MMA over both groups' columns, the two diagonal terms into their
    // column ranges (half the tiles of one group each, and fewer MMAs); for
    // the fused gate/up each of those is a gate MMA and an up MMA
    const int n = (int)(2 * bo);
    p.swap = 0;
    p.xr = 128;
    p.wn = n;
    p.n_mma = n;
    p.a_rows = 128;
    p.b_rows = n;
    p.b_aw = bo % 64 == 0 ? 64 : 16;
    p.rg_n = (int)bo;
    p.idesc = make_idesc(128, n, false, true);
    p.idesc_one = make_idesc(128, (int)bo, false, true);
    p.fuse_b = 0;
    if (!finish_plan(p, dual ? 1 : 0)) return AAL_ERR_UNSUPPORTED;
    if (!map_kmajor(&p.mapA[0], X, q, 128)) return AAL_ERR_UNSUPPORTED;
    if (!map_mnmajor(&p.mapB[0], Wg, 1, p.b_aw)) return AAL_ERR_UNSUPPORTED;
    if (dual && !map_mnmajor(&p.mapB[1], *Wu, 1, p.b_aw)) return AAL_ERR_UNSUPPORTED;
    p.b_merged = 0;  // a diagonal segment loads only its group's atoms
    if (!out_map(p, Y, q)) return AAL_ERR_UNSUPPORTED;
    p.n1 = (int)((p.Mq + 127) / 128);
    p.n2 = q;
    p.n3 = 1;
    ntiles = (long long)q * p.n1 * (q / 2);
    return dual ? launch<false, true, 1, false, 1>(p, ntiles, s) : launch<false, true, 0, false, 1>(p, ntiles, s);
  }
  if (!swap) {
    const int n = pick_n(bo, dual ? 128 : 256);
    if (!n) return AAL_ERR_UNSUPPORTED;
    p.swap = 0;
    p.xr = 128;
    p.wn = n;
    p.n_mma = n;
    p.a_rows = 128;
    p.b_rows = n;
    p.b_aw = n % 64 == 0 ? 64 : 16;
    p.idesc = make_idesc(128, n, false, true);
    // gate and up tiles form one MN-major operand when the atom stride is uniform
    p.fuse_b = dual && p.b_aw == 64 && 2 * n <= 256;
    p.idesc2 = p.fuse_b ? make_idesc(128, 2 * n, false, true) : 0;
    if (!finish_plan(p, dual ? 1 : 0)) return AAL_ERR_UNSUPPORTED;
    if (!map_kmajor(&p.mapA[0], X, q, 128)) return AAL_ERR_UNSUPPORTED;
    int mg1 = 1;
    if (!map_mn(&p.mapB[0], Wg, 1, p.b_aw, p.b_rows, &p.b_merged)) return AAL_ERR_UNSUPPORTED;
    if (dual && !map_mn(&p.mapB[1], *Wu, 1, p.b_aw, p.b_rows, &mg1)) return AAL_ERR_UNSUPPORTED;
    if (!mg1 && p.b_merged) {
      p.b_merged = 0;
      if (!map_mnmajor(&p.mapB[0], Wg, 1, p.b_aw)) return AAL_ERR_UNSUPPORTED;
    }
    if (!out_map(p, Y, q)) return AAL_ERR_UNSUPPORTED;
    p.n1 = (int)((p.Mq + 127) / 128);
    p.n2 = q;
    p.n3 = (int)(bo / n);
    ntiles = (long long)q * p.n1 * p.n2 * p.n3;
    return dual ? launch<false, true, 1>(p, ntiles, s) : launch<false, true, 0>(p, ntiles, s);
  }
  const int ntok = (int)((p.Mq + 15) / 16 * 16);
  // Class groups under Q_q: G classes share the diagonal term's weight tile
  // and one wide MMA (G * ntok columns of TMEM per accumulator, at most 128:
  // wider groups leave too few tiles to spread over the SMs; on the
  // Qwen3-8B-shaped down projection G = 4 ran 50.6 us, G = 2 46.4 us, one
  // class per tile 48.6 us)
  int G = 0;
  if (law == AAL_LAW_Q) {
    for (int g = grp_max(); g >= 2; g >>= 1)
      if (q % g == 0 && g * ntok <= 128) { G = g; break; }
  }
  p.swap = 1;
  p.xr = ntok;
  p.wn = 128;
  p.n_mma = G ? G * ntok : ntok;
  p.a_rows = 128;
  p.b_rows = p.n_mma;
  p.a_aw = 64;
  p.idesc = make_idesc(128, p.n_mma, true, false);
  if (G) {
    p.grp = G;
    p.grp_n = ntok;
    p.idesc_one = make_idesc(128, ntok, true, false);
    p.box_bytes = (uint32_t)ntok * 128u;
  }
  if (!finish_plan(p, dual ? 2 : 0)) return AAL_ERR_UNSUPPORTED;
  int mg1 = 1;
  if (!map_mn(&p.mapA[0], Wg, 1, 64, 128, &p.a_merged)) return AAL_ERR_UNSUPPORTED;
  if (dual && !map_mn(&p.mapA[1], *Wu, 1, 64, 128, &mg1)) return AAL_ERR_UNSUPPORTED;
  if (!mg1 && p.a_merged) {
    p.a_merged = 0;
    if (!map_mnmajor(&p.mapA[0], Wg, 1, 64)) return AAL_ERR_UNSUPPORTED;
  }
  if (!map_kmajor(&p.mapB[0], X, q, ntok)) return AAL_ERR_UNSUPPORTED;
  if (!out_map(p, Y, q)) return AAL_ERR_UNSUPPORTED;
  p.n1 = 1;
  p.n2 = q;
  p.n3 = (int)(bo / 128);
  ntiles = (long long)(G ? q / G : q) * p.n2 * p.n3;
  return dual ? launch<true, false, 2>(p, ntiles, s) : launch<true, false, 0>(p, ntiles, s);
}

// Segment mode of the forward ops: Xg holds the rows gathered type by type
// (tile table, count and permutation on the device), so a type's rows are
// contiguous whatever the positions or explicit types were; Y receives row
// perm[x] for gathered row x, and ``copy`` (if given) the same tiles in the
// gathered order.  ``tmax`` bounds the table length.
aal_status tc_project_seg(int law, int q, long long rows, const aal_mat& Xg, const aal_mat& Wg,
                          const aal_mat* Wu, const aal_mat& Y, const int4* tiles, const int* count,
                          const int* perm, int tmax, const aal_mat* copy, cudaStream_t s) {
  if (!is_sm100()) return AAL_ERR_UNSUPPORTED;
  if (!tc_aligned(Xg) || !tc_aligned(Wg) || !tc_aligned(Y) || (Wu && !tc_aligned(*Wu)) ||
      (copy && !tc_aligned(*copy)))
    return AAL_ERR_UNSUPPORTED;
  const long long bi = Xg.cols / q, bo = Wg.cols / q;
  if (bi % 16 || bo % 16 || bi > INT_MAX || bo > INT_MAX || rows > INT_MAX) return AAL_ERR_UNSUPPORTED;
  const bool dual = Wu != nullptr;
  Params p;
  memset(&p, 0, sizeof(p));
  p.law = law;
  p.q = q;
  p.qv = 1;
  p.Mq = rows;
  p.Mall = rows;
  p.op = dual ? OP_SWIGLU : OP_FWD;
  p.bi = (int)bi;
  p.bo = (int)bo;
  p.swiglu = dual;
  p.out = (__nv_bfloat16*)Y.ptr;
  p.ldo = Y.ld;
  p.seg_mode = 1;
  p.seg_tiles = tiles;
  p.seg_count = count;
  p.seg_perm = perm;
  if (copy) {
    p.seg_copy = (__nv_bfloat16*)copy->ptr;
    p.ld_copy = copy->ld;
  }
  if (law == AAL_LAW_Q && q % 2 == 0 && 2 * bo <= (dual ? 128 : 256) && rg_enabled()) {
    // output-group pairs, as on the strided path: tile (j, kp) is table
    // entry j against output groups 2 kp and 2 kp + 1
    const int n = (int)(2 * bo);
    p.swap = 0;
    p.xr = 128;
    p.wn = n;
    p.n_mma = n;
    p.a_rows = 128;
    p.b_rows = n;
    p.b_aw = bo % 64 == 0 ? 64 : 16;
    p.rg_n = (int)bo;
    p.idesc = make_idesc(128, n, false, true);
    p.idesc_one = make_idesc(128, (int)bo, false, true);
    p.fuse_b = 0;
    if (!finish_plan(p, dual ? 1 : 0)) return AAL_ERR_UNSUPPORTED;
    if (!map_kmajor(&p.mapA[0], Xg, 1, 128)) return AAL_ERR_UNSUPPORTED;
    if (!map_mnmajor(&p.mapB[0], Wg, 1, p.b_aw)) return AAL_ERR_UNSUPPORTED;
    if (dual && !map_mnmajor(&p.mapB[1], *Wu, 1, p.b_aw)) return AAL_ERR_UNSUPPORTED;
    p.b_merged = 0;  // a diagonal segment loads only its group's atoms
    if (!out_map(p, Y, 1)) return AAL_ERR_UNSUPPORTED;
    p.n1 = 1;
    p.n2 = q;
    p.n3 = 1;
    const long long ntiles = (long long)tmax * (q / 2);
    return dual ? launch<false, true, 1, false, 1>(p, ntiles, s) : launch<false, true, 0, false, 1>(p, ntiles, s);
  }
  const int n = pick_n(bo, dual ? 128 : 256);
  if (!n) return AAL_ERR_UNSUPPORTED;
  p.swap = 0;
  p.xr = 128;
  p.wn = n;
  p.n_mma = n;
  p.a_rows = 128;
  p.b_rows = n;
  p.b_aw = n % 64 == 0 ? 64 : 16;
  p.idesc = make_idesc(128, n, false, true);
  p.fuse_b = dual && p.b_aw == 64 && 2 * n <= 256;
  p.idesc2 = p.fuse_b ? make_idesc(128, 2 * n, false, true) : 0;
  if (!finish_plan(p, dual ? 1 : 0)) return AAL_ERR_UNSUPPORTED;
  if (!map_kmajor(&p.mapA[0], Xg, 1, 128)) return AAL_ERR_UNSUPPORTED;
  int mg1 = 1;
  if (!map_mn(&p.mapB[0], Wg, 1, p.b_aw, p.b_rows, &p.b_merged)) return AAL_ERR_UNSUPPORTED;
  if (dual && !map_mn(&p.mapB[1], *Wu, 1, p.b_aw, p.b_rows, &mg1)) return AAL_ERR_UNSUPPORTED;
  if (!mg1 && p.b_merged) {
    p.b_merged = 0;
    if (!map_mnmajor(&p.mapB[0], Wg, 1, p.b_aw)) return AAL_ERR_UNSUPPORTED;
  }
  if (!out_map(p, Y, 1)) return AAL_ERR_UNSUPPORTED;
  p.n1 = 1;
  p.n2 = q;
  p.n3 = (int)(bo / n);
  const long long ntiles = (long long)tmax * q * p.n3;
  return dual ? launch<false, true, 1>(p, ntiles, s) : launch<false, true, 0>(p, ntiles, s);
}

aal_status tc_project(int law, int q, const RowTypes& rt, long long rows, const aal_mat& X,
                      const aal_mat& W, const aal_mat& Y, cudaStream_t s) {
  return tc_project_impl(law, q, rt, rows, X, W, nullptr, Y, s);
}

aal_status tc_swiglu_gate_up(int law, int q, const RowTypes& rt, long long rows, const aal_mat& X,
                             const aal_mat& Wg, const aal_mat& Wu, const aal_mat& H,
                             cudaStream_t s) {
  return tc_project_impl(law, q, rt, rows, X, Wg, &Wu, H, s);
}

// dX of a row-typed projection; with ``act`` (G, U, dU) the SwiGLU
// backward's SiLU' chain runs in the epilogue: dX is then dG (the gradient of
// the gate pre-activation) and dU receives the gradient of the up projection.
static aal_status bwd_dx_impl(int law, int q, const RowTypes& rt, long long rows, const aal_mat& dY,
                              const aal_mat& W, const aal_mat& dX, int accumulate,
                              const aal_mat* G, const aal_mat* U, const aal_mat* dU, cudaStream_t s) {
  if (!is_sm100() || !position_rule_ok(rt, q, rows)) return AAL_ERR_UNSUPPORTED;
  if (!tc_aligned(dY) || !tc_aligned(W) || !tc_aligned(dX)) return AAL_ERR_UNSUPPORTED;
  if (G && (!tc_aligned(*G) || !tc_aligned(*U) || !tc_aligned(*dU) || G->ld != dX.ld ||
            U->ld != dX.ld || dU->ld != dX.ld))
    return AAL_ERR_UNSUPPORTED;
  const long long bi = W.rows / q, bo = W.cols / q;
  if (bi % 16 || bo % 16) return AAL_ERR_UNSUPPORTED;
  Params p;
  base_params(p, law, q, rt, rows);
  p.op = OP_DX;
  p.bi = (int)bi;
  p.bo = (int)bo;
  p.out = (__nv_bfloat16*)dX.ptr;
  p.ldo = dX.ld;
  p.accumulate = accumulate ? 1 : 0;
  if (G) {
    p.swiglu_bwd = 1;
    p.g_in = (const __nv_bfloat16*)G->ptr;
    p.u_in = (const __nv_bfloat16*)U->ptr;
    p.out2 = (__nv_bfloat16*)dU->ptr;
  }
  const int n = pick_n(bi, 256);
  if (!n) return AAL_ERR_UNSUPPORTED;
  p.xr = 128;
  p.wn = n;
  p.n_mma = n;
  p.a_rows = 128;
  p.b_rows = n;
  p.idesc = make_idesc(128, n, false, false);
  if (!finish_plan(p, 0)) return AAL_ERR_UNSUPPORTED;
  if (!map_kmajor(&p.mapA[0], dY, q, 128)) return AAL_ERR_UNSUPPORTED;
  if (!map_kmajor(&p.mapB[0], W, 1, n)) return AAL_ERR_UNSUPPORTED;
  if (!out_map(p, dX, q)) return AAL_ERR_UNSUPPORTED;
  p.n1 = (int)((p.Mq + 127) / 128);
  p.n2 = q;
  p.n3 = (int)(bi / n);
  const long long base = (long long)q * p.n1 * p.n2 * p.n3, nheavy = (long long)q * p.n1 * p.n3;
  // heavy tiles (a == t) run over all q output groups; the SiLU' epilogue needs
  // the whole sum in one place, so the dH kernel keeps them whole
  if (law == AAL_LAW_Q && q > 1 && !G) plan_split(p, (long long)q * bo, bo, nheavy, base - nheavy);
  return launch_split<false, false, 0>(p, base, nheavy, s);
}

// dX of the SwiGLU backward in one launch: dX = dG Wg^T + dU Wu^T through the
// transposed table, both products of a tile accumulated in the same TMEM
// accumulator (one rounding to bf16).
aal_status tc_swiglu_bwd_dx(int law, int q, const RowTypes& rt, long long rows, const aal_mat& dG,
                            const aal_mat& Wg, const aal_mat& dU, const aal_mat& Wu, const aal_mat& dX,
                            cudaStream_t s) {
  if (!is_sm100() || !position_rule_ok(rt, q, rows)) return AAL_ERR_UNSUPPORTED;
  if (!tc_aligned(dG) || !tc_aligned(dU) || !tc_aligned(Wg) || !tc_aligned(Wu) || !tc_aligned(dX))
    return AAL_ERR_UNSUPPORTED;
  const long long bi = Wg.rows / q, bo = Wg.cols / q;
  if (bi % 16 || bo % 16) return AAL_ERR_UNSUPPORTED;
  Params p;
  base_params(p, law, q, rt, rows);
  p.op = OP_DX;
  p.bi = (int)bi;
  p.bo = (int)bo;
  p.out = (__nv_bfloat16*)dX.ptr;
  p.ldo = dX.ld;
  const int n = pick_n(bi, 256);
  if (!n) return AAL_ERR_UNSUPPORTED;
  p.xr = 128;
  p.wn = n;
  p.n_mma = n;
  p.a_rows = 128;
  p.b_rows = n;
  p.idesc = make_idesc(128, n, false, false);
  if (!finish_plan(p, 3)) return AAL_ERR_UNSUPPORTED;
  if (!map_kmajor(&p.mapA[0], dG, q, 128) || !map_kmajor(&p.mapA[1], dU, q, 128)) return AAL_ERR_UNSUPPORTED;
  if (!map_kmajor(&p.mapB[0], Wg, 1, n) || !map_kmajor(&p.mapB[1], Wu, 1, n)) return AAL_ERR_UNSUPPORTED;
  if (!out_map(p, dX, q)) return AAL_ERR_UNSUPPORTED;
  p.n1 = (int)((p.Mq + 127) / 128);
  p.n2 = q;
  p.n3 = (int)(bi / n);
  const long long base = (long long)q * p.n1 * p.n2 * p.n3, nheavy = (long long)q * p.n1 * p.n3;
  if (law == AAL_LAW_Q && q > 1) plan_split(p, (long long)q * bo, bo, nheavy, base - nheavy);
  return launch_split<false, false, 3>(p, base, nheavy, s);
}

aal_status tc_project_bwd_dx(int law, int q, const RowTypes& rt, long long rows, const aal_mat& dY,
                             const aal_mat& W, const aal_mat& dX, int accumulate, cudaStream_t s) {
  return bwd_dx_impl(law, q, rt, rows, dY, W, dX, accumulate, nullptr, nullptr, nullptr, s);
}

aal_status tc_swiglu_bwd_dh(int law, int q, const RowTypes& rt, long long rows, const aal_mat& dY,
                            const aal_mat& Wd, const aal_mat& G, const aal_mat& U,
                            const aal_mat& dG, const aal_mat& dU, cudaStream_t s) {
  return bwd_dx_impl(law, q, rt, rows, dY, Wd, dG, 0, &G, &U, &dU, s);
}

void tc_bwd_split_parts(int law, int q, long long rows, long long din, long long dout, int64_t* dx,
                        int64_t* dw) {
  *dx = *dw = 0;
  if (law != AAL_LAW_Q || q < 2 || rows % q || din % q || dout % q) return;
  const long long bi = din / q, bo = dout / q;
  if (bi % 16 || bo % 16) return;
  *dx = split_bytes(geom_dx(q, rows, bi, bo));
  *dw = split_bytes(geom_dw(q, rows, bi, bo));
}

// AAL_TC_SIDE_BY_SIDE=0 in the environment keeps a projection backward's dX
// and dW launches one after the other on the caller's stream (read once).
static bool side_by_side_enabled() {
  static const int v = [] {
    const char* e = getenv("AAL_TC_SIDE_BY_SIDE");
    return (e && e[0] == '0') ? 0 : 1;
  }();
  return v != 0;
}

bool tc_bwd_side_by_side(long long rows, long long din, long long dout) {
  // small problems only: a few tiles a CTA, so that the launches' fixed
  // start-up and drain overlap; larger ones fill the GPU one at a time
  return side_by_side_enabled() && rows > 0 && din > 0 && dout > 0 &&
         (double)rows * (double)din * (double)dout <= 8.6e9;
}

int64_t tc_bwd_split_bytes(int law, int q, long long rows, long long din, long long dout) {
  int64_t a = 0, b = 0;
  tc_bwd_split_parts(law, q, rows, din, dout, &a, &b);
  int64_t need = a > b ? a : b;
  if (tc_bwd_side_by_side(rows, din, dout)) {
    // side by side: dX's partials first, dW's after them, each planned on half the SMs
    const int keep = t_sm_share;
    t_sm_share = all_sms() / 2;
    tc_bwd_split_parts(law, q, rows, din, dout, &a, &b);
    t_sm_share = keep;
    const int64_t both = ((a + 255) & ~(int64_t)255) + b;
    if (both > need) need = both;
  }
  return need;
}

int64_t tc_swiglu_bwd_split_bytes(int law, int q, long long rows, long long D, long long F) {
  const int64_t a = tc_bwd_split_bytes(law, q, rows, D, F), b = tc_bwd_split_bytes(law, q, rows, F, D);
  int64_t need = a > b ? a : b;
  if (tc_bwd_side_by_side(rows, D, F)) {
    // dX (gate + up) then dWu on the caller's stream, dWd then dWg on the
    // side stream after them in the workspace, all planned on half the SMs
    const int keep = t_sm_share;
    t_sm_share = all_sms() / 2;
    int64_t dx = 0, dw = 0, dx2 = 0, dwd = 0;
    tc_bwd_split_parts(law, q, rows, D, F, &dx, &dw);
    tc_bwd_split_parts(law, q, rows, F, D, &dx2, &dwd);
    t_sm_share = keep;
    const int64_t both = (((dx > dw ? dx : dw) + 255) & ~(int64_t)255) + (dw > dwd ? dw : dwd);
    if (both > need) need = both;
  }
  return need;
}

aal_status tc_project_bwd_dw(int law, int q, const RowTypes& rt, long long rows, const aal_mat& X,
                             const aal_mat& dY, const aal_mat& dW, int accumulate,
                             cudaStream_t s) {
  if (!is_sm100() || !position_rule_ok(rt, q, rows)) return AAL_ERR_UNSUPPORTED;
  if (!tc_aligned(X) || !tc_aligned(dY) || !tc_aligned(dW)) return AAL_ERR_UNSUPPORTED;
  const long long bi = dW.rows / q, bo = dW.cols / q;
  if (bi % 16 || bo % 16 || rows > INT_MAX) return AAL_ERR_UNSUPPORTED;
  Params p;
  base_params(p, law, q, rt, rows);
  p.op = OP_DW;
  p.bi = (int)bi;
  p.bo = (int)bo;
  p.out = (__nv_bfloat16*)dW.ptr;
  p.ldo = dW.ld;
  p.accumulate = accumulate ? 1 : 0;
  // MMA M = 128 features of group a (or of group k when swapped), N the other side
  const bool swap = bi % 128 != 0;
  if (swap && bo % 128 != 0) return AAL_ERR_UNSUPPORTED;
  const int n = pick_n(swap ? bi : bo, 256);
  if (!n) return AAL_ERR_UNSUPPORTED;
  p.swap = swap;
  p.wn = n;
  p.n_mma = n;
  p.a_rows = 128;
  p.b_rows = n;
  p.a_aw = 64;
  p.b_aw = n % 64 == 0 ? 64 : 16;
  p.idesc = make_idesc(128, n, true, true);
  if (!finish_plan(p, 0)) return AAL_ERR_UNSUPPORTED;
  const aal_mat& A = swap ? dY : X;
  const aal_mat& B = swap ? X : dY;
  {
    int ma0 = 0, ma1 = 0, mb0 = 0, mb1 = 0;
    if (!map_mn(&p.mapA[0], A, q, 64, 128, &ma0) || !map_mn(&p.mapA[1], A, 1, 64, 128, &ma1))
      return AAL_ERR_UNSUPPORTED;
    if (!map_mn(&p.mapB[0], B, q, p.b_aw, n, &mb0) || !map_mn(&p.mapB[1], B, 1, p.b_aw, n, &mb1))
      return AAL_ERR_UNSUPPORTED;
    if (!(ma0 && ma1)) {
      if (!map_mnmajor(&p.mapA[0], A, q, 64) || !map_mnmajor(&p.mapA[1], A, 1, 64))
        return AAL_ERR_UNSUPPORTED;
    }
    if (!(mb0 && mb1)) {
      if (!map_mnmajor(&p.mapB[0], B, q, p.b_aw) || !map_mnmajor(&p.mapB[1], B, 1, p.b_aw))
        return AAL_ERR_UNSUPPORTED;
    }
    p.a_merged = ma0 && ma1;
    p.b_merged = mb0 && mb1;
  }
  if (!out_map(p, dW, 1)) return AAL_ERR_UNSUPPORTED;
  if (!swap) { p.n1 = (int)(bi / 128); p.n3 = (int)(bo / n); }
  else { p.n1 = (int)(bi / n); p.n3 = (int)(bo / 128); }
  p.n2 = q;
  const long long base = (long long)q * p.n1 * p.n2 * p.n3, nheavy = (long long)q * p.n1 * p.n3;
  // heavy tiles: the diagonal blocks, whose K runs over every token
  if (law == AAL_LAW_Q && q > 1) plan_split(p, rows, p.Mq, nheavy, base - nheavy);
  return launch_split<true, true, 0>(p, base, nheavy, s);
}

aal_status tc_square(int law, int q, const aal_mat& X, const aal_mat& W, const aal_mat& Z,
                     cudaStream_t s) {
  if (!is_sm100()) return AAL_ERR_UNSUPPORTED;
  if (!tc_aligned(X) || !tc_aligned(W) || !tc_aligned(Z)) return AAL_ERR_UNSUPPORTED;
  const long long n = X.rows, b = n / q;
  if (b % 128 || b > INT_MAX) return AAL_ERR_UNSUPPORTED;
  Params p;
  memset(&p, 0, sizeof(p));
  p.op = OP_SQUARE;
  p.law = law;
  p.q = q;
  p.qv = 1;
  p.bi = (int)b;
  p.bo = (int)b;
  p.out = (__nv_bfloat16*)Z.ptr;
  p.ldo = Z.ld;
  if (law == AAL_LAW_Q && q % 2 == 0 && b == 128 && rg_enabled()) {
    // column-block pairs: X_ii W_i,[k0, k0 + 2) as one N = 256 MMA, then the
    // diagonal terms X_ig W_gg into their blocks' column ranges
    p.xr = 128;
    p.wn = 256;
    p.n_mma = 256;
    p.a_rows = 128;
    p.b_rows = 256;
    p.b_aw = 64;
    p.rg_n = 128;
    p.idesc = make_idesc(128, 256, false, true);
    p.idesc_one = make_idesc(128, 128, false, true);
    if (!finish_plan(p, 0)) return AAL_ERR_UNSUPPORTED;
    if (!map_kmajor(&p.mapA[0], X, 1, 128)) return AAL_ERR_UNSUPPORTED;
    if (!map_mnmajor(&p.mapB[0], W, 1, 64)) return AAL_ERR_UNSUPPORTED;
    p.b_merged = 0;
    if (!out_map(p, Z, 1)) return AAL_ERR_UNSUPPORTED;
    p.n1 = 1;
    p.n2 = q;
    p.n3 = 1;
    return launch<false, true, 0, false, 1>(p, (long long)(q / 2) * q, s);
  }
  const int nn = pick_n(b, 256);
  p.xr = 128;
  p.wn = nn;
  p.n_mma = nn;
  p.a_rows = 128;
  p.b_rows = nn;
  p.b_aw = nn % 64 == 0 ? 64 : 16;
  p.idesc = make_idesc(128, nn, false, true);
  if (!finish_plan(p, 0)) return AAL_ERR_UNSUPPORTED;
  if (!map_kmajor(&p.mapA[0], X, 1, 128)) return AAL_ERR_UNSUPPORTED;
  if (!map_mn(&p.mapB[0], W, 1, p.b_aw, nn, &p.b_merged)) return AAL_ERR_UNSUPPORTED;
  if (!out_map(p, Z, 1)) return AAL_ERR_UNSUPPORTED;
  p.n1 = (int)(b / 128);
  p.n2 = q;
  p.n3 = (int)(b / nn);
  return launch<false, true, 0>(p, (long long)q * p.n1 * p.n2 * p.n3, s);
}

}  // namespace aal
