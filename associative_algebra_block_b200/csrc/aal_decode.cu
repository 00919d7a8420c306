// Decode step: one new token per batch entry, y_b = row t_b of the table
// applied to x_b (agihunt.info digest: decoding evaluates only the new
// position's row, as a matrix-vector product with a kernel of its own).
//
// The work is a stream over the weight rows that some entry of the batch
// needs: a weight block is loaded only when some entry's table row uses it,
// so one row type touches (2q-1)/q^2 of W (9/16 for Q2xQ2).  Kernels, in the
// order the dispatcher tries them:
//   k_decode_mma (bf16, <= 256 entries, 64-column output groups): warp-level
//     tensor-core MMAs, split-K over an 8-CTA cluster (clusters of 2, 4 and
//     16 measured slower on B200), also the fused gate/up/SiLU step of a
//     SwiGLU FFN;
//   k_decode_typed (bf16, 32-column groups): a CTA per column slab and row
//     type streams only the rows of S(t, k);
//   k_decode_split (bf16, 64-column groups): weight rows split across a
//     cluster, activations staged in shared memory;
//   k_decode_vec (16-byte vector loads, fp32 included) and k_decode (scalar)
//     for everything else.
#include <cooperative_groups.h>
#include <limits.h>
#include <stdlib.h>

#include "aal_internal.h"

namespace cg = cooperative_groups;

namespace aal {

constexpr int kDecodeBT = 16;       // batch entries per CTA
constexpr int kDecodeCols = 64;     // weight columns per CTA
constexpr int kDecodeWarps = 8;

template <typename T>
__device__ __forceinline__ float dec_ld(const T* p);
template <>
__device__ __forceinline__ float dec_ld<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float dec_ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}
template <typename T>
__device__ __forceinline__ void dec_st(T* p, float v);
template <>
__device__ __forceinline__ void dec_st<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void dec_st<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

template <typename T>
__global__ void __launch_bounds__(kDecodeWarps * 32)
k_decode(int law, int q, const int64_t* __restrict__ pos, long long B, const T* __restrict__ x,
         long long ldx, const T* __restrict__ W, long long ldw, T* __restrict__ y, long long ldy,
         int bi, int bo) {
  __shared__ float red[kDecodeWarps][kDecodeBT][kDecodeCols];
  __shared__ int types[kDecodeBT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long din = (long long)bi * q, dout = (long long)bo * q;
  const long long c0 = (long long)blockIdx.x * kDecodeCols + 2 * lane;
  const long long b0 = (long long)blockIdx.y * kDecodeBT;
  const int nb = (int)min((long long)kDecodeBT, B - b0);

  if (threadIdx.x < kDecodeBT) {
    int t = -1;
    if ((int)threadIdx.x < nb) {
      const long long p = pos[b0 + threadIdx.x];
      if (p < 0) flag_device_error(kDevBounds);
      else t = (int)(p % q);
    }
    types[threadIdx.x] = t;
  }
  __syncthreads();

  const bool v0 = c0 < dout, v1 = c0 + 1 < dout;
  const int k0 = v0 ? (int)(c0 / bo) : 0, k1 = v1 ? (int)((c0 + 1) / bo) : 0;
  float acc0[kDecodeBT], acc1[kDecodeBT];
#pragma unroll
  for (int b = 0; b < kDecodeBT; ++b) { acc0[b] = 0.f; acc1[b] = 0.f; }

  for (long long j = warp; j < din; j += kDecodeWarps) {
    const int a = (int)(j / bi);
    // which (entry, column) pairs of this lane use group a
    unsigned m0 = 0, m1 = 0;
#pragma unroll
    for (int b = 0; b < kDecodeBT; ++b) {
      const int t = types[b];
      if (t < 0) continue;
      if (v0 && in_table(law, t, k0, a)) m0 |= 1u << b;
      if (v1 && in_table(law, t, k1, a)) m1 |= 1u << b;
    }
    if ((m0 | m1) == 0) continue;
    const float w0 = m0 ? dec_ld(W + j * ldw + c0) : 0.f;
    const float w1 = m1 ? dec_ld(W + j * ldw + c0 + 1) : 0.f;
#pragma unroll
    for (int b = 0; b < kDecodeBT; ++b) {
      if (!((m0 | m1) >> b & 1u)) continue;
      const float xv = dec_ld(x + (b0 + b) * ldx + j);
      if (m0 >> b & 1u) acc0[b] = fmaf(xv, w0, acc0[b]);
      if (m1 >> b & 1u) acc1[b] = fmaf(xv, w1, acc1[b]);
    }
  }
#pragma unroll
  for (int b = 0; b < kDecodeBT; ++b) {
    red[warp][b][2 * lane] = acc0[b];
    red[warp][b][2 * lane + 1] = acc1[b];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kDecodeBT * kDecodeCols; e += blockDim.x) {
    const int b = e / kDecodeCols, cc = e % kDecodeCols;
    const long long col = (long long)blockIdx.x * kDecodeCols + cc;
    if (b >= nb || col >= dout || types[b] < 0) continue;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) s += red[w][b][cc];
    dec_st(y + (b0 + b) * ldy + col, s);
  }
}

// Vectorised variant: every thread owns VEC adjacent columns (16 bytes of a
// weight row) and, per pass, keeps up to kRP independent 16-byte weight loads
// in flight before consuming them, so the stream is bandwidth- rather than
// latency-bound.  Thread (cv, rl): cv picks the column vector (4 per CTA), rl
// the row lane (64 per CTA, rows rl, rl + 64, ...).  Partial sums over the row
// lanes meet first through warp shuffles (8 row lanes per warp), then through
// shared memory (8 warps).
constexpr int kVecBB = 8;  // batch entries per CTA
constexpr int kRP = 8;     // weight rows per thread per pass

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& u, float* f);
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& u, float* f) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}

template <typename T>
__global__ void __launch_bounds__(256)
k_decode_vec(int law, int q, const int64_t* __restrict__ pos, int B, const T* __restrict__ x,
             long long ldx, const T* __restrict__ W, long long ldw, T* __restrict__ y,
             long long ldy, int bi, int bo, int din, int dout) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int CW = 4 * VEC;  // columns per CTA
  __shared__ int s_type[kVecBB];
  __shared__ float red[8][kVecBB][CW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cv = lane & 3, rl = warp * 8 + (lane >> 2);
  const int col = blockIdx.x * CW + cv * VEC;
  const bool cvalid = col < dout;
  const int k = cvalid ? col / bo : 0;
  const int b0 = blockIdx.y * kVecBB;

  if (threadIdx.x < kVecBB) {
    int t = -1;
    const int b = b0 + threadIdx.x;
    if (b < B) {
      const long long p = pos[b];
      if (p < 0) flag_device_error(kDevBounds);
      else t = (int)(p % q);
    }
    s_type[threadIdx.x] = t;
  }
  __syncthreads();
  int types[kVecBB];
#pragma unroll
  for (int b = 0; b < kVecBB; ++b) types[b] = s_type[b];

  float acc[kVecBB][VEC];
#pragma unroll
  for (int b = 0; b < kVecBB; ++b)
#pragma unroll
    for (int c = 0; c < VEC; ++c) acc[b][c] = 0.f;

  for (int j0 = 0; j0 < din; j0 += 64 * kRP) {
    uint4 wv[kRP];
    unsigned use[kRP];  // bit b: entry b of the tile needs this row
#pragma unroll
    for (int i = 0; i < kRP; ++i) {
      const int j = j0 + rl + 64 * i;
      unsigned m = 0;
      if (cvalid && j < din) {
        const int a = j / bi;
#pragma unroll
        for (int b = 0; b < kVecBB; ++b)
          if (types[b] >= 0 && in_table(law, types[b], k, a)) m |= 1u << b;
      }
      use[i] = m;
      if (m) wv[i] = __ldg(reinterpret_cast<const uint4*>(W + (long long)j * ldw + col));
    }
    float w[kRP][VEC];
#pragma unroll
    for (int i = 0; i < kRP; ++i) {
      if (use[i]) unpack16<T>(wv[i], w[i]);
      else
#pragma unroll
        for (int c = 0; c < VEC; ++c) w[i][c] = 0.f;
    }
    // one batch entry at a time: its kRP activations are independent loads
#pragma unroll
    for (int b = 0; b < kVecBB; ++b) {
      float xv[kRP];
#pragma unroll
      for (int i = 0; i < kRP; ++i) {
        const int j = j0 + rl + 64 * i;
        xv[i] = (use[i] >> b & 1u) ? dec_ld(x + (long long)(b0 + b) * ldx + j) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kRP; ++i)
#pragma unroll
        for (int c = 0; c < VEC; ++c) acc[b][c] = fmaf(xv[i], w[i][c], acc[b][c]);
    }
  }
  // reduce over the 8 row lanes of this warp (lane bits 2..4)
#pragma unroll
  for (int b = 0; b < kVecBB; ++b)
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
      float v = acc[b][c];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      acc[b][c] = v;
    }
  if ((lane >> 2) == 0) {
#pragma unroll
    for (int b = 0; b < kVecBB; ++b)
#pragma unroll
      for (int c = 0; c < VEC; ++c) red[warp][b][cv * VEC + c] = acc[b][c];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kVecBB * CW; e += blockDim.x) {
    const int b = e / CW, cc = e % CW;
    const int c = blockIdx.x * CW + cc;
    if (b0 + b >= B || c >= dout || s_type[b] < 0) continue;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += red[w][b][cc];
    dec_st(y + (long long)(b0 + b) * ldy + c, sum);
  }
}

// Split-K cluster variant (the default for aligned bf16 weights).  A
// thread-block cluster of CL CTAs shares one 64-column slab (inside one output
// group k) and one tile of TB batch entries; CTA z of the cluster streams
// weight rows [z*R, (z+1)*R).
//  - The batch is ranked by row type (ties by index) so that a tile, and the
//    NB entries of one thread, mostly share a type; a thread skips the rows
//    none of its entries needs, so arithmetic follows (2q-1)/q^2 of W.
//  - The first round of weight loads is issued before anything else.
//  - Activations are staged once with 16-byte loads, already masked by the
//    table (x[b][j] = 0 unless the group of j is in S(t_b, k)) and widened to
//    fp32.
//  - Partial sums meet through warp shuffles and shared memory; across the
//    cluster every CTA finalises an equal share of the outputs, reading its
//    peers' partial sums through distributed shared memory.
// Thread layout: cv = lane & 7 picks 8 columns; the 32 slots (warp, lane>>3)
// are split into BL batch lanes x RL row lanes; a thread owns NB entries.
constexpr int kMaxRowsCta = 192;  // multiple of 8
constexpr int kRound = 8;       // weight rows per thread per round
constexpr int kRankMax = 256;   // batches up to this size are ranked by type

template <int NB, int RL>
__global__ void __launch_bounds__(256)
k_decode_split(int law, int q, const int64_t* __restrict__ pos, int B,
               const __nv_bfloat16* __restrict__ x, long long ldx,
               const __nv_bfloat16* __restrict__ W, long long ldw, __nv_bfloat16* __restrict__ y,
               long long ldy, int bi, int bo, int din, int rows_per_cta) {
  constexpr int BL = 32 / RL;
  constexpr int TB = NB * BL;  // batch entries per CTA
  constexpr int CW = 64;
  __shared__ __align__(16) float xs[TB][kMaxRowsCta];  // masked fp32 activations
  __shared__ float red[RL == 32 ? 8 : 1][TB][CW];
  __shared__ int s_type[TB];
  __shared__ int s_idx[TB];
  __shared__ int s_tall[kRankMax];

  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cv = lane & 7, slot = warp * 4 + (lane >> 3);
  const int rl = slot % RL, bl = slot / RL;
  const int col0 = blockIdx.x * CW, col = col0 + cv * 8;
  const int k = col0 / bo;
  const int y0 = blockIdx.y * TB;
  const int r0 = blockIdx.z * rows_per_cta;
  const int r1 = min(din, r0 + rows_per_cta);
  const int R = r1 - r0;
  // 1. first round of weight rows, unconditionally
  uint4 wv[kRound];
#pragma unroll
  for (int u = 0; u < kRound; ++u) {
    const int j = r0 + rl + RL * u;
    if (j < r1) wv[u] = __ldg(reinterpret_cast<const uint4*>(W + (long long)j * ldw + col));
  }
  // 2. row types; the tile = entries of rank y0 .. y0+TB-1 in type order
  const bool ranked = B <= kRankMax;
  if (ranked) {
    for (int b = tid; b < B; b += blockDim.x) {
      const long long p = pos[b];
      s_tall[b] = p < 0 ? q : (int)(p % q);  // invalid positions sort last
    }
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) {
      const int t = s_tall[b];
      int r = 0;
      for (int c = 0; c < B; ++c) {
        const int u = s_tall[c];
        r += (u < t) || (u == t && c < b);
      }
      if (r >= y0 && r < y0 + TB) {
        s_idx[r - y0] = b;
        s_type[r - y0] = t < q ? t : -1;
        if (t >= q && blockIdx.x == 0 && blockIdx.z == 0) flag_device_error(kDevBounds);
      }
    }
    if (tid < TB && y0 + tid >= B) { s_idx[tid] = 0; s_type[tid] = -1; }
  } else if (tid < TB) {
    int t = -1;
    const int b = y0 + tid;
    if (b < B) {
      const long long p = pos[b];
      if (p < 0) { if (blockIdx.x == 0 && blockIdx.z == 0) flag_device_error(kDevBounds); }
      else t = (int)(p % q);
    }
    s_idx[tid] = b < B ? b : 0;
    s_type[tid] = t;
  }
  __syncthreads();

  // 3. masked, widened activations of this CTA's rows (16-byte loads; rows
  // of entries outside the batch stay unread)
  const int nvec = R >> 3;  // R is a multiple of 8 when this kernel runs
  const int nvalid = min(TB, B - y0);
  for (int e = tid; e < TB * nvec; e += blockDim.x) {
    const int i = e / nvec, v8 = e - i * nvec, jj = v8 * 8, j = r0 + jj;
    const int t = i < nvalid ? s_type[i] : -1;
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (t >= 0) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + (long long)s_idx[i] * ldx + j));
      unpack16<__nv_bfloat16>(u, f);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (!in_table(law, t, k, (j + m) / bi)) f[m] = 0.f;
    }
    float4* d = reinterpret_cast<float4*>(&xs[i][jj]);
    d[0] = make_float4(f[0], f[1], f[2], f[3]);
    d[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
  __syncthreads();

  int types[NB];
#pragma unroll
  for (int n = 0; n < NB; ++n) types[n] = s_type[bl * NB + n];
  float acc[NB][8];
#pragma unroll
  for (int n = 0; n < NB; ++n)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[n][c] = 0.f;

  for (int jr = r0 + rl; jr < r1; jr += RL * kRound) {
    uint4 nxt[kRound];
    const int jn = jr + RL * kRound;
#pragma unroll
    for (int u = 0; u < kRound; ++u) {  // next round in flight while this one computes
      const int j = jn + RL * u;
      if (j < r1) nxt[u] = __ldg(reinterpret_cast<const uint4*>(W + (long long)j * ldw + col));
    }
#pragma unroll
    for (int u = 0; u < kRound; ++u) {
      const int j = jr + RL * u;
      if (j >= r1) continue;
      const int a = j / bi;
      bool need = false;
#pragma unroll
      for (int n = 0; n < NB; ++n) need |= types[n] >= 0 && in_table(law, types[n], k, a);
      if (!need) continue;
      float w[8];
      unpack16<__nv_bfloat16>(wv[u], w);
#pragma unroll
      for (int n = 0; n < NB; ++n) {
        const float xv = xs[bl * NB + n][j - r0];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[n][c] = fmaf(xv, w[c], acc[n][c]);
      }
    }
#pragma unroll
    for (int u = 0; u < kRound; ++u) wv[u] = nxt[u];
  }

  // 5. reduce over the row lanes: shuffles over lane bits 3..4, then warps
#pragma unroll
  for (int n = 0; n < NB; ++n)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float v = acc[n][c];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      acc[n][c] = v;
    }
  const float* part;
  if constexpr (RL == 32) {
    if ((lane >> 3) == 0) {
#pragma unroll
      for (int n = 0; n < NB; ++n)
#pragma unroll
        for (int c = 0; c < 8; ++c) red[warp][n][cv * 8 + c] = acc[n][c];
    }
    __syncthreads();
    for (int e = tid; e < TB * CW; e += blockDim.x) {
      const int b = e / CW, cc = e % CW;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) sum += red[w][b][cc];
      red[0][b][cc] = sum;
    }
    part = &red[0][0][0];
  } else {  // RL == 4: each warp holds distinct entries after the shuffles
    if ((lane >> 3) == 0) {
#pragma unroll
      for (int n = 0; n < NB; ++n)
#pragma unroll
        for (int c = 0; c < 8; ++c) red[0][bl * NB + n][cv * 8 + c] = acc[n][c];
    }
    part = &red[0][0][0];
  }
  __syncthreads();

  // 4. across the cluster: CTA r sums outputs r, r + CL, ... of every CTA's
  // partials through distributed shared memory and writes them
  cluster.sync();
  const int cl = (int)cluster.num_blocks(), me = (int)cluster.block_rank();
  for (int e = me * blockDim.x + tid; e < TB * CW; e += cl * blockDim.x) {
    const int b = e / CW, cc = e % CW;
    if (y0 + b >= B || s_type[b] < 0) continue;
    float sum = 0.f;
    for (int r = 0; r < cl; ++r) sum += *cluster.map_shared_rank(part + e, r);
    y[(long long)s_idx[b] * ldy + col0 + cc] = __float2bfloat16_rn(sum);
  }
  cluster.sync();  // peers keep their shared memory until every CTA has read it
}

template <int NB, int RL>
static cudaError_t launch_split(const cudaLaunchConfig_t& cfg0, int cl, int law, int q,
                                const int64_t* positions, int B, const aal_mat& x,
                                const aal_mat& W, const aal_mat& y, int bi, int bo, int rows) {
  cudaLaunchConfig_t cfg = cfg0;
  constexpr int TB = NB * (32 / RL);
  cfg.gridDim.y = (unsigned)((B + TB - 1) / TB);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = cl;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_decode_split<NB, RL>, law, q, positions, B,
                            (const __nv_bfloat16*)x.ptr, x.ld, (const __nv_bfloat16*)W.ptr, W.ld,
                            (__nv_bfloat16*)y.ptr, y.ld, bi, bo, (int)x.cols, rows);
}

// Type-major variant (the default for aligned bf16 weights).  CTA (slab, t)
// owns a 32-column slab inside output group k and the batch entries of row
// type t: it gathers their indices, streams only the weight rows of the
// groups in S(t, k) (agihunt.info digest, multiplication-table paragraph) and
// computes the type's entries CH at a time from them, so no weight row is
// read for an entry that does not use it.  The chunk's activations on those
// rows are staged in shared memory as [row][entry] so that one weight row
// feeds CH entries x 8 columns of FMAs from CH/8 128-bit shared loads.
// Thread (cv, rl): cv = lane & 3 picks 8 of the 32 columns, rl =
// (warp, lane >> 2) one of 64 row lanes; partial sums over the row lanes meet
// through warp shuffles and shared memory.
constexpr int kTmMaxB = 1024;    // batch entries scanned per CTA
constexpr int kTmRound = 4;      // weight rows in flight per thread

template <int CH>
__global__ void __launch_bounds__(256)
k_decode_typed(int law, int q, const int64_t* __restrict__ pos, int B,
               const __nv_bfloat16* __restrict__ x, long long ldx,
               const __nv_bfloat16* __restrict__ W, long long ldw, __nv_bfloat16* __restrict__ y,
               long long ldy, int bi, int bo) {
  constexpr int XS = CH < 8 ? 8 : CH;  // entries per staged row (padded to 16 bytes)
  extern __shared__ __align__(16) uint8_t dsm[];
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(dsm);  // [needed row][XS]
  __shared__ float red[8][CH][32];
  __shared__ int s_idx[kTmMaxB];
  __shared__ int s_wbase[8];
  __shared__ int s_cnt;
  __shared__ int s_grp[4];
  __shared__ int s_ngrp;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cv = lane & 3, rl = warp * 8 + (lane >> 2);
  const int col0 = blockIdx.x * 32, col = col0 + cv * 8;
  const int k = col0 / bo;
  const int t = blockIdx.y;

  // 1. entries of type t (ballot compaction, order preserved)
  if (tid == 0) s_cnt = 0;
  __syncthreads();
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + tid;
    bool mine = false;
    if (b < B) {
      const long long p = pos[b];
      if (p < 0) {
        if (t == 0 && blockIdx.x == 0) flag_device_error(kDevBounds);
      } else {
        mine = (int)(p % q) == t;
      }
    }
    const unsigned m = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) s_wbase[warp] = __popc(m);
    __syncthreads();
    if (tid == 0) {
      int acc = s_cnt;
      for (int w = 0; w < 8; ++w) { const int c = s_wbase[w]; s_wbase[w] = acc; acc += c; }
      s_cnt = acc;
    }
    __syncthreads();
    if (mine) s_idx[s_wbase[warp] + __popc(m & ((1u << lane) - 1u))] = b;
    __syncthreads();
  }
  const int cnt = s_cnt;
  if (cnt == 0) return;
  // 2. the groups this type needs for output group k
  if (tid == 0) {
    int mem[4];
    s_ngrp = table_members(law, q, t, k, mem);
    for (int i = 0; i < s_ngrp; ++i) s_grp[i] = mem[i];
  }
  __syncthreads();
  const int ngrp = s_ngrp;
  const int nvec = bi >> 3;  // 8-row pieces per group

  for (int e0 = 0; e0 < cnt; e0 += CH) {
    const int ne = min(CH, cnt - e0);
    // 3. stage: item = (needed 8-row piece, entry); entries vary fastest
    for (int i = tid; i < XS * ngrp * nvec; i += blockDim.x) {
      const int e = i % XS, pv = i / XS, g = pv / nvec, r8 = (pv - g * nvec) * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (e < ne)
        v = __ldg(reinterpret_cast<const uint4*>(x + (long long)s_idx[e0 + e] * ldx + s_grp[g] * bi + r8));
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
      __nv_bfloat16* d = xs + (size_t)(g * bi + r8) * XS + e;
#pragma unroll
      for (int m = 0; m < 8; ++m) d[m * XS] = h[m];
    }
    __syncthreads();
    float acc[CH][8];
#pragma unroll
    for (int e = 0; e < CH; ++e)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[e][c] = 0.f;
    for (int g = 0; g < ngrp; ++g) {
      const __nv_bfloat16* wg = W + (long long)s_grp[g] * bi * ldw + col;
      const __nv_bfloat16* xg = xs + (size_t)g * bi * XS;
      for (int r0 = rl; r0 < bi; r0 += 64 * kTmRound) {
        uint4 wv[kTmRound];
#pragma unroll
        for (int u = 0; u < kTmRound; ++u) {
          const int r = r0 + 64 * u;
          if (r < bi) wv[u] = __ldg(reinterpret_cast<const uint4*>(wg + (long long)r * ldw));
        }
#pragma unroll
        for (int u = 0; u < kTmRound; ++u) {
          const int r = r0 + 64 * u;
          if (r >= bi) continue;
          float w[8];
          unpack16<__nv_bfloat16>(wv[u], w);
          const uint4* xr = reinterpret_cast<const uint4*>(xg + (size_t)r * XS);
#pragma unroll
          for (int e8 = 0; e8 < (CH + 7) / 8; ++e8) {
            float xf[8];
            unpack16<__nv_bfloat16>(xr[e8], xf);
#pragma unroll
            for (int m = 0; m < 8 && e8 * 8 + m < CH; ++m)
#pragma unroll
              for (int c = 0; c < 8; ++c) acc[e8 * 8 + m][c] = fmaf(xf[m], w[c], acc[e8 * 8 + m][c]);
          }
        }
      }
    }
    // 4. reduce over the 64 row lanes: shuffles over lane bits 2..4, then warps
#pragma unroll
    for (int e = 0; e < CH; ++e)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v = acc[e][c];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        acc[e][c] = v;
      }
    if ((lane >> 2) == 0) {
#pragma unroll
      for (int e = 0; e < CH; ++e)
#pragma unroll
        for (int c = 0; c < 8; ++c) red[warp][e][cv * 8 + c] = acc[e][c];
    }
    __syncthreads();
    for (int i = tid; i < ne * 32; i += blockDim.x) {
      const int e = i >> 5, cc = i & 31;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) sum += red[w][e][cc];
      y[(long long)s_idx[e0 + e] * ldy + col0 + cc] = __float2bfloat16_rn(sum);
    }
    __syncthreads();  // xs and red are reused by the next chunk
  }
}

template <int CH>
static cudaError_t launch_typed(int law, int q, const int64_t* positions, int B, const aal_mat& x,
                                const aal_mat& W, const aal_mat& y, int bi, int bo, long long dout,
                                cudaStream_t s) {
  constexpr int XS = CH < 8 ? 8 : CH;
  const size_t xs_bytes = (size_t)4 * bi * XS * 2;  // at most 4 groups of bi rows
  static unsigned long long attr_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done & bit)) {
    e = cudaFuncSetAttribute(k_decode_typed<CH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             160 * 1024);
    if (e != cudaSuccess) return e;
    attr_done |= bit;
  }
  dim3 grd((unsigned)(dout / 32), (unsigned)q);
  k_decode_typed<CH><<<grd, 256, xs_bytes, s>>>(law, q, positions, B, (const __nv_bfloat16*)x.ptr,
                                                x.ld, (const __nv_bfloat16*)W.ptr, W.ld,
                                                (__nv_bfloat16*)y.ptr, y.ld, bi, bo);
  return cudaGetLastError();
}


// ---------------------------------------------------------------------------
// Tensor-core decode.  A decode batch is a skinny product Y = X W in which
// entry b may only use the weight blocks (a, k) with a in S(t_b, k)
// (agihunt.info digest, multiplication-table paragraph and Transformer-mapping
// paragraph).  Writing it as a dense product whose activations are zeroed
// where the table says "not used" turns it into warp-level tensor-core MMAs
// (mma.sync m16n8k16, bf16 in, fp32 accumulate); the weight blocks that no
// entry of the batch needs are neither loaded nor multiplied, so HBM traffic
// stays the table's.  CTA (column tile, z) owns 64 output columns (inside one
// output group k) and the K slice z of the weight rows; the slices of one
// column tile form a thread-block cluster and each pushes its fp32 partial
// products into the shared memory of the CTA that owns the entry, which sums
// and writes it.
// Operand orientation: the MMA's M is the 64 output columns (A = W^T, read
// from the row-major weight tile with ldmatrix .trans), N the batch entries
// (B = X^T, rows of X), K the weight rows.
constexpr int kMmaCols = 64;      // output columns per CTA
constexpr int kMmaMaxB = 256;     // batch entries per launch
constexpr int kMmaMaxBGU = 128;   // batch entries per launch of the fused gate/up kernel
constexpr int kMmaKc = 192;       // weight rows staged per round, at most
constexpr int kMmaWStride = 72;   // staged weight row: 64 columns + 8 pad (144 bytes)
constexpr int kMmaPStride = 68;   // fp32 partial row: 64 columns + 4 pad

// Shared memory of the staging area (weight rows + activations) for rounds of
// kcr weight rows (a multiple of 16), 16-byte multiple.  Sizing it by the
// slice rather than the largest round lets two or three CTAs share an SM.
__host__ __device__ inline size_t mma_stage_bytes(int Bp, int nw, int kcr) {
  return (size_t)nw * kcr * kMmaWStride * 2 + (size_t)Bp * (kcr + 8) * 2;
}
__device__ __forceinline__ uint32_t dec_smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  // src_bytes 0 fills the 16 bytes with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
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
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// NT: n-tiles (8 entries) per warp; warps 0..3 take the four 16-column
// m-tiles, warps 4..7 the same m-tiles for the odd n-tiles.
// Latency is the cost at these sizes, so: each thread's position load is in
// flight while the first round's copies are issued (all weight rows of the
// round, the activations unmasked; later rounds fetch only the groups some
// entry uses); an entry's table row is applied to its operand fragment in
// registers; and the split-K partials are pushed into the owning CTA's
// shared memory, so one cluster barrier (whose arrival half is posted at the
// start) separates the MMAs from the sums and no CTA reads a peer afterwards.
// Entry n is owned (summed and written) by CTA n mod cl of the cluster.
// GU: the gate/up pair of a SwiGLU FFN in one launch: W is Wg and W2 is Wu
// (same shape and stride), both read against the same staged activations, and
// the owner writes y = silu(x Wg) * (x Wu) (agihunt.info digest, SwiGLU
// figures; the activation is applied to the fp32 sums, rounded once to bf16).
template <int NT, bool GU>
__global__ void __launch_bounds__(256)
k_decode_mma(int law, int q, const int64_t* __restrict__ pos, int B,
             const __nv_bfloat16* __restrict__ x, long long ldx,
             const __nv_bfloat16* __restrict__ W, const __nv_bfloat16* __restrict__ W2,
             long long ldw, __nv_bfloat16* __restrict__ y,
             long long ldy, int bi, int bo, int slice) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ int s_type[kMmaMaxB];
  __shared__ unsigned s_pres[8][2];
  __shared__ unsigned char s_used[64];  // groups of the CTA's K slice that some entry uses
  cg::cluster_group cluster = cg::this_cluster();
  // a launch that depends on this one (programmatic stream serialization)
  // may start now: it only prefetches its weights before waiting for us
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // every CTA of the cluster is running before any writes into a peer
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = blockIdx.x * kMmaCols;
  const int k = c0 / bo;
  const int ks0 = blockIdx.z * slice;  // first weight row of this CTA
  const int Bp = (B + 7) & ~7;
  const int ntiles = Bp >> 3;
  const int cl = (int)gridDim.z;
  const int rows_own = (Bp + cl - 1) / cl;  // entries owned per CTA (upper bound)
  const int kcr = min(kMmaKc, slice);      // weight rows per staging round
  const int xs_stride = kcr + 8;            // staged activation row, bf16
  constexpr int NW = GU ? 2 : 1;  // weight tiles staged per round
  __nv_bfloat16* Ws = reinterpret_cast<__nv_bfloat16*>(dsm);
  __nv_bfloat16* Xs = Ws + NW * kcr * kMmaWStride;
  // receive area: [operand][source rank][owned entry][64 columns] fp32, after staging
  float* R = reinterpret_cast<float*>(dsm + mma_stage_bytes(Bp, NW, kcr));
  const int g0 = ks0 / bi, ng = (ks0 + slice - 1) / bi - g0 + 1;

  // the position of entry tid is in flight while the copies are issued
  long long my_pos = -1;
  if (tid < B) my_pos = pos[tid];

  auto stage_w = [&](int r0, int rows, bool all_rows) {
    for (int i = tid; i < rows * 8; i += blockDim.x) {
      const int r = i >> 3, ch = i & 7;
      if (all_rows || s_used[(r0 + r) / bi - g0]) {
        cp_async16(dec_smem_u32(Ws + r * kMmaWStride + ch * 8),
                   W + (long long)(r0 + r) * ldw + c0 + ch * 8, 16);
        if (GU)
          cp_async16(dec_smem_u32(Ws + (kcr + r) * kMmaWStride + ch * 8),
                     W2 + (long long)(r0 + r) * ldw + c0 + ch * 8, 16);
      }
    }
  };
  auto stage_x = [&](int r0, int rows) {
    // item i = n * xch + ch, walked without a division per item
    const int xch = rows >> 3, dq = 256 / xch, dr = 256 - dq * xch;
    int n = tid / xch, ch = tid - n * xch;
    for (; n < Bp; n += dq, ch += dr) {
      if (ch >= xch) { ch -= xch; ++n; if (n >= Bp) break; }
      const bool in = n < B;
      cp_async16(dec_smem_u32(Xs + n * xs_stride + ch * 8),
                 in ? x + (long long)n * ldx + r0 + ch * 8 : x, in ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  // round 0's copies go out first.  When this launch depends on the previous
  // one (the down projection of an FFN decode step, launched with
  // programmatic stream serialization while the gate/up kernel still runs),
  // only the weights are fetched before griddepcontrol.wait: the activations
  // are that kernel's output.  Without such a dependency the wait returns at
  // once.
  stage_w(ks0, kcr, true);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  stage_x(ks0, kcr);

  // 1. row type of every entry (-1 for padding and invalid positions) and
  //    the set of types present
  int t = -1;
  if (tid < B) {
    if (my_pos < 0) {
      if (blockIdx.x == 0 && blockIdx.z == 0) flag_device_error(kDevBounds);
    } else {
      t = (int)(my_pos % q);
    }
  }
  if (tid < Bp) s_type[tid] = t;
  const unsigned lo = __reduce_or_sync(0xffffffffu, (t >= 0 && t < 32) ? 1u << t : 0u);
  const unsigned hi = __reduce_or_sync(0xffffffffu, t >= 32 ? 1u << (t - 32) : 0u);
  if (lane == 0) { s_pres[warp][0] = lo; s_pres[warp][1] = hi; }
  __syncthreads();
  // 2. which groups a of the slice some present type uses with output group k
  if (tid < ng) {
    unsigned long long pres = 0ull;
#pragma unroll
    for (int w = 0; w < 8; ++w)
      pres |= (unsigned long long)s_pres[w][0] | ((unsigned long long)s_pres[w][1] << 32);
    const int a = g0 + tid;
    bool u = false;
    for (int tt = 0; tt < q && !u; ++tt)
      if ((pres >> tt) & 1ull) u = in_table(law, tt, k, a);
    s_used[tid] = u ? 1 : 0;
  }

  float acc[NW][NT][4];
#pragma unroll
  for (int o = 0; o < NW; ++o)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[o][j][e] = 0.f;
  const int mt = warp & 3, nt0 = warp >> 2;
  const int g = lane >> 2;
  int my_t[NT];  // row types of the entries whose B fragments this thread holds
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int n = (nt0 + 2 * j) * 8 + g;
    my_t[j] = n < Bp ? s_type[n] : -1;
  }

  for (int kc = 0; kc < slice; kc += kcr) {
    const int rows = min(kcr, slice - kc);
    const int r0 = ks0 + kc;  // first weight row of this round
    if (kc > 0) {
      stage_w(r0, rows, false);
      stage_x(r0, rows);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    // 3. MMAs over the used 16-row steps; an entry whose table row does not
    //    use the step's group contributes zeros
    int a = r0 / bi, a_end = (a + 1) * bi - r0;  // group of step kk, and where it ends
    bool used = s_used[a - g0];
    unsigned keep = 0;  // bit j: entry of n-tile j uses group a
#pragma unroll
    for (int j = 0; j < NT; ++j)
      if (my_t[j] >= 0 && in_table(law, my_t[j], k, a)) keep |= 1u << j;
#pragma unroll 2
    for (int kk = 0; kk < rows; kk += 16) {
      if (kk >= a_end) {
        ++a;
        a_end += bi;
        used = s_used[a - g0];
        keep = 0;
#pragma unroll
        for (int j = 0; j < NT; ++j)
          if (my_t[j] >= 0 && in_table(law, my_t[j], k, a)) keep |= 1u << j;
      }
      if (!used) continue;
      uint32_t af[NW][4];
      const int arow = kk + (lane & 7) + ((lane >> 4) << 3);
      const int acol = mt * 16 + (((lane >> 3) & 1) << 3);
#pragma unroll
      for (int o = 0; o < NW; ++o)
        ldsm_x4_trans(dec_smem_u32(Ws + (o * kcr + arow) * kMmaWStride + acol), af[o]);
      uint32_t bf[NT][2];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const int nt = nt0 + 2 * j;
        if (nt < ntiles) {
          const int brow = nt * 8 + (lane & 7);
          const int bcol = kk + (((lane >> 3) & 1) << 3);
          ldsm_x2(dec_smem_u32(Xs + brow * xs_stride + bcol), bf[j]);
          if (!((keep >> j) & 1u)) { bf[j][0] = 0u; bf[j][1] = 0u; }
        }
      }
#pragma unroll
      for (int j = 0; j < NT; ++j)
        if (nt0 + 2 * j < ntiles) {
#pragma unroll
          for (int o = 0; o < NW; ++o) mma_bf16_16816(acc[o][j], af[o], bf[j]);
        }
    }
    if (kc + kcr < slice) __syncthreads();  // staging is refilled next round
  }
  // 4. push the fp32 partials to their owners: entry n -> CTA n mod cl,
  //    slot [this rank][n / cl]
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  const int c = lane & 3;
  const unsigned my_rank = cluster.block_rank();
  const int rstride = rows_own * kMmaPStride;  // floats per source rank
  const int ostride = cl * rstride;             // floats per operand
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int nt = nt0 + 2 * j;
    if (nt < ntiles) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int n = nt * 8 + 2 * c + e;
        float* dst = cluster.map_shared_rank(R, n % cl) + my_rank * rstride + (n / cl) * kMmaPStride;
        const int m = mt * 16 + g;
#pragma unroll
        for (int o = 0; o < NW; ++o) {
          dst[o * ostride + m] = acc[o][j][e];
          dst[o * ostride + m + 8] = acc[o][j][2 + e];
        }
      }
    }
  }
  cluster.sync();  // every partial has landed in its owner
  // 5. owners sum their entries over the cluster's ranks and write them
  for (int i = tid; i < rows_own * 16; i += blockDim.x) {
    const int jr = i >> 4, ch = i & 15;
    const int n = (int)my_rank + cl * jr;
    if (n >= B || s_type[n] < 0) continue;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < cl; ++r) {
      const float4 u = *reinterpret_cast<const float4*>(R + r * rstride + jr * kMmaPStride + ch * 4);
      v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
    }
    if (GU) {
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r = 0; r < cl; ++r) {
        const float4 u = *reinterpret_cast<const float4*>(R + ostride + r * rstride + jr * kMmaPStride + ch * 4);
        w.x += u.x; w.y += u.y; w.z += u.z; w.w += u.w;
      }
      // silu(g) * u = g / (1 + e^-g) * u
      v.x = __fdividef(v.x, 1.0f + __expf(-v.x)) * w.x;
      v.y = __fdividef(v.y, 1.0f + __expf(-v.y)) * w.y;
      v.z = __fdividef(v.z, 1.0f + __expf(-v.z)) * w.z;
      v.w = __fdividef(v.w, 1.0f + __expf(-v.w)) * w.w;
    }
    uint2 o;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
    h[0] = __floats2bfloat162_rn(v.x, v.y);
    h[1] = __floats2bfloat162_rn(v.z, v.w);
    *reinterpret_cast<uint2*>(y + (long long)n * ldy + c0 + ch * 4) = o;
  }
}

static size_t mma_smem_bytes(int Bp, int cl, int nw, int kcr) {
  const size_t recv = (size_t)nw * cl * ((Bp + cl - 1) / cl) * kMmaPStride * 4;
  return mma_stage_bytes(Bp, nw, kcr) + recv;
}

template <int NT, bool GU>
static cudaError_t launch_mma(int cl, int law, int q, const int64_t* positions, int B,
                              const aal_mat& x, const aal_mat& W, const aal_mat* W2, const aal_mat& y,
                              int bi, int bo, long long dout, cudaStream_t s, bool pdl = false) {
  constexpr int NW = GU ? 2 : 1;
  const int Bp = (B + 7) & ~7;
  const int slice = (int)(x.cols / cl);
  const size_t smem = mma_smem_bytes(Bp, cl, NW, slice < kMmaKc ? slice : kMmaKc);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static unsigned long long attr_done = 0;  // per device (bit dev % 64)
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done & bit)) {
    e = cudaFuncSetAttribute(k_decode_mma<NT, GU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)mma_smem_bytes(GU ? kMmaMaxBGU : kMmaMaxB, 8, NW, kMmaKc));
    if (e != cudaSuccess) return e;
    attr_done |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(dout / kMmaCols), 1, (unsigned)cl);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = cl;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_decode_mma<NT, GU>, law, q, positions, B,
                            (const __nv_bfloat16*)x.ptr, x.ld, (const __nv_bfloat16*)W.ptr,
                            (const __nv_bfloat16*)(GU ? W2->ptr : W.ptr), W.ld,
                            (__nv_bfloat16*)y.ptr, y.ld, bi, bo, slice);
}

static bool aligned16(const aal_mat& m) {
  return ((uintptr_t)m.ptr % 16) == 0 && m.ld % 8 == 0;
}

// AAL_DECODE_MMA=0 in the environment turns the tensor-core decode off.
static bool mma_disabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("AAL_DECODE_MMA");
    v = (e && e[0] == '0') ? 1 : 0;
  }
  return v == 1;
}

// AAL_DECODE_TYPED=0 in the environment selects the cluster kernel instead.
static bool typed_disabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("AAL_DECODE_TYPED");
    v = (e && e[0] == '0') ? 1 : 0;
  }
  return v == 1;
}

// Gate and up projections of a SwiGLU FFN for a decode batch in one launch,
// h = silu(x Wg) * (x Wu); batches above 128 entries go in chunks of 128.
aal_status decode_gate_up(int law, int q, const int64_t* positions, const aal_mat& x,
                          const aal_mat& Wg, const aal_mat& Wu, const aal_mat& h, cudaStream_t s,
                          bool* handled) {
  *handled = false;
  const long long B = x.rows, dout = Wg.cols;
  if (B == 0 || dout == 0) { *handled = true; return AAL_OK; }
  const int bi = (int)(x.cols / q), bo = (int)(dout / q);
  if (!(x.dtype == AAL_BF16 && Wg.dtype == AAL_BF16 && Wu.dtype == AAL_BF16 && h.dtype == AAL_BF16 &&
        q <= 64 && bo % kMmaCols == 0 && bi % 16 == 0 && aligned16(x) && aligned16(Wg) &&
        aligned16(Wu) && Wg.ld == Wu.ld && aligned16(h) && x.cols <= INT_MAX && dout <= INT_MAX &&
        !mma_disabled()))
    return AAL_OK;
  *handled = true;
  // split-K over an 8-CTA cluster (measured on B200 with the current kernel:
  // one FFN decode step at 64 entries 17.8 us with 8, 20.9 us with 4)
  int cl = 8;
  while (cl > 1 && (x.cols % (16 * cl)) != 0) cl >>= 1;
  for (long long b0 = 0; b0 < B; b0 += kMmaMaxBGU) {
    const int nb = (int)(B - b0 < kMmaMaxBGU ? B - b0 : kMmaMaxBGU);
    aal_mat xs = x, hs = h;
    xs.ptr = (char*)x.ptr + (size_t)b0 * x.ld * 2;
    xs.rows = nb;
    hs.ptr = (char*)h.ptr + (size_t)b0 * h.ld * 2;
    hs.rows = nb;
    cudaError_t e;
    if (nb <= 16) e = launch_mma<1, true>(cl, law, q, positions + b0, nb, xs, Wg, &Wu, hs, bi, bo, dout, s);
    else if (nb <= 64) e = launch_mma<4, true>(cl, law, q, positions + b0, nb, xs, Wg, &Wu, hs, bi, bo, dout, s);
    else e = launch_mma<8, true>(cl, law, q, positions + b0, nb, xs, Wg, &Wu, hs, bi, bo, dout, s);
    note_launch();
    if (e != cudaSuccess) return AAL_ERR_CUDA;
  }
  return AAL_OK;
}

aal_status decode_matvec(int law, int q, const int64_t* positions, const aal_mat& x,
                         const aal_mat& W, const aal_mat& y, cudaStream_t s, bool* handled, bool pdl) {
  *handled = true;
  const long long B = x.rows, dout = W.cols;
  if (B == 0 || dout == 0) return AAL_OK;
  const int bi = (int)(x.cols / q), bo = (int)(dout / q);
  const int es = x.dtype == AAL_F32 ? 4 : 2, vec = 16 / es;
  const bool vec_ok = ((uintptr_t)W.ptr % 16) == 0 && W.ld % vec == 0 && bo % vec == 0 &&
                      x.cols <= INT_MAX && dout <= INT_MAX && B <= INT_MAX;
  // tensor-core kernel: bf16, 64-column tiles inside one output group,
  // 16-row steps inside one input group, at most 256 entries
  if (x.dtype == AAL_BF16 && W.dtype == AAL_BF16 && y.dtype == AAL_BF16 && B <= kMmaMaxB &&
      q <= 64 && bo % kMmaCols == 0 && bi % 16 == 0 && aligned16(x) && aligned16(W) &&
      aligned16(y) && x.cols <= INT_MAX && dout <= INT_MAX && !mma_disabled()) {
    int cl = 8;
    while (cl > 1 && (x.cols % (16 * cl)) != 0) cl >>= 1;
    cudaError_t e;
    if (B <= 16) e = launch_mma<1, false>(cl, law, q, positions, (int)B, x, W, nullptr, y, bi, bo, dout, s, pdl);
    else if (B <= 64) e = launch_mma<4, false>(cl, law, q, positions, (int)B, x, W, nullptr, y, bi, bo, dout, s, pdl);
    else e = launch_mma<16, false>(cl, law, q, positions, (int)B, x, W, nullptr, y, bi, bo, dout, s, pdl);
    note_launch();
    return cuda_status(e);
  }
  // type-major kernel: bf16, 32-column slabs inside one group, groups a
  // multiple of 8 rows, at most 4 groups per table entry
  if (vec_ok && x.dtype == AAL_BF16 && bo % 32 == 0 && bi % 8 == 0 && B <= kTmMaxB && q <= 65535 &&
      x.ld % 8 == 0 && ((uintptr_t)x.ptr % 16) == 0 && (size_t)4 * bi * 16 * 2 <= 160 * 1024 &&
      !typed_disabled() && (B <= 4 || B > 16 || bo % 64 != 0)) {
    // measured on B200: the type-major kernel is fastest for small and large
    // batches; between them the cluster kernel below is
    cudaError_t e;
    if (B <= 1) e = launch_typed<1>(law, q, positions, (int)B, x, W, y, bi, bo, dout, s);
    else if (B <= 2) e = launch_typed<2>(law, q, positions, (int)B, x, W, y, bi, bo, dout, s);
    else if (B <= 4) e = launch_typed<4>(law, q, positions, (int)B, x, W, y, bi, bo, dout, s);
    else if (B <= 16) e = launch_typed<8>(law, q, positions, (int)B, x, W, y, bi, bo, dout, s);
    else e = launch_typed<16>(law, q, positions, (int)B, x, W, y, bi, bo, dout, s);
    note_launch();
    return cuda_status(e);
  }
  // fp32 stays on the exact vector path below
  if (vec_ok && x.dtype == AAL_BF16 && bo % 64 == 0) {
    int cl = 1;
    while (cl < 8 && (x.cols + cl - 1) / cl > kMaxRowsCta) cl <<= 1;
    const int rows = (int)(((x.cols + cl - 1) / cl + 7) / 8 * 8);
    if (rows <= kMaxRowsCta && x.cols % 8 == 0 && x.ld % 8 == 0 && ((uintptr_t)x.ptr % 16) == 0 &&
        (B + 7) / 8 <= 65535) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(dout / 64), 1, (unsigned)cl);
      cfg.blockDim = dim3(256);
      cfg.stream = s;
      const cudaError_t e =
          B <= 8 ? launch_split<8, 32>(cfg, cl, law, q, positions, (int)B, x, W, y, bi, bo, rows)
                 : launch_split<4, 4>(cfg, cl, law, q, positions, (int)B, x, W, y, bi, bo, rows);
      note_launch();
      return cuda_status(e);
    }
  }
  if (vec_ok) {
    dim3 grd((unsigned)((dout + 4 * vec - 1) / (4 * vec)), (unsigned)((B + kVecBB - 1) / kVecBB));
    if (grd.y <= 65535) {
      if (x.dtype == AAL_F32)
        k_decode_vec<float><<<grd, 256, 0, s>>>(law, q, positions, (int)B, (const float*)x.ptr,
                                                x.ld, (const float*)W.ptr, W.ld, (float*)y.ptr,
                                                y.ld, bi, bo, (int)x.cols, (int)dout);
      else
        k_decode_vec<__nv_bfloat16><<<grd, 256, 0, s>>>(
            law, q, positions, (int)B, (const __nv_bfloat16*)x.ptr, x.ld,
            (const __nv_bfloat16*)W.ptr, W.ld, (__nv_bfloat16*)y.ptr, y.ld, bi, bo, (int)x.cols,
            (int)dout);
      note_launch();
      return cuda_status(cudaGetLastError());
    }
  }
  dim3 grd((unsigned)((dout + kDecodeCols - 1) / kDecodeCols),
           (unsigned)((B + kDecodeBT - 1) / kDecodeBT));
  if (grd.y > 65535) { *handled = false; return AAL_ERR_UNSUPPORTED; }
  dim3 blk(kDecodeWarps * 32);
  if (x.dtype == AAL_F32)
    k_decode<float><<<grd, blk, 0, s>>>(law, q, positions, B, (const float*)x.ptr, x.ld,
                                        (const float*)W.ptr, W.ld, (float*)y.ptr, y.ld, bi, bo);
  else
    k_decode<__nv_bfloat16><<<grd, blk, 0, s>>>(law, q, positions, B,
                                                (const __nv_bfloat16*)x.ptr, x.ld,
                                                (const __nv_bfloat16*)W.ptr, W.ld,
                                                (__nv_bfloat16*)y.ptr, y.ld, bi, bo);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace aal
