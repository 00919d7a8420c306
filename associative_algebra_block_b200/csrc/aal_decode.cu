// Decode step: one new token per batch entry, y_b = row t_b of the table
// applied to x_b (agihunt.info digest: decoding evaluates only the new
// position's row, as a matrix-vector product with a kernel of its own).
//
// The work is a stream over the weight rows that some entry of the batch
// needs.  A CTA owns a 64-column slab of W and a tile of up to kDecodeBT batch
// entries; its 8 warps split the weight rows, every lane owns two adjacent
// columns, and the warps' partial sums meet in shared memory.  A weight row is
// loaded only when some entry of the tile needs its group for one of the
// lane's columns, so one row type touches (2q-1)/q^2 of W (9/16 for Q2xQ2).
#include "aal_internal.h"

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

aal_status decode_matvec(int law, int q, const int64_t* positions, const aal_mat& x,
                         const aal_mat& W, const aal_mat& y, cudaStream_t s, bool* handled) {
  *handled = true;
  const long long B = x.rows, dout = W.cols;
  if (B == 0 || dout == 0) return AAL_OK;
  const int bi = (int)(x.cols / q), bo = (int)(dout / q);
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
