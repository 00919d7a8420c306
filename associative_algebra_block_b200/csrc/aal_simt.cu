// General CUDA path: one thread per output element, fp32 accumulation.
//
// Serves every call for any shape the header allows: fp32 (the Q_2 fp32
// workload), explicit row types, sequence lengths that are not a multiple of
// q, and the ragged tail rows the tensor-core path leaves.  The loops follow
// the table directly: output block (t, k) of a row of type t sums x_a W_ak
// over a in S(t, k) (agihunt.info digest, multiplication-table paragraph).
#include "aal_internal.h"

namespace aal {

__device__ __forceinline__ float ld_elem(const float* p) { return *p; }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// --------------------------------------------------------------------------
// Y[r, c] = sum_{a in S(t_r, k)} sum_j X[r, a*bi + j] W[a*bi + j, c], k = c / bo
// Rows [row_begin, rows) only.
// --------------------------------------------------------------------------
template <typename T>
__global__ void k_project(int law, int q, RowTypes rt, long long row_begin, long long rows,
                          const T* __restrict__ X, long long ldx, const T* __restrict__ W,
                          long long ldw, T* __restrict__ Y, long long ldy, int bi, int bo) {
  const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long r = row_begin + (long long)blockIdx.y * blockDim.y + threadIdx.y;
  const long long dout = (long long)bo * q;
  if (c >= dout || r >= rows) return;
  const int t = row_type(rt, r);
  if (t < 0) return;
  const int k = (int)(c / bo);
  int members[4];
  const int n = table_members(law, q, t, k, members);
  float acc = 0.f;
  for (int m = 0; m < n; ++m) {
    const long long j0 = (long long)members[m] * bi;
    const T* xr = X + r * ldx + j0;
    const T* wc = W + j0 * ldw + c;
    for (int j = 0; j < bi; ++j) acc = fmaf(ld_elem(xr + j), ld_elem(wc + (long long)j * ldw), acc);
  }
  st_elem(Y + r * ldy + c, acc);
}

// H[r, c] = silu(G) * U with G, U the row-typed projections through Wg, Wu.
template <typename T>
__global__ void k_swiglu_gate_up(int law, int q, RowTypes rt, long long rows,
                                 const T* __restrict__ X, long long ldx,
                                 const T* __restrict__ Wg, long long ldg,
                                 const T* __restrict__ Wu, long long ldu,
                                 T* __restrict__ H, long long ldh, int bi, int bo) {
  const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long r = (long long)blockIdx.y * blockDim.y + threadIdx.y;
  const long long F = (long long)bo * q;
  if (c >= F || r >= rows) return;
  const int t = row_type(rt, r);
  if (t < 0) return;
  const int k = (int)(c / bo);
  int members[4];
  const int n = table_members(law, q, t, k, members);
  float g = 0.f, u = 0.f;
  for (int m = 0; m < n; ++m) {
    const long long j0 = (long long)members[m] * bi;
    const T* xr = X + r * ldx + j0;
    for (int j = 0; j < bi; ++j) {
      const float xv = ld_elem(xr + j);
      g = fmaf(xv, ld_elem(Wg + (j0 + j) * ldg + c), g);
      u = fmaf(xv, ld_elem(Wu + (j0 + j) * ldu + c), u);
    }
  }
  const float h = g / (1.f + expf(-g)) * u;
  st_elem(H + r * ldh + c, h);
}

// dX[r, j] for j in group a: sum over k with a in S(t, k) of
// sum_c dY[r, k*bo + c] W[j, k*bo + c].
template <typename T>
__global__ void k_bwd_dx(int law, int q, RowTypes rt, long long rows, const T* __restrict__ dY,
                         long long ldy, const T* __restrict__ W, long long ldw, T* __restrict__ dX,
                         long long ldx, int bi, int bo, int accumulate) {
  const long long j = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long r = (long long)blockIdx.y * blockDim.y + threadIdx.y;
  const long long din = (long long)bi * q;
  if (j >= din || r >= rows) return;
  const int t = row_type(rt, r);
  if (t < 0) return;
  const int a = (int)(j / bi);
  float acc = 0.f;
  for (int k = 0; k < q; ++k) {
    if (!in_table(law, t, k, a)) continue;
    const T* dyr = dY + r * ldy + (long long)k * bo;
    const T* wr = W + j * ldw + (long long)k * bo;
    for (int c = 0; c < bo; ++c) acc = fmaf(ld_elem(dyr + c), ld_elem(wr + c), acc);
  }
  if (accumulate) acc += ld_elem(dX + r * ldx + j);
  st_elem(dX + r * ldx + j, acc);
}

// SiLU' chain of the SwiGLU backward, elementwise on rows of a valid type:
// dG holds dH on entry; dG = dH u silu'(g) and dU = dH silu(g) on exit, with
// silu'(g) = s (1 + g (1 - s)), s = 1 / (1 + e^-g).
template <typename T>
__global__ void k_swiglu_bwd_act(int q, RowTypes rt, long long rows, long long F,
                                 const T* __restrict__ G, long long ldg, const T* __restrict__ U,
                                 long long ldu, T* __restrict__ dG, long long lddg,
                                 T* __restrict__ dU, long long lddu) {
  const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long r = (long long)blockIdx.y * blockDim.y + threadIdx.y;
  if (c >= F || r >= rows) return;
  if (row_type(rt, r) < 0) return;
  const float g = ld_elem(G + r * ldg + c), u = ld_elem(U + r * ldu + c);
  const float dh = ld_elem(dG + r * lddg + c);
  const float sg = 1.f / (1.f + expf(-g));
  st_elem(dU + r * lddu + c, dh * g * sg);
  st_elem(dG + r * lddg + c, dh * u * sg * (1.f + g * (1.f - sg)));
}

// dW[j, c] (block (a, k)) = sum over rows r with a in S(t_r, k) of X[r, j] dY[r, c].
template <typename T>
__global__ void k_bwd_dw(int law, int q, RowTypes rt, long long rows, const T* __restrict__ X,
                         long long ldx, const T* __restrict__ dY, long long ldy,
                         T* __restrict__ dW, long long ldw, int bi, int bo, int accumulate) {
  const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long j = (long long)blockIdx.y * blockDim.y + threadIdx.y;
  const long long din = (long long)bi * q, dout = (long long)bo * q;
  if (c >= dout || j >= din) return;
  const int a = (int)(j / bi), k = (int)(c / bo);
  float acc = 0.f;
  for (long long r = 0; r < rows; ++r) {
    const int t = row_type(rt, r);
    if (t < 0 || !in_table(law, t, k, a)) continue;
    acc = fmaf(ld_elem(X + r * ldx + j), ld_elem(dY + r * ldy + c), acc);
  }
  T* out = dW + j * ldw + c;
  if (accumulate) acc += ld_elem(out);
  st_elem(out, acc);
}

// Z[row, col] = sum_{a in S(i, k)} sum_j X[row, a*b + j] W[a*b + j, col],
// i = row / b, k = col / b.
template <typename T>
__global__ void k_square(int law, int q, long long n, const T* __restrict__ X, long long ldx,
                         const T* __restrict__ W, long long ldw, T* __restrict__ Z, long long ldz,
                         int b) {
  const long long col = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = (long long)blockIdx.y * blockDim.y + threadIdx.y;
  if (col >= n || row >= n) return;
  const int i = (int)(row / b), k = (int)(col / b);
  int members[4];
  const int m = table_members(law, q, i, k, members);
  float acc = 0.f;
  for (int s = 0; s < m; ++s) {
    const long long j0 = (long long)members[s] * b;
    const T* xr = X + row * ldx + j0;
    const T* wc = W + j0 * ldw + col;
    for (int j = 0; j < b; ++j) acc = fmaf(ld_elem(xr + j), ld_elem(wc + (long long)j * ldw), acc);
  }
  st_elem(Z + row * ldz + col, acc);
}

// --------------------------------------------------------------------------
// Launchers
// --------------------------------------------------------------------------
static dim3 grid2(long long nx, long long ny, dim3 blk) {
  return dim3((unsigned)((nx + blk.x - 1) / blk.x), (unsigned)((ny + blk.y - 1) / blk.y));
}

static bool grid_ok(long long nx, long long ny, dim3 blk) {
  return (ny + blk.y - 1) / blk.y <= 65535 && (nx + blk.x - 1) / blk.x <= 0x7fffffffLL;
}

aal_status simt_project_rows(int law, int q, const RowTypes& rt, long long row_begin,
                             const aal_mat& X, const aal_mat& W, const aal_mat& Y, cudaStream_t s) {
  const long long rows = X.rows, dout = W.cols;
  const int bi = (int)(X.cols / q), bo = (int)(dout / q);
  if (rows <= row_begin || dout == 0) return AAL_OK;
  dim3 blk(32, 8);
  if (!grid_ok(dout, rows - row_begin, blk)) return AAL_ERR_UNSUPPORTED;
  dim3 grd = grid2(dout, rows - row_begin, blk);
  if (X.dtype == AAL_F32)
    k_project<float><<<grd, blk, 0, s>>>(law, q, rt, row_begin, rows, (const float*)X.ptr, X.ld,
                                         (const float*)W.ptr, W.ld, (float*)Y.ptr, Y.ld, bi, bo);
  else
    k_project<__nv_bfloat16><<<grd, blk, 0, s>>>(law, q, rt, row_begin, rows,
                                                 (const __nv_bfloat16*)X.ptr, X.ld,
                                                 (const __nv_bfloat16*)W.ptr, W.ld,
                                                 (__nv_bfloat16*)Y.ptr, Y.ld, bi, bo);
  note_launch();
  return cuda_status(cudaGetLastError());
}

aal_status simt_project(int law, int q, const RowTypes& rt, const aal_mat& X, const aal_mat& W,
                        const aal_mat& Y, cudaStream_t s) {
  return simt_project_rows(law, q, rt, 0, X, W, Y, s);
}

aal_status simt_swiglu_gate_up(int law, int q, const RowTypes& rt, const aal_mat& X,
                               const aal_mat& Wg, const aal_mat& Wu, const aal_mat& H,
                               cudaStream_t s) {
  const long long rows = X.rows, F = Wg.cols;
  const int bi = (int)(X.cols / q), bo = (int)(F / q);
  if (rows == 0 || F == 0) return AAL_OK;
  dim3 blk(32, 8);
  if (!grid_ok(F, rows, blk)) return AAL_ERR_UNSUPPORTED;
  dim3 grd = grid2(F, rows, blk);
  if (X.dtype == AAL_F32)
    k_swiglu_gate_up<float><<<grd, blk, 0, s>>>(law, q, rt, rows, (const float*)X.ptr, X.ld,
                                                (const float*)Wg.ptr, Wg.ld, (const float*)Wu.ptr,
                                                Wu.ld, (float*)H.ptr, H.ld, bi, bo);
  else
    k_swiglu_gate_up<__nv_bfloat16><<<grd, blk, 0, s>>>(
        law, q, rt, rows, (const __nv_bfloat16*)X.ptr, X.ld, (const __nv_bfloat16*)Wg.ptr, Wg.ld,
        (const __nv_bfloat16*)Wu.ptr, Wu.ld, (__nv_bfloat16*)H.ptr, H.ld, bi, bo);
  note_launch();
  return cuda_status(cudaGetLastError());
}

aal_status simt_project_bwd_dx(int law, int q, const RowTypes& rt, const aal_mat& dY,
                               const aal_mat& W, const aal_mat& dX, cudaStream_t s, int accumulate) {
  const long long rows = dY.rows, din = W.rows;
  const int bi = (int)(din / q), bo = (int)(W.cols / q);
  if (rows == 0 || din == 0) return AAL_OK;
  dim3 blk(32, 8);
  if (!grid_ok(din, rows, blk)) return AAL_ERR_UNSUPPORTED;
  dim3 grd = grid2(din, rows, blk);
  if (dY.dtype == AAL_F32)
    k_bwd_dx<float><<<grd, blk, 0, s>>>(law, q, rt, rows, (const float*)dY.ptr, dY.ld,
                                        (const float*)W.ptr, W.ld, (float*)dX.ptr, dX.ld, bi, bo,
                                        accumulate);
  else
    k_bwd_dx<__nv_bfloat16><<<grd, blk, 0, s>>>(law, q, rt, rows, (const __nv_bfloat16*)dY.ptr,
                                                dY.ld, (const __nv_bfloat16*)W.ptr, W.ld,
                                                (__nv_bfloat16*)dX.ptr, dX.ld, bi, bo, accumulate);
  note_launch();
  return cuda_status(cudaGetLastError());
}

aal_status simt_swiglu_bwd_act(int q, const RowTypes& rt, const aal_mat& G, const aal_mat& U,
                               const aal_mat& dG, const aal_mat& dU, cudaStream_t s) {
  const long long rows = G.rows, F = G.cols;
  if (rows == 0 || F == 0) return AAL_OK;
  dim3 blk(32, 8);
  if (!grid_ok(F, rows, blk)) return AAL_ERR_UNSUPPORTED;
  dim3 grd = grid2(F, rows, blk);
  if (G.dtype == AAL_F32)
    k_swiglu_bwd_act<float><<<grd, blk, 0, s>>>(q, rt, rows, F, (const float*)G.ptr, G.ld,
                                                (const float*)U.ptr, U.ld, (float*)dG.ptr, dG.ld,
                                                (float*)dU.ptr, dU.ld);
  else
    k_swiglu_bwd_act<__nv_bfloat16><<<grd, blk, 0, s>>>(
        q, rt, rows, F, (const __nv_bfloat16*)G.ptr, G.ld, (const __nv_bfloat16*)U.ptr, U.ld,
        (__nv_bfloat16*)dG.ptr, dG.ld, (__nv_bfloat16*)dU.ptr, dU.ld);
  note_launch();
  return cuda_status(cudaGetLastError());
}

aal_status simt_project_bwd_dw(int law, int q, const RowTypes& rt, const aal_mat& X,
                               const aal_mat& dY, const aal_mat& dW, int accumulate,
                               cudaStream_t s) {
  const long long rows = X.rows, din = dW.rows, dout = dW.cols;
  const int bi = (int)(din / q), bo = (int)(dout / q);
  if (din == 0 || dout == 0) return AAL_OK;
  dim3 blk(32, 8);
  if (!grid_ok(dout, din, blk)) return AAL_ERR_UNSUPPORTED;
  dim3 grd = grid2(dout, din, blk);
  if (X.dtype == AAL_F32)
    k_bwd_dw<float><<<grd, blk, 0, s>>>(law, q, rt, rows, (const float*)X.ptr, X.ld,
                                        (const float*)dY.ptr, dY.ld, (float*)dW.ptr, dW.ld, bi, bo,
                                        accumulate);
  else
    k_bwd_dw<__nv_bfloat16><<<grd, blk, 0, s>>>(law, q, rt, rows, (const __nv_bfloat16*)X.ptr,
                                                X.ld, (const __nv_bfloat16*)dY.ptr, dY.ld,
                                                (__nv_bfloat16*)dW.ptr, dW.ld, bi, bo, accumulate);
  note_launch();
  return cuda_status(cudaGetLastError());
}

aal_status simt_square(int law, int q, const aal_mat& X, const aal_mat& W, const aal_mat& Z,
                       cudaStream_t s) {
  const long long n = X.rows;
  const int b = (int)(n / q);
  if (n == 0) return AAL_OK;
  dim3 blk(32, 8);
  if (!grid_ok(n, n, blk)) return AAL_ERR_UNSUPPORTED;
  dim3 grd = grid2(n, n, blk);
  if (X.dtype == AAL_F32)
    k_square<float><<<grd, blk, 0, s>>>(law, q, n, (const float*)X.ptr, X.ld, (const float*)W.ptr,
                                        W.ld, (float*)Z.ptr, Z.ld, b);
  else
    k_square<__nv_bfloat16><<<grd, blk, 0, s>>>(law, q, n, (const __nv_bfloat16*)X.ptr, X.ld,
                                                (const __nv_bfloat16*)W.ptr, W.ld,
                                                (__nv_bfloat16*)Z.ptr, Z.ld, b);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace aal
