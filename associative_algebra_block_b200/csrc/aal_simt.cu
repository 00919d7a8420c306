// General CUDA path, fp32 accumulation.
//
// Serves every call for any shape the header allows: fp32 (the Q_2 fp32
// workload), explicit row types without a workspace, sequence lengths that
// are not a multiple of q, the backward with such rules, and shapes the
// tensor-core path does not take.  The sums follow the table directly: output
// block (t, k) of a row of type t sums x_a W_ak over a in S(t, k) (agihunt.info
// digest, multiplication-table paragraph).  Projections and dX with at least
// half a tile of rows, and every dW, run on shared-memory tiles that keep only
// the rows each table entry applies to; small calls (decode rows) and the
// SwiGLU and square-product kernels compute one output per thread.
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

// Y (kDx false) or dX (kDx true) on tiles of 64 rows by up to 64 outputs of
// one group g, 256 threads of 4 x 4 products.  For each group m of the
// contraction the tile keeps the rows whose type t has the table entry (Y:
// m in S(t, g); dX: g in S(t, m)), stages their operand slices 32 contraction
// steps at a time beside the matching weight slice, and adds the products to
// an accumulator in shared memory; the work follows the table row by row and
// every weight element is read once per tile.
//   Y:  A = X,  contraction group width L = bi, output group width G = bo,
//       weight W[m*bi + c, g*bo + f]
//   dX: A = dY, L = bo, G = bi, weight W[g*bi + f, m*bo + c]
constexpr int kRtRows = 64, kRtOut = 64, kRtK = 32;
template <typename T, bool kDx>
__global__ void __launch_bounds__(256) k_rows_tiled(int law, int q, RowTypes rt, long long row_begin,
                                                    long long rows, const T* __restrict__ A, long long lda,
                                                    const T* __restrict__ W, long long ldw, T* __restrict__ O,
                                                    long long ldo, int L, int G, int accumulate) {
  __shared__ float acc_s[kRtRows][kRtOut + 1];
  __shared__ float as[kRtRows][kRtK + 1];
  __shared__ float bs[kRtOut][kRtK + 1];
  __shared__ int s_t[kRtRows];
  __shared__ int s_idx[kRtRows];
  __shared__ unsigned s_mask[kRtRows / 32];
  const int ot_per = (G + kRtOut - 1) / kRtOut;
  const int g = (int)(blockIdx.x / (unsigned)ot_per);
  const int o_lo = (int)(blockIdx.x - (unsigned)g * ot_per) * kRtOut;
  const int no = G - o_lo < kRtOut ? G - o_lo : kRtOut;
  const long long r0 = row_begin + (long long)blockIdx.y * kRtRows;
  const int nr = (int)(rows - r0 < kRtRows ? rows - r0 : kRtRows);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int e = tid; e < kRtRows * (kRtOut + 1); e += 256) (&acc_s[0][0])[e] = 0.f;
  if (tid < kRtRows) s_t[tid] = tid < nr ? row_type(rt, r0 + tid) : -1;
  __syncthreads();
  for (int m = 0; m < q; ++m) {
    // the rows of the tile that take part in group m, packed in row order
    if (tid < kRtRows) {
      const int t = s_t[tid];
      const bool keep = t >= 0 && (kDx ? in_table(law, t, m, g) : in_table(law, t, g, m));
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if ((tid & 31) == 0) s_mask[tid >> 5] = bal;
    }
    __syncthreads();
    const unsigned m0 = s_mask[0], m1 = s_mask[1];
    const int n = __popc(m0) + __popc(m1);
    if (n > 0) {
      if (tid < kRtRows) {
        const unsigned mine = tid < 32 ? m0 : m1;
        const int bit = tid & 31;
        if ((mine >> bit) & 1u)
          s_idx[(tid < 32 ? 0 : __popc(m0)) + __popc(mine & ((1u << bit) - 1u))] = tid;
      }
      __syncthreads();
      float part[4][4] = {};
      for (int c0 = 0; c0 < L; c0 += kRtK) {
        const int nc = L - c0 < kRtK ? L - c0 : kRtK;
        for (int e = tid; e < n * kRtK; e += 256) {
          const int sl = e / kRtK, cc = e - sl * kRtK;
          as[sl][cc] = cc < nc ? ld_elem(A + (r0 + s_idx[sl]) * lda + (long long)m * L + c0 + cc) : 0.f;
        }
        for (int e = tid; e < kRtOut * kRtK; e += 256) {
          // consecutive threads take consecutive elements of the weight's rows
          const int f = kDx ? e / kRtK : e % kRtOut, cc = kDx ? e % kRtK : e / kRtOut;
          float v = 0.f;
          if (f < no && cc < nc)
            v = kDx ? ld_elem(W + ((long long)g * G + o_lo + f) * ldw + (long long)m * L + c0 + cc)
                    : ld_elem(W + ((long long)m * L + c0 + cc) * ldw + (long long)g * G + o_lo + f);
          bs[f][cc] = v;
        }
        __syncthreads();
        // a thread whose first slot is past the kept rows has none (slots ty + 16 u)
        for (int cc = 0; cc < (ty < n ? nc : 0); ++cc) {
          float av[4], bv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            av[u] = as[ty + 16 * u][cc];
            bv[u] = bs[tx + 16 * u][cc];
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) part[u][v] = fmaf(av[u], bv[v], part[u][v]);
        }
        __syncthreads();
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int sl = ty + 16 * u;
        if (sl < n) {
          const int i = s_idx[sl];
#pragma unroll
          for (int v = 0; v < 4; ++v) acc_s[i][tx + 16 * v] += part[u][v];
        }
      }
    }
    __syncthreads();  // before the masks and the packed rows are rewritten
  }
  for (int e = tid; e < kRtRows * kRtOut; e += 256) {
    const int i = e / kRtOut, f = e - i * kRtOut;
    if (i < nr && f < no && s_t[i] >= 0) {
      T* out = O + (r0 + i) * ldo + (long long)g * G + o_lo + f;
      float v = acc_s[i][f];
      if (accumulate) v += ld_elem(out);
      st_elem(out, v);
    }
  }
}

// Launches k_rows_tiled when the rows fill at least half a tile, q is small
// enough and the grid fits; returns false (nothing launched) otherwise.  Each
// of the q contraction groups stages its whole weight slice whatever the
// number of rows it applies to, so the tiles pay off for small q only: the
// projection at q <= 8 (Q2xQ2 pilot shape 4.06 -> 1.25 ms; at q = 16 one
// output a thread was faster), dX at q <= 32 (q = 16: 1.51 -> 0.30 ms).
template <bool kDx>
static bool launch_rows_tiled(int law, int q, const RowTypes& rt, long long row_begin, long long rows,
                              const aal_mat& A, const aal_mat& W, const aal_mat& O, int L, int G,
                              int accumulate, cudaStream_t s) {
  const long long n = rows - row_begin;
  const long long gx = (long long)q * ((G + kRtOut - 1) / kRtOut), gy = (n + kRtRows - 1) / kRtRows;
  if (q > (kDx ? 32 : 8)) return false;
  if (n < kRtRows / 2 || G <= 0 || gx > 0x7fffffffLL || gy > 65535) return false;
  const dim3 grd((unsigned)gx, (unsigned)gy);
  if (A.dtype == AAL_F32)
    k_rows_tiled<float, kDx><<<grd, 256, 0, s>>>(law, q, rt, row_begin, rows, (const float*)A.ptr, A.ld,
                                                 (const float*)W.ptr, W.ld, (float*)O.ptr, O.ld, L, G,
                                                 accumulate);
  else
    k_rows_tiled<__nv_bfloat16, kDx><<<grd, 256, 0, s>>>(
        law, q, rt, row_begin, rows, (const __nv_bfloat16*)A.ptr, A.ld, (const __nv_bfloat16*)W.ptr, W.ld,
        (__nv_bfloat16*)O.ptr, O.ld, L, G, accumulate);
  return true;
}

// The same dW on tiles that each lie inside one block (a, k): up to 64 of
// group a's features by up to 64 of group k's columns, 256 threads of 4 x 4
// outputs.  The tile walks the rows 32 at a time; a warp keeps the rows of the
// step whose type t has a in S(t, k), packed to the front of shared memory
// with their X and dY slices, so the tile does only the products the table
// asks for (every row for a diagonal block, under Q_q the rows of type a or k
// for the others) with every operand read once per tile.
constexpr int kDwTile = 64, kDwRows = 32;
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_dw_tiled(int law, int q, RowTypes rt, long long rows,
                                                      const T* __restrict__ X, long long ldx,
                                                      const T* __restrict__ dY, long long ldy,
                                                      T* __restrict__ dW, long long ldw, int bi, int bo,
                                                      int accumulate) {
  __shared__ float xs[kDwRows][kDwTile];
  __shared__ float ys[kDwRows][kDwTile];
  __shared__ long long rs[kDwRows];
  __shared__ int s_n;
  const int jt_per = (bi + kDwTile - 1) / kDwTile, ct_per = (bo + kDwTile - 1) / kDwTile;
  const int a = (int)(blockIdx.x / jt_per), k = (int)(blockIdx.y / ct_per);
  const int j_lo = (int)(blockIdx.x - (unsigned)a * jt_per) * kDwTile;  // within group a
  const int c_lo = (int)(blockIdx.y - (unsigned)k * ct_per) * kDwTile;  // within group k
  const int nj = bi - j_lo < kDwTile ? bi - j_lo : kDwTile;
  const int nc = bo - c_lo < kDwTile ? bo - c_lo : kDwTile;
  const long long j0 = (long long)a * bi + j_lo, c0 = (long long)k * bo + c_lo;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  for (long long r0 = 0; r0 < rows; r0 += kDwRows) {
    if (tid < 32) {
      const long long r = r0 + tid;
      const int t = r < rows ? row_type(rt, r) : -1;
      const bool keep = t >= 0 && in_table(law, t, k, a);
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) rs[__popc(m & ((1u << tid) - 1u))] = r;
      if (tid == 0) s_n = __popc(m);
    }
    __syncthreads();
    const int n = s_n;
    for (int e = tid; e < n * kDwTile; e += 256) {
      const int i = e / kDwTile, x = e - i * kDwTile;
      const long long r = rs[i];
      xs[i][x] = x < nj ? ld_elem(X + r * ldx + j0 + x) : 0.f;
      ys[i][x] = x < nc ? ld_elem(dY + r * ldy + c0 + x) : 0.f;
    }
    __syncthreads();
    for (int i = 0; i < n; ++i) {
      float xv[4], yv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        xv[u] = xs[i][ty + 16 * u];
        yv[u] = ys[i][tx + 16 * u];
      }
#pragma unroll
      for (int uj = 0; uj < 4; ++uj)
#pragma unroll
        for (int uc = 0; uc < 4; ++uc) acc[uj][uc] = fmaf(xv[uj], yv[uc], acc[uj][uc]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int uj = 0; uj < 4; ++uj) {
    const int jj = ty + 16 * uj;
    if (jj >= nj) continue;
#pragma unroll
    for (int uc = 0; uc < 4; ++uc) {
      const int cc = tx + 16 * uc;
      if (cc >= nc) continue;
      T* out = dW + (j0 + jj) * ldw + c0 + cc;
      float v = acc[uj][uc];
      if (accumulate) v += ld_elem(out);
      st_elem(out, v);
    }
  }
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
  if (launch_rows_tiled<false>(law, q, rt, row_begin, rows, X, W, Y, bi, bo, 0, s)) {
    note_launch();
    return cuda_status(cudaGetLastError());
  }
  // a few rows (decode) or a grid too large for the tiles: one thread per output
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
  if (launch_rows_tiled<true>(law, q, rt, 0, rows, dY, W, dX, bo, bi, accumulate, s)) {
    note_launch();
    return cuda_status(cudaGetLastError());
  }
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
  const long long gx = (long long)q * ((bi + kDwTile - 1) / kDwTile);
  const long long gy = (long long)q * ((bo + kDwTile - 1) / kDwTile);
  if (gx <= 0x7fffffffLL && gy <= 65535) {
    const dim3 grd((unsigned)gx, (unsigned)gy);
    if (X.dtype == AAL_F32)
      k_bwd_dw_tiled<float><<<grd, 256, 0, s>>>(law, q, rt, rows, (const float*)X.ptr, X.ld,
                                                (const float*)dY.ptr, dY.ld, (float*)dW.ptr, dW.ld, bi,
                                                bo, accumulate);
    else
      k_bwd_dw_tiled<__nv_bfloat16><<<grd, 256, 0, s>>>(
          law, q, rt, rows, (const __nv_bfloat16*)X.ptr, X.ld, (const __nv_bfloat16*)dY.ptr, dY.ld,
          (__nv_bfloat16*)dW.ptr, dW.ld, bi, bo, accumulate);
    note_launch();
    return cuda_status(cudaGetLastError());
  }
  // more tile columns than a grid's y extent holds: one thread per output
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
