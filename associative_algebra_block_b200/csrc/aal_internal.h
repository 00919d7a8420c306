// Internal declarations shared by the libaal translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "aal.h"

namespace aal {

// Device status word (one per device that loaded the library).  Kernels set it
// with atomicCAS from 0 so the first error wins; aal_get_device_status reads
// and clears it.  Defined here: the library is a single translation unit.
enum DeviceCode : int { kDevOk = 0, kDevTimeout = 1, kDevBounds = 2 };
__device__ int g_device_status = 0;

__device__ __forceinline__ void flag_device_error(int code) {
  atomicCAS(&g_device_status, 0, code);
}

// Where a row's type comes from.
enum RowTypeKind : int { kTypesPosition = 0, kTypesExplicit = 1, kTypesPositions64 = 2 };

struct RowTypes {
  int kind;
  int q;
  long long seq_len;
  long long pos_offset;
  const int32_t* types;      // kind 1
  const int64_t* positions;  // kind 2 (decode)
};

// Row type of row r; -1 (and the bounds flag) for an explicit type outside
// [0, q) or a negative position.
// It is split into the load of the stored value (explicit type or position;
// nothing for position types) and its decoding, so that a thread can issue
// the loads of several rows before any check: a check may set the device
// status, and a load after that store cannot be moved ahead of it.
__device__ __forceinline__ long long row_type_raw(const RowTypes& rt, long long r) {
  if (rt.kind == kTypesExplicit) return rt.types[r];
  if (rt.kind == kTypesPositions64) return rt.positions[r];
  return 0;
}

__device__ __forceinline__ int row_type_decode(const RowTypes& rt, long long r, long long raw) {
  if (rt.kind == kTypesPosition) {
    return (int)(((r % rt.seq_len) + rt.pos_offset) % rt.q);
  }
  if (rt.kind == kTypesExplicit) {
    if (raw < 0 || raw >= rt.q) { flag_device_error(kDevBounds); return -1; }
    return (int)raw;
  }
  if (raw < 0) { flag_device_error(kDevBounds); return -1; }
  return (int)(raw % rt.q);
}

__device__ __forceinline__ int row_type(const RowTypes& rt, long long r) {
  return row_type_decode(rt, r, row_type_raw(rt, r));
}

// Membership a in S(t, k) of the multiplication table.
//  Q_q:      S(t, t) = {t}, S(t, k) = {t, k}
//  Q2 x Q2:  groups are pairs g = 2*g1 + g2 and membership factorises.
__host__ __device__ __forceinline__ bool in_table(int law, int t, int k, int a) {
  if (law == AAL_LAW_Q) return a == t || a == k;
  const int t1 = t >> 1, t2 = t & 1, k1 = k >> 1, k2 = k & 1, a1 = a >> 1, a2 = a & 1;
  return (a1 == t1 || a1 == k1) && (a2 == t2 || a2 == k2);
}

// The members of S(t, k) in ascending order; returns their count (1, 2 or 4).
__host__ __device__ __forceinline__ int table_members(int law, int q, int t, int k, int* a) {
  if (law == AAL_LAW_Q) {
    if (t == k) { a[0] = t; return 1; }
    a[0] = t < k ? t : k;
    a[1] = t < k ? k : t;
    return 2;
  }
  int n = 0;
  for (int g = 0; g < q; ++g)
    if (in_table(law, t, k, g)) a[n++] = g;
  return n;
}

// Per-thread launch accounting and path bookkeeping (api.cu).
void note_launch(int n = 1);
void note_path(int path);

// ---------------------------------------------------------------- general path
aal_status simt_project(int law, int q, const RowTypes& rt, const aal_mat& X, const aal_mat& W,
                        const aal_mat& Y, cudaStream_t s);
aal_status simt_swiglu_gate_up(int law, int q, const RowTypes& rt, const aal_mat& X,
                               const aal_mat& Wg, const aal_mat& Wu, const aal_mat& H, cudaStream_t s);
aal_status simt_project_bwd_dx(int law, int q, const RowTypes& rt, const aal_mat& dY,
                               const aal_mat& W, const aal_mat& dX, cudaStream_t s, int accumulate = 0);
aal_status simt_swiglu_bwd_act(int q, const RowTypes& rt, const aal_mat& G, const aal_mat& U,
                               const aal_mat& dG, const aal_mat& dU, cudaStream_t s);
aal_status simt_project_bwd_dw(int law, int q, const RowTypes& rt, const aal_mat& X,
                               const aal_mat& dY, const aal_mat& dW, int accumulate, cudaStream_t s);
aal_status simt_square(int law, int q, const aal_mat& X, const aal_mat& W, const aal_mat& Z,
                       cudaStream_t s);

// ----------------------------------------------------------------- decode path
aal_status decode_gate_up(int law, int q, const int64_t* positions, const aal_mat& x,
                          const aal_mat& Wg, const aal_mat& Wu, const aal_mat& h, cudaStream_t s,
                          bool* handled);
// pdl: launch with programmatic stream serialization (the kernel fetches its
// weights while the previous launch on the stream finishes).
aal_status decode_matvec(int law, int q, const int64_t* positions, const aal_mat& x,
                         const aal_mat& W, const aal_mat& y, cudaStream_t s, bool* handled,
                         bool pdl = false);
// One-launch FFN decode step (gate/up/SiLU and down in one kernel).
bool ffn_decode_fused_ok(int law, int q, const aal_mat& x, const aal_mat& Wg, const aal_mat& Wu,
                         const aal_mat& Wd, const aal_mat& h, const aal_mat& y);
aal_status ffn_decode_fused(int law, int q, const int64_t* positions, const aal_mat& x,
                            const aal_mat& Wg, const aal_mat& Wu, const aal_mat& Wd, const aal_mat& h,
                            const aal_mat& y, cudaStream_t s);

// ------------------------------------------------------------ tensor-core path
// Each returns AAL_ERR_UNSUPPORTED (launching nothing) when the shape is not
// one the tensor-core kernels serve.
aal_status tc_project(int law, int q, const RowTypes& rt, long long rows, const aal_mat& X,
                      const aal_mat& W, const aal_mat& Y, cudaStream_t s);
aal_status tc_swiglu_gate_up(int law, int q, const RowTypes& rt, long long rows, const aal_mat& X,
                             const aal_mat& Wg, const aal_mat& Wu, const aal_mat& H, cudaStream_t s);
aal_status tc_project_bwd_dx(int law, int q, const RowTypes& rt, long long rows, const aal_mat& dY,
                             const aal_mat& W, const aal_mat& dX, int accumulate, cudaStream_t s);
aal_status tc_swiglu_bwd_dx(int law, int q, const RowTypes& rt, long long rows, const aal_mat& dG,
                            const aal_mat& Wg, const aal_mat& dU, const aal_mat& Wu, const aal_mat& dX,
                            cudaStream_t s);
aal_status tc_swiglu_bwd_dh(int law, int q, const RowTypes& rt, long long rows, const aal_mat& dY,
                            const aal_mat& Wd, const aal_mat& G, const aal_mat& U,
                            const aal_mat& dG, const aal_mat& dU, cudaStream_t s);
aal_status tc_project_bwd_dw(int law, int q, const RowTypes& rt, long long rows, const aal_mat& X,
                             const aal_mat& dY, const aal_mat& dW, int accumulate, cudaStream_t s);
aal_status tc_square(int law, int q, const aal_mat& X, const aal_mat& W, const aal_mat& Z,
                     cudaStream_t s);
aal_status tc_project_seg(int law, int q, long long rows, const aal_mat& Xg, const aal_mat& Wg,
                          const aal_mat* Wu, const aal_mat& Y, const int4* tiles, const int* count,
                          const int* perm, int tmax, const aal_mat* copy, cudaStream_t s);

// ------------------------------------------- explicit / ragged row types
bool seg_needed(const RowTypes& rt, int q, long long rows);
// The caller's workspace of this host thread (aal_set_workspace), or null.
void* current_workspace(uint64_t* bytes);
// Workspace bytes the tensor-core backward of a projection W [din, dout]
// uses to split its heavy Q_q tiles (0: no split for these sizes).
int64_t tc_bwd_split_bytes(int law, int q, long long rows, long long din, long long dout);
// Split-K workspace bytes of a projection backward's dX and dW launches at the
// SM share in force.
void tc_bwd_split_parts(int law, int q, long long rows, long long din, long long dout, int64_t* dx,
                        int64_t* dw);
// The same for a SwiGLU backward of X [rows, D] through a hidden width F.
int64_t tc_swiglu_bwd_split_bytes(int law, int q, long long rows, long long D, long long F);
// Whether a projection backward runs dX and dW side by side on two streams.
bool tc_bwd_side_by_side(long long rows, long long din, long long dout);
// SMs of the current device, and the share of them that the tensor-core
// launches of this thread may use (0: all).
int device_sms();
void set_sm_share(int n);
int64_t seg_workspace_bytes(int q, long long rows, long long w1, long long w2);
aal_status seg_project_fwd(int law, int q, const RowTypes& rt, const aal_mat& X, const aal_mat& W,
                           const aal_mat& Y, void* ws, uint64_t ws_bytes, cudaStream_t s);
aal_status seg_swiglu_fwd(int law, int q, const RowTypes& rt, const aal_mat& X, const aal_mat& Wg,
                          const aal_mat& Wu, const aal_mat& Wd, const aal_mat& H, const aal_mat& Y, void* ws,
                          uint64_t ws_bytes, cudaStream_t s);

inline aal_status cuda_status(cudaError_t e) { return e == cudaSuccess ? AAL_OK : AAL_ERR_CUDA; }

}  // namespace aal
