// The C-ABI entry points of libaal: argument checks, path choice, launches.
#include <string.h>

#include "aal_internal.h"

namespace aal {

static thread_local int t_policy = AAL_PATH_AUTO;
static thread_local void* t_ws = nullptr;        // aal_set_workspace
static thread_local uint64_t t_ws_bytes = 0;
static thread_local int t_last_path = 0;
static thread_local long long t_launches = 0;

void note_launch(int n) { t_launches += n; }
void note_path(int path) { t_last_path = path; }

static thread_local cudaEvent_t t_ev_before[16] = {};
static thread_local cudaEvent_t t_ev_after[16] = {};

// Records an event on ``s``; while ``s`` is being captured into a CUDA graph
// the record becomes an event-record node, so the event still timestamps the
// launch each time the graph runs.
static cudaError_t record_event(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return cudaErrorUnknown;
  if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  return cudaEventRecord(e, s);
}

// Records the one-shot timing events of ``kind`` around ``launch``.
template <typename F>
static aal_status timed(int kind, cudaStream_t s, F launch) {
  cudaEvent_t b = t_ev_before[kind], a = t_ev_after[kind];
  if (b && record_event(b, s) != cudaSuccess) return AAL_ERR_CUDA;
  aal_status st = launch();
  if (a && st == AAL_OK && record_event(a, s) != cudaSuccess) return AAL_ERR_CUDA;
  if (st == AAL_OK) { t_ev_before[kind] = nullptr; t_ev_after[kind] = nullptr; }
  return st;
}

static bool valid_law(int law, int q) {
  if (q < 1 || q > (1 << 16)) return false;
  if (law == AAL_LAW_Q) return true;
  if (law == AAL_LAW_Q2XQ2) return q == 4;
  return false;
}

static bool valid_mat(const aal_mat& m) {
  if (m.dtype != AAL_BF16 && m.dtype != AAL_F32) return false;
  if (m.rows < 0 || m.cols < 0 || m.ld < m.cols || m.ld < 0) return false;
  if (m.rows > 0 && m.cols > 0 && m.ptr == nullptr) return false;
  const size_t es = m.dtype == AAL_F32 ? 4 : 2;
  if (m.ptr && ((uintptr_t)m.ptr % es) != 0) return false;
  return true;
}

static bool valid_rule(const aal_row_type_rule& r, long long rows) {
  if (r.kind == AAL_TYPES_POSITION) return r.seq_len > 0 && r.pos_offset >= 0;
  if (r.kind == AAL_TYPES_EXPLICIT) return rows == 0 || r.types != nullptr;
  return false;
}

static RowTypes make_types(const aal_row_type_rule& r, int q) {
  RowTypes rt;
  rt.kind = r.kind == AAL_TYPES_POSITION ? kTypesPosition : kTypesExplicit;
  rt.q = q;
  rt.seq_len = r.seq_len > 0 ? r.seq_len : 1;
  rt.pos_offset = r.pos_offset;
  rt.types = r.types;
  rt.positions = nullptr;
  return rt;
}

// Runs the tensor-core launcher when the policy allows it, else the general
// one.  ``tc`` returns AAL_ERR_UNSUPPORTED without launching anything when it
// cannot serve the shape.
template <typename TC, typename GEN>
static aal_status dispatch(int kind, cudaStream_t s, TC tc_launch, GEN gen_launch) {
  auto tc = [&] { return timed(kind, s, tc_launch); };
  auto gen = [&] { return timed(kind, s, gen_launch); };
  if (t_policy != AAL_PATH_GENERAL) {
    aal_status st = tc();
    if (st == AAL_OK) { note_path(AAL_PATH_TENSOR); return AAL_OK; }
    if (st != AAL_ERR_UNSUPPORTED || t_policy == AAL_PATH_TENSOR) return st;
  }
  aal_status st = gen();
  if (st == AAL_OK) note_path(AAL_PATH_GENERAL);
  return st;
}

void* current_workspace(uint64_t* bytes) {
  *bytes = t_ws_bytes;
  return t_ws;
}

// A second stream of this host thread on each device it uses, with the events
// that fork it from the caller's stream and join it back.  The fork and join
// are an event record and a stream wait, so they work the same way while the
// caller's stream is being captured into a CUDA graph (the second stream then
// joins the capture).
struct SideStream {
  int dev = -1;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
static thread_local SideStream t_side[8];

// The side stream, ordered after everything queued on ``s`` so far; null if
// it cannot be had (the caller then stays on ``s``).
static cudaStream_t fork_side(cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  SideStream* ss = nullptr;
  for (SideStream& e : t_side)
    if (e.dev == dev) { ss = &e; break; }
  if (!ss) {
    // created outside a capture only (a failing call inside one would end it)
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return nullptr;
    for (SideStream& e : t_side)
      if (e.dev < 0) { ss = &e; break; }
    if (!ss) return nullptr;
    if (cudaStreamCreateWithFlags(&ss->s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&ss->fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss->join, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamDestroy(ss->s);
      if (ss->fork) cudaEventDestroy(ss->fork);
      *ss = SideStream();
      return nullptr;
    }
    ss->dev = dev;
  }
  if (cudaEventRecord(ss->fork, s) != cudaSuccess) return nullptr;
  if (cudaStreamWaitEvent(ss->s, ss->fork, 0) != cudaSuccess) return nullptr;
  return ss->s;
}

// Orders ``s`` after everything queued on the side stream ``side`` so far.
static aal_status join_side(cudaStream_t s, cudaStream_t side) {
  for (SideStream& e : t_side)
    if (e.s == side) {
      if (cudaEventRecord(e.join, side) != cudaSuccess || cudaStreamWaitEvent(s, e.join, 0) != cudaSuccess)
        return AAL_ERR_CUDA;
      return AAL_OK;
    }
  return AAL_ERR_CUDA;
}

}  // namespace aal

using namespace aal;

extern "C" {

aal_status aal_project_fwd(int32_t law, int32_t q, aal_row_type_rule rule, aal_mat X, aal_mat W,
                           aal_mat Y, void* stream) {
  if (!valid_law(law, q) || !valid_mat(X) || !valid_mat(W) || !valid_mat(Y))
    return AAL_ERR_INVALID_ARG;
  if (X.dtype != W.dtype || X.dtype != Y.dtype) return AAL_ERR_UNSUPPORTED;
  if (W.rows != X.cols || Y.rows != X.rows || Y.cols != W.cols) return AAL_ERR_INVALID_ARG;
  if (X.cols % q || W.cols % q) return AAL_ERR_INVALID_ARG;
  if (!valid_rule(rule, X.rows)) return AAL_ERR_INVALID_ARG;
  note_path(0);
  if (X.rows == 0 || Y.cols == 0) return AAL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  RowTypes rt = make_types(rule, q);
  if (t_policy != AAL_PATH_GENERAL && t_ws && X.dtype == AAL_BF16 && seg_needed(rt, q, X.rows)) {
    // explicit or ragged types: rows sorted by type into the workspace, then
    // the tensor-core path in segment mode
    const aal_status st = timed(AAL_KERNEL_PROJECT, s, [&] {
      return seg_project_fwd(law, q, rt, X, W, Y, t_ws, t_ws_bytes, s);
    });
    if (st == AAL_OK) { note_path(AAL_PATH_TENSOR); return AAL_OK; }
    if (st != AAL_ERR_UNSUPPORTED) return st;
  }
  return dispatch(AAL_KERNEL_PROJECT, s, [&] { return tc_project(law, q, rt, X.rows, X, W, Y, s); },
                  [&] { return simt_project(law, q, rt, X, W, Y, s); });
}

aal_status aal_swiglu_fwd(int32_t law, int32_t q, aal_row_type_rule rule, aal_mat X, aal_mat Wg,
                          aal_mat Wu, aal_mat Wd, aal_mat H, aal_mat Y, void* stream) {
  if (!valid_law(law, q) || !valid_mat(X) || !valid_mat(Wg) || !valid_mat(Wu) ||
      !valid_mat(Wd) || !valid_mat(H) || !valid_mat(Y))
    return AAL_ERR_INVALID_ARG;
  const int dt = X.dtype;
  if (Wg.dtype != dt || Wu.dtype != dt || Wd.dtype != dt || H.dtype != dt || Y.dtype != dt)
    return AAL_ERR_UNSUPPORTED;
  const long long M = X.rows, D = X.cols, F = Wg.cols;
  if (Wg.rows != D || Wu.rows != D || Wu.cols != F || Wd.rows != F || Wd.cols != D ||
      H.rows != M || H.cols != F || Y.rows != M || Y.cols != D)
    return AAL_ERR_INVALID_ARG;
  if (D % q || F % q) return AAL_ERR_INVALID_ARG;
  if (!valid_rule(rule, M)) return AAL_ERR_INVALID_ARG;
  note_path(0);
  if (M == 0 || D == 0) return AAL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  RowTypes rt = make_types(rule, q);
  if (t_policy != AAL_PATH_GENERAL && t_ws && dt == AAL_BF16 && seg_needed(rt, q, M)) {
    const aal_status st = timed(AAL_KERNEL_GATE_UP, s, [&] {
      return seg_swiglu_fwd(law, q, rt, X, Wg, Wu, Wd, H, Y, t_ws, t_ws_bytes, s);
    });
    if (st == AAL_OK) { note_path(AAL_PATH_TENSOR); return AAL_OK; }
    if (st != AAL_ERR_UNSUPPORTED) return st;
  }
  int path_gu = 0;
  aal_status st = dispatch(AAL_KERNEL_GATE_UP, s, [&] { return tc_swiglu_gate_up(law, q, rt, M, X, Wg, Wu, H, s); },
                           [&] { return simt_swiglu_gate_up(law, q, rt, X, Wg, Wu, H, s); });
  if (st != AAL_OK) return st;
  path_gu = t_last_path;
  st = dispatch(AAL_KERNEL_PROJECT, s, [&] { return tc_project(law, q, rt, M, H, Wd, Y, s); },
                [&] { return simt_project(law, q, rt, H, Wd, Y, s); });
  if (st == AAL_OK && path_gu != t_last_path) note_path(AAL_PATH_GENERAL);
  return st;
}

aal_status aal_project_bwd(int32_t law, int32_t q, aal_row_type_rule rule, aal_mat X, aal_mat W,
                           aal_mat dY, aal_mat dX, aal_mat dW, int32_t accumulate_dW,
                           void* stream) {
  if (!valid_law(law, q) || !valid_mat(X) || !valid_mat(W) || !valid_mat(dY))
    return AAL_ERR_INVALID_ARG;
  const bool want_dx = dX.ptr != nullptr, want_dw = dW.ptr != nullptr;
  if ((want_dx && !valid_mat(dX)) || (want_dw && !valid_mat(dW))) return AAL_ERR_INVALID_ARG;
  const int dt = X.dtype;
  if (W.dtype != dt || dY.dtype != dt || (want_dx && dX.dtype != dt) ||
      (want_dw && dW.dtype != dt))
    return AAL_ERR_UNSUPPORTED;
  const long long M = X.rows, din = X.cols, dout = W.cols;
  if (W.rows != din || dY.rows != M || dY.cols != dout) return AAL_ERR_INVALID_ARG;
  if (want_dx && (dX.rows != M || dX.cols != din)) return AAL_ERR_INVALID_ARG;
  if (want_dw && (dW.rows != din || dW.cols != dout)) return AAL_ERR_INVALID_ARG;
  if (din % q || dout % q) return AAL_ERR_INVALID_ARG;
  if (!valid_rule(rule, M)) return AAL_ERR_INVALID_ARG;
  note_path(0);
  cudaStream_t s = (cudaStream_t)stream;
  RowTypes rt = make_types(rule, q);
  int paths = 0;
  // Small problems run dX (on s) and dW (on a side stream) side by side, each
  // on half of the SMs, with the split-K partials of dW placed after dX's in
  // the workspace.
  cudaStream_t sw = s;
  void* const ws0 = t_ws;
  const uint64_t ws0_bytes = t_ws_bytes;
  int64_t dw_off = 0;
  if (want_dx && want_dw && M > 0 && t_policy != AAL_PATH_GENERAL && X.dtype == AAL_BF16 &&
      tc_bwd_side_by_side(M, din, dout)) {
    cudaStream_t side = fork_side(s);
    if (side) {
      sw = side;
      set_sm_share(device_sms() / 2);
      int64_t a = 0, b = 0;
      tc_bwd_split_parts(law, q, M, din, dout, &a, &b);
      dw_off = (a + 255) & ~(int64_t)255;
    }
  }
  aal_status st = AAL_OK;
  if (want_dx && M > 0 && din > 0) {
    st = dispatch(AAL_KERNEL_BWD_DX, s, [&] { return tc_project_bwd_dx(law, q, rt, M, dY, W, dX, 0, s); },
                  [&] { return simt_project_bwd_dx(law, q, rt, dY, W, dX, s); });
    if (st == AAL_OK) paths |= 1 << t_last_path;
  }
  if (st == AAL_OK && want_dw && din > 0 && dout > 0) {
    if (sw != s) {
      const bool fits = ws0 && (uint64_t)dw_off < ws0_bytes;
      t_ws = fits ? (char*)ws0 + dw_off : nullptr;
      t_ws_bytes = fits ? ws0_bytes - (uint64_t)dw_off : 0;
    }
    st = dispatch(AAL_KERNEL_BWD_DW, sw, [&] { return tc_project_bwd_dw(law, q, rt, M, X, dY, dW, accumulate_dW, sw); },
                  [&] { return simt_project_bwd_dw(law, q, rt, X, dY, dW, accumulate_dW, sw); });
    t_ws = ws0;
    t_ws_bytes = ws0_bytes;
    if (st == AAL_OK) paths |= 1 << t_last_path;
  }
  if (sw != s) {
    set_sm_share(0);
    const aal_status sj = join_side(s, sw);  // always: a capture must end joined
    if (st == AAL_OK) st = sj;
  }
  if (st != AAL_OK) return st;
  if (paths) note_path((paths & (1 << AAL_PATH_GENERAL)) ? AAL_PATH_GENERAL : AAL_PATH_TENSOR);
  return AAL_OK;
}

aal_status aal_swiglu_bwd(int32_t law, int32_t q, aal_row_type_rule rule, aal_mat X, aal_mat Wg,
                          aal_mat Wu, aal_mat Wd, aal_mat H, aal_mat dY, aal_mat G, aal_mat U,
                          aal_mat dG, aal_mat dU, aal_mat dX, aal_mat dWg, aal_mat dWu,
                          aal_mat dWd, void* stream) {
  const aal_mat* all[] = {&X, &Wg, &Wu, &Wd, &H, &dY, &G, &U, &dG, &dU, &dX, &dWg, &dWu, &dWd};
  if (!valid_law(law, q)) return AAL_ERR_INVALID_ARG;
  for (const aal_mat* m : all)
    if (!valid_mat(*m)) return AAL_ERR_INVALID_ARG;
  for (const aal_mat* m : all)
    if (m->dtype != X.dtype) return AAL_ERR_UNSUPPORTED;
  const long long M = X.rows, D = X.cols, F = Wg.cols;
  auto is = [](const aal_mat& m, long long r, long long c) { return m.rows == r && m.cols == c; };
  if (!is(Wg, D, F) || !is(Wu, D, F) || !is(Wd, F, D) || !is(H, M, F) || !is(dY, M, D) ||
      !is(G, M, F) || !is(U, M, F) || !is(dG, M, F) || !is(dU, M, F) || !is(dX, M, D) ||
      !is(dWg, D, F) || !is(dWu, D, F) || !is(dWd, F, D))
    return AAL_ERR_INVALID_ARG;
  if (D % q || F % q) return AAL_ERR_INVALID_ARG;
  if (!valid_rule(rule, M)) return AAL_ERR_INVALID_ARG;
  note_path(0);
  if (D == 0 || F == 0) return AAL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  RowTypes rt = make_types(rule, q);
  int paths = 0;
  aal_status st = AAL_OK;
  auto note = [&] { paths |= 1 << t_last_path; };
  // weight gradient i: dWd (needs only H and dY), dWg, dWu
  const aal_mat* dw_in[3][3] = {{&H, &dY, &dWd}, {&X, &dG, &dWg}, {&X, &dU, &dWu}};
  auto weight_grad = [&](int i, cudaStream_t on) {
    const aal_mat &A = *dw_in[i][0], &B = *dw_in[i][1], &O = *dw_in[i][2];
    aal_status e = dispatch(AAL_KERNEL_BWD_DW, on, [&] { return tc_project_bwd_dw(law, q, rt, M, A, B, O, 0, on); },
                            [&] { return simt_project_bwd_dw(law, q, rt, A, B, O, 0, on); });
    if (e == AAL_OK) note();
    return e;
  };
  if (M > 0) {
    // 1. the gate and up pre-activations, recomputed
    st = dispatch(AAL_KERNEL_PROJECT, s, [&] { return tc_project(law, q, rt, M, X, Wg, G, s); },
                  [&] { return simt_project(law, q, rt, X, Wg, G, s); });
    if (st == AAL_OK) {
      note();
      st = dispatch(AAL_KERNEL_PROJECT, s, [&] { return tc_project(law, q, rt, M, X, Wu, U, s); },
                    [&] { return simt_project(law, q, rt, X, Wu, U, s); });
    }
    if (st == AAL_OK) note();
    // 2. dH = dY through the down projection's transposed table, and the
    //    SiLU' chain: dG = dH u silu'(g), dU = dH silu(g)
    if (st == AAL_OK)
      st = dispatch(AAL_KERNEL_SWIGLU_BWD, s,
                    [&] { return tc_swiglu_bwd_dh(law, q, rt, M, dY, Wd, G, U, dG, dU, s); },
                    [&] {
                      aal_status e = simt_project_bwd_dx(law, q, rt, dY, Wd, dG, s);
                      return e != AAL_OK ? e : simt_swiglu_bwd_act(q, rt, G, U, dG, dU, s);
                    });
    if (st == AAL_OK) note();
  }
  if (st != AAL_OK) return st;
  // Small problems run the four launches after dH side by side, every launch
  // on half of the SMs: dX then dWu on the caller's stream, dWd then dWg on a
  // side stream, whose split-K partials follow the caller stream's in the
  // workspace.
  cudaStream_t sw = s;
  if (M > 0 && t_policy != AAL_PATH_GENERAL && X.dtype == AAL_BF16 && tc_bwd_side_by_side(M, D, F)) {
    cudaStream_t side = fork_side(s);
    if (side) {
      sw = side;
      set_sm_share(device_sms() / 2);
      int64_t dx = 0, dw = 0;
      tc_bwd_split_parts(law, q, M, D, F, &dx, &dw);
      const int64_t off = ((dx > dw ? dx : dw) + 255) & ~(int64_t)255;
      void* const ws0 = t_ws;
      const uint64_t ws0_bytes = t_ws_bytes;
      const bool fits = ws0 && (uint64_t)off < ws0_bytes;
      t_ws = fits ? (char*)ws0 + off : nullptr;
      t_ws_bytes = fits ? ws0_bytes - (uint64_t)off : 0;
      st = weight_grad(0, sw);
      if (st == AAL_OK) st = weight_grad(1, sw);
      t_ws = ws0;
      t_ws_bytes = ws0_bytes;
    }
  }
  if (st == AAL_OK && M > 0) {
    // 3. dX = dG Wg^T + dU Wu^T over the table: one tensor-core launch with
    //    both products in the same accumulator, else two general passes
    st = dispatch(AAL_KERNEL_BWD_DX, s, [&] { return tc_swiglu_bwd_dx(law, q, rt, M, dG, Wg, dU, Wu, dX, s); },
                  [&] {
                    aal_status e = simt_project_bwd_dx(law, q, rt, dG, Wg, dX, s);
                    return e != AAL_OK ? e : simt_project_bwd_dx(law, q, rt, dU, Wu, dX, s, 1);
                  });
    if (st == AAL_OK) note();
  }
  // 4. weight gradients (zero when there are no rows)
  if (sw != s) {
    if (st == AAL_OK) st = weight_grad(2, s);
    set_sm_share(0);
    const aal_status sj = join_side(s, sw);  // always: a capture must end joined
    if (st == AAL_OK) st = sj;
  } else {
    for (int i = 0; i < 3 && st == AAL_OK; ++i) st = weight_grad(i, s);
  }
  if (st != AAL_OK) return st;
  note_path((paths & (1 << AAL_PATH_GENERAL)) ? AAL_PATH_GENERAL : AAL_PATH_TENSOR);
  return AAL_OK;
}

aal_status aal_decode_matvec(int32_t law, int32_t q, const int64_t* positions, aal_mat x,
                             aal_mat W, aal_mat y, void* stream) {
  if (!valid_law(law, q) || !valid_mat(x) || !valid_mat(W) || !valid_mat(y))
    return AAL_ERR_INVALID_ARG;
  if (x.dtype != W.dtype || x.dtype != y.dtype) return AAL_ERR_UNSUPPORTED;
  if (W.rows != x.cols || y.rows != x.rows || y.cols != W.cols) return AAL_ERR_INVALID_ARG;
  if (x.cols % q || W.cols % q) return AAL_ERR_INVALID_ARG;
  if (x.rows > 0 && positions == nullptr) return AAL_ERR_INVALID_ARG;
  note_path(0);
  if (x.rows == 0 || y.cols == 0) return AAL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (t_policy != AAL_PATH_GENERAL) {
    bool handled = false;
    aal_status st = timed(AAL_KERNEL_DECODE, s, [&] {
      return decode_matvec(law, q, positions, x, W, y, s, &handled);
    });
    if (handled) {
      if (st == AAL_OK) note_path(AAL_PATH_DECODE);
      return st;
    }
    if (t_policy == AAL_PATH_TENSOR) return AAL_ERR_UNSUPPORTED;
  }
  RowTypes rt;
  rt.kind = kTypesPositions64;
  rt.q = q;
  rt.seq_len = 1;
  rt.pos_offset = 0;
  rt.types = nullptr;
  rt.positions = positions;
  aal_status st = simt_project(law, q, rt, x, W, y, s);
  if (st == AAL_OK) note_path(AAL_PATH_GENERAL);
  return st;
}

aal_status aal_swiglu_decode(int32_t law, int32_t q, const int64_t* positions, aal_mat x,
                             aal_mat Wg, aal_mat Wu, aal_mat Wd, aal_mat h, aal_mat y, void* stream) {
  if (!valid_law(law, q) || !valid_mat(x) || !valid_mat(Wg) || !valid_mat(Wu) || !valid_mat(Wd) ||
      !valid_mat(h) || !valid_mat(y))
    return AAL_ERR_INVALID_ARG;
  if (x.dtype != Wg.dtype || x.dtype != Wu.dtype || x.dtype != Wd.dtype || x.dtype != h.dtype ||
      x.dtype != y.dtype)
    return AAL_ERR_UNSUPPORTED;
  const long long B = x.rows, D = x.cols, F = Wg.cols;
  if (Wg.rows != D || Wu.rows != D || Wu.cols != F || Wd.rows != F || Wd.cols != D ||
      h.rows != B || h.cols != F || y.rows != B || y.cols != D)
    return AAL_ERR_INVALID_ARG;
  if (D % q || F % q) return AAL_ERR_INVALID_ARG;
  if (B > 0 && positions == nullptr) return AAL_ERR_INVALID_ARG;
  note_path(0);
  if (B == 0 || D == 0 || F == 0) return AAL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (t_policy != AAL_PATH_GENERAL && ffn_decode_fused_ok(law, q, x, Wg, Wu, Wd, h, y)) {
    const aal_status fs = timed(AAL_KERNEL_FFN_DECODE, s, [&] {
      return ffn_decode_fused(law, q, positions, x, Wg, Wu, Wd, h, y, s);
    });
    if (fs == AAL_OK) note_path(AAL_PATH_DECODE);
    return fs;
  }
  int path = AAL_PATH_DECODE;
  aal_status st = AAL_OK;
  bool handled = false;
  if (t_policy != AAL_PATH_GENERAL) {
    st = timed(AAL_KERNEL_DECODE_GATE_UP, s, [&] {
      return decode_gate_up(law, q, positions, x, Wg, Wu, h, s, &handled);
    });
    if (st != AAL_OK) return st;
    if (!handled && t_policy == AAL_PATH_TENSOR) return AAL_ERR_UNSUPPORTED;
  }
  RowTypes rt;
  rt.kind = kTypesPositions64;
  rt.q = q;
  rt.seq_len = 1;
  rt.pos_offset = 0;
  rt.types = nullptr;
  rt.positions = positions;
  if (!handled) {
    st = timed(AAL_KERNEL_DECODE_GATE_UP, s, [&] { return simt_swiglu_gate_up(law, q, rt, x, Wg, Wu, h, s); });
    if (st != AAL_OK) return st;
    path = AAL_PATH_GENERAL;
  }
  handled = false;
  if (t_policy != AAL_PATH_GENERAL) {
    // up to 16 entries the down decode starts while the gate/up kernel runs
    // and waits for h on the device (programmatic dependent launch; measured
    // on B200: 9.2 -> 8.4 us per FFN step at one entry, slower at 64)
    st = timed(AAL_KERNEL_DECODE, s, [&] {
      return decode_matvec(law, q, positions, h, Wd, y, s, &handled, path == AAL_PATH_DECODE && B <= 16);
    });
    if (st != AAL_OK) return st;
  }
  if (!handled) {
    if (t_policy == AAL_PATH_TENSOR) return AAL_ERR_UNSUPPORTED;
    st = simt_project(law, q, rt, h, Wd, y, s);
    if (st != AAL_OK) return st;
    path = AAL_PATH_GENERAL;
  }
  note_path(path);
  return AAL_OK;
}

aal_status aal_square_product(int32_t law, int32_t q, aal_mat X, aal_mat W, aal_mat Z,
                              void* stream) {
  if (!valid_law(law, q) || !valid_mat(X) || !valid_mat(W) || !valid_mat(Z))
    return AAL_ERR_INVALID_ARG;
  if (X.dtype != W.dtype || X.dtype != Z.dtype) return AAL_ERR_UNSUPPORTED;
  const long long n = X.rows;
  if (X.cols != n || W.rows != n || W.cols != n || Z.rows != n || Z.cols != n)
    return AAL_ERR_INVALID_ARG;
  if (n % q) return AAL_ERR_INVALID_ARG;
  if (n > 0 && (Z.ptr == X.ptr || Z.ptr == W.ptr)) return AAL_ERR_INVALID_ARG;
  note_path(0);
  if (n == 0) return AAL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  return dispatch(AAL_KERNEL_SQUARE, s, [&] { return tc_square(law, q, X, W, Z, s); },
                  [&] { return simt_square(law, q, X, W, Z, s); });
}

aal_status aal_block_table(int32_t law, int32_t q, uint8_t* S) {
  if (!valid_law(law, q) || S == nullptr) return AAL_ERR_INVALID_ARG;
  for (int i = 0; i < q; ++i)
    for (int k = 0; k < q; ++k)
      for (int a = 0; a < q; ++a)
        S[((size_t)i * q + k) * q + a] = in_table(law, i, k, a) ? 1 : 0;
  return AAL_OK;
}

int64_t aal_block_product_count(int32_t law, int32_t q, int32_t row_typed) {
  if (!valid_law(law, q)) return -1;
  int64_t n = 0;
  const int rows = row_typed ? 1 : q;
  for (int i = 0; i < rows; ++i)
    for (int k = 0; k < q; ++k) {
      int members[4];
      n += table_members(law, q, i, k, members);
    }
  return n;
}

aal_status aal_get_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return AAL_ERR_CUDA;
  int code = 0;
  if (cudaMemcpyFromSymbol(&code, g_device_status, sizeof(int)) != cudaSuccess)
    return AAL_ERR_CUDA;
  if (code != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
      return AAL_ERR_CUDA;
  }
  if (code == kDevTimeout) return AAL_ERR_DEVICE_TIMEOUT;
  if (code == kDevBounds) return AAL_ERR_DEVICE_BOUNDS;
  return AAL_OK;
}

const char* aal_status_string(int32_t status) {
  switch (status) {
    case AAL_OK: return "ok";
    case AAL_ERR_INVALID_ARG: return "invalid argument";
    case AAL_ERR_UNSUPPORTED: return "not supported by the library";
    case AAL_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case AAL_ERR_CUDA: return "CUDA runtime error";
    case AAL_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
    case AAL_ERR_DEVICE_BOUNDS: return "a kernel met an out-of-range row type or position";
    case AAL_ERR_SCRATCH_LIMIT: return "request larger than the library's fixed device scratch";
    default: return "unknown status";
  }
}

aal_status aal_set_timing_events(int32_t kernel, void* before, void* after) {
  if (kernel < AAL_KERNEL_PROJECT || kernel > AAL_KERNEL_FFN_DECODE) return AAL_ERR_INVALID_ARG;
  t_ev_before[kernel] = (cudaEvent_t)before;
  t_ev_after[kernel] = (cudaEvent_t)after;
  return AAL_OK;
}

int64_t aal_workspace_size(int32_t call, int32_t law, int32_t q, aal_row_type_rule rule, int64_t rows,
                           int64_t d_in, int64_t d_hidden) {
  if (!valid_law(law, q) || rows < 0 || d_in < 0 || d_hidden < 0 || !valid_rule(rule, rows)) return -1;
  if (call < AAL_CALL_PROJECT_FWD || call > AAL_CALL_SWIGLU_BWD) return -1;
  const RowTypes rt = make_types(rule, q);
  if (rows == 0) return 0;
  if (call == AAL_CALL_PROJECT_BWD || call == AAL_CALL_SWIGLU_BWD) {
    // split K of the heavy tiles (position rules on the tensor-core path only)
    if (seg_needed(rt, q, rows)) return 0;
    return call == AAL_CALL_SWIGLU_BWD ? tc_swiglu_bwd_split_bytes(law, q, rows, d_in, d_hidden)
                                       : tc_bwd_split_bytes(law, q, rows, d_in, d_hidden);
  }
  if (!seg_needed(rt, q, rows)) return 0;
  return seg_workspace_bytes(q, rows, d_in, call == AAL_CALL_SWIGLU_FWD ? d_hidden : 0);
}


aal_status aal_set_workspace(void* device_ptr, uint64_t bytes) {
  if (device_ptr && ((uintptr_t)device_ptr % 256) != 0) return AAL_ERR_ALIGNMENT;
  t_ws = bytes ? device_ptr : nullptr;
  t_ws_bytes = device_ptr ? bytes : 0;
  return AAL_OK;
}

aal_status aal_set_path_policy(int32_t policy) {
  if (policy < AAL_PATH_AUTO || policy > AAL_PATH_GENERAL) return AAL_ERR_INVALID_ARG;
  t_policy = policy;
  return AAL_OK;
}

int32_t aal_last_path(void) { return t_last_path; }

int64_t aal_launch_count(int32_t reset) {
  const long long n = t_launches;
  if (reset) t_launches = 0;
  return n;
}

int32_t aal_version(void) { return 100; }

}  // extern "C"
