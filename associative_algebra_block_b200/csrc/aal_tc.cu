// Tensor-core path (tcgen05 / TMEM / TMA) — filled in below.
#include "aal_internal.h"

namespace aal {

aal_status tc_project(int, int, const RowTypes&, long long, const aal_mat&, const aal_mat&,
                      const aal_mat&, cudaStream_t) { return AAL_ERR_UNSUPPORTED; }
aal_status tc_swiglu_gate_up(int, int, const RowTypes&, long long, const aal_mat&, const aal_mat&,
                             const aal_mat&, const aal_mat&, cudaStream_t) {
  return AAL_ERR_UNSUPPORTED;
}
aal_status tc_project_bwd_dx(int, int, const RowTypes&, long long, const aal_mat&, const aal_mat&,
                             const aal_mat&, cudaStream_t) { return AAL_ERR_UNSUPPORTED; }
aal_status tc_project_bwd_dw(int, int, const RowTypes&, long long, const aal_mat&, const aal_mat&,
                             const aal_mat&, int, cudaStream_t) { return AAL_ERR_UNSUPPORTED; }
aal_status tc_square(int, int, const aal_mat&, const aal_mat&, const aal_mat&, cudaStream_t) {
  return AAL_ERR_UNSUPPORTED;
}

}  // namespace aal
