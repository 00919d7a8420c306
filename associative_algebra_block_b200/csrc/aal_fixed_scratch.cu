// FFN decode step for callers that cannot allocate device memory.
//
// aal_swiglu_decode needs a caller buffer for the activation h [B, F] between
// the gate/up and the down projections.  Some callers have no way to provide
// one: a plug-in running inside a host application that owns every device
// allocation through its own pool and forbids direct cudaMalloc, or a
// real-time decode loop in which cudaMalloc's implicit device-wide
// synchronisation is not allowed.  aal_swiglu_decode_noalloc keeps h in the
// fixed array below instead and otherwise runs exactly the kernels of
// aal_swiglu_decode.
#include <mutex>

#include "aal_internal.h"

namespace aal {

// Largest activation the entry point holds: B * F elements of the call's
// dtype in at most 4 MiB.  Every device that loads the library keeps this
// array until the process exits.
constexpr size_t kFixedScratchBytes = (size_t)4 << 20;
static __device__ __align__(256) unsigned char g_ffn_decode_h[kFixedScratchBytes];

// Device address of g_ffn_decode_h, looked up once per device ordinal (with
// that device current).  In host code the symbol itself is only a host-side
// stand-in; kernels must be given this address.
constexpr int kFixedScratchDevices = 64;
static std::mutex g_fixed_scratch_mu;
static void* g_fixed_scratch_ptr[kFixedScratchDevices] = {};

static aal_status fixed_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AAL_ERR_CUDA;
  if (dev >= 0 && dev < kFixedScratchDevices) {
    std::lock_guard<std::mutex> lock(g_fixed_scratch_mu);
    if (g_fixed_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_ffn_decode_h) != cudaSuccess || p == nullptr)
        return AAL_ERR_CUDA;
      g_fixed_scratch_ptr[dev] = p;
    }
    *out = g_fixed_scratch_ptr[dev];
    return AAL_OK;
  }
  // more devices than the cache holds: look the address up on every call
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_ffn_decode_h) != cudaSuccess || p == nullptr) return AAL_ERR_CUDA;
  *out = p;
  return AAL_OK;
}

}  // namespace aal

extern "C" aal_status aal_swiglu_decode_noalloc(int32_t law, int32_t q, const int64_t* positions,
                                                aal_mat x, aal_mat Wg, aal_mat Wu, aal_mat Wd,
                                                aal_mat y, void* stream) {
  using namespace aal;
  if (x.dtype != AAL_BF16 && x.dtype != AAL_F32) return AAL_ERR_INVALID_ARG;
  if (x.rows < 0 || Wg.cols < 0) return AAL_ERR_INVALID_ARG;
  const long long B = x.rows, F = Wg.cols;
  const size_t es = x.dtype == AAL_F32 ? 4 : 2;
  // the size limit is checked before anything touches the device
  if (B > 0 && F > 0 && (unsigned long long)B > kFixedScratchBytes / es / (unsigned long long)F)
    return AAL_ERR_SCRATCH_LIMIT;
  aal_mat h;
  h.ptr = nullptr;
  h.dtype = x.dtype;
  h.rows = B;
  h.cols = F;
  h.ld = F;
  if (B > 0 && F > 0) {
    const aal_status st = fixed_scratch_address(&h.ptr);
    if (st != AAL_OK) return st;
  }
  return aal_swiglu_decode(law, q, positions, x, Wg, Wu, Wd, h, y, stream);
}
