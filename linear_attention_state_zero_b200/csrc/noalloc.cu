// noalloc.cu -- tr_state_error_noalloc: the state-error reduction with its scratch
// space in a fixed array inside the library instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point of the
// call -- a serving engine whose allocator owns every byte of the device and hands
// out no scratch to a library, or code running where cudaMalloc/cudaFree are not
// allowed because they synchronize the device.  They pass only inputs and outputs.
//
// The scratch array lives in device memory for as long as the library is loaded,
// on every GPU that loads it (kStaticMats * 2 doubles = 1 MiB).  All calls share it:
// two calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on it.  Every entry a call reads was written earlier by the
// same call, so nothing needs clearing between calls.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/tr.h"
#include "tr_internal.h"

namespace {

constexpr int64_t kStaticMats = 65536;  // largest n_mats one call accepts

// (sum (S - S_hat)^2, sum S^2) of each matrix piece of the last call (at most
// kStaticMats pieces: a matrix is cut into fewer pieces when n_mats is large).
static __device__ __align__(256) double g_noalloc_scratch[2 * kStaticMats];

constexpr int kMaxDevices = 64;
double *g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array for the current device, looked up once per
// device (with that device current).  Host code must not use the array's name as a
// device address: in host code it names a host-side stand-in.
cudaError_t scratch_for_current_device(double **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<double *>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" tr_status tr_state_error_noalloc(const float *S, const float *S_hat, int64_t n_mats,
                                            int32_t d_k, int32_t d_v, double *err_per_mat,
                                            double *err_total, void *stream) {
  if (n_mats < 0 || d_k <= 0 || d_v <= 0)
    return tr::record_error(TR_ERR_INVALID_ARG, "bad sizes");
  if (n_mats > kStaticMats)
    return tr::record_error(TR_ERR_UNSUPPORTED,
                            "n_mats = %lld exceeds the fixed scratch of %lld matrices; use "
                            "tr_state_error with a workspace",
                            (long long)n_mats, (long long)kStaticMats);
  if (n_mats > 0 && (!S || !S_hat)) return tr::record_error(TR_ERR_INVALID_ARG, "S or S_hat is NULL");
  if (!aligned16(S) || !aligned16(S_hat)) return tr::record_error(TR_ERR_ALIGNMENT, "S/S_hat alignment");
  if (!err_per_mat && !err_total) return tr::record_error(TR_OK, "");
  double *scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess)
    return tr::record_error(TR_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
  const int64_t elems = (int64_t)d_k * d_v;
  e = tr::launch_state_error(S, S_hat, n_mats, elems, tr::state_error_splits(n_mats, elems, kStaticMats),
                             scratch, err_per_mat, err_total, static_cast<cudaStream_t>(stream),
                             true);
  if (e != cudaSuccess)
    return tr::record_error(TR_ERR_CUDA, "state error: %s", cudaGetErrorString(e));
  return tr::record_error(TR_OK, "");
}
