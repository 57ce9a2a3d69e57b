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

// Device address of the scratch array in the current device's context.  Host code must
// not use the array's name as a device address: in host code it names a host-side
// stand-in.  The address is looked up again on every call made outside stream capture
// (so a context created anew after cudaDeviceReset gets its own module's address); a
// call made while `s` is capturing reuses the address the last uncaptured call on this
// device found, because lookups that may load a module do not belong in a capture.
cudaError_t scratch_for_current_device(cudaStream_t s, double **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone || !g_scratch_ptr[dev]) {
    if (cap != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
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
  cudaError_t e = scratch_for_current_device(static_cast<cudaStream_t>(stream), &scratch);
  if (e == cudaErrorStreamCaptureUnsupported)
    return tr::record_error(TR_ERR_INVALID_ARG,
                            "the first call on a device must come before any stream capture");
  if (e != cudaSuccess)
    return tr::record_error(TR_ERR_CUDA, "scratch address: %s", cudaGetErrorString(e));
  const int64_t elems = (int64_t)d_k * d_v;
  e = tr::launch_state_error(S, S_hat, n_mats, elems, tr::state_error_splits(n_mats, elems, kStaticMats),
                             scratch, err_per_mat, err_total, static_cast<cudaStream_t>(stream),
                             true);
  if (e != cudaSuccess)
    return tr::record_error(TR_ERR_CUDA, "state error: %s", cudaGetErrorString(e));
  return tr::record_error(TR_OK, "");
}
