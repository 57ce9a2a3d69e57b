// state_error.cu -- ||S - S_hat||_F / ||S||_F per matrix and in total, with fp64
// accumulation of the fp32 states.  HBM-bound: each state is read once.
//   pass 1: one block per matrix -> (sum (S - S_hat)^2, sum S^2) into `partials`,
//           and the per-matrix ratio
//   pass 2: one block folds the partials in a fixed order -> the total ratio
// The reduction order is fixed, so results are bitwise reproducible.
#include <math.h>

#include "tr_internal.h"

namespace tr {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ double ratio_or_special(double num, double den) {
  if (den > 0.0) return sqrt(num / den);
  return num > 0.0 ? __longlong_as_double(0x7ff0000000000000ll) : 0.0;  // +inf or 0
}

__device__ __forceinline__ void block_sum2(double &a, double &b) {
  __shared__ double sa[kThreads / 32], sb[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    sa[w] = a;
    sb[w] = b;
  }
  __syncthreads();
  if (w == 0) {
    a = (l < kThreads / 32) ? sa[l] : 0.0;
    b = (l < kThreads / 32) ? sb[l] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
    }
  }
}

__global__ void __launch_bounds__(kThreads)
    state_error_partial(const float *__restrict__ S, const float *__restrict__ Sh, int64_t n_mats,
                        int64_t mat_elems, double *__restrict__ partials,
                        double *__restrict__ err_per) {
  for (int64_t m = blockIdx.x; m < n_mats; m += gridDim.x) {
    const float *a = S + m * mat_elems;
    const float *b = Sh + m * mat_elems;
    double num = 0.0, den = 0.0;
    if ((mat_elems & 3) == 0) {
      const float4 *a4 = reinterpret_cast<const float4 *>(a);
      const float4 *b4 = reinterpret_cast<const float4 *>(b);
      for (int64_t i = threadIdx.x; i < mat_elems / 4; i += kThreads) {
        const float4 x = a4[i], y = b4[i];
        const double d0 = (double)x.x - y.x, d1 = (double)x.y - y.y, d2 = (double)x.z - y.z,
                     d3 = (double)x.w - y.w;
        num += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
        den += (double)x.x * x.x + (double)x.y * x.y + (double)x.z * x.z + (double)x.w * x.w;
      }
    } else {
      for (int64_t i = threadIdx.x; i < mat_elems; i += kThreads) {
        const double d = (double)a[i] - b[i];
        num += d * d;
        den += (double)a[i] * a[i];
      }
    }
    block_sum2(num, den);
    if (threadIdx.x == 0) {
      partials[2 * m] = num;
      partials[2 * m + 1] = den;
      if (err_per) err_per[m] = ratio_or_special(num, den);
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads)
    state_error_total(const double *__restrict__ partials, int64_t n_mats, double *err_total) {
  double num = 0.0, den = 0.0;
  for (int64_t m = threadIdx.x; m < n_mats; m += kThreads) {
    num += partials[2 * m];
    den += partials[2 * m + 1];
  }
  block_sum2(num, den);
  if (threadIdx.x == 0) *err_total = ratio_or_special(num, den);
}

}  // namespace

cudaError_t launch_state_error(const float *S, const float *Sh, int64_t n_mats, int64_t mat_elems,
                               double *partials, double *err_per, double *err_total,
                               cudaStream_t s) {
  if (n_mats > 0) {
    const int64_t grid = n_mats < 65535 * 8 ? n_mats : 65535 * 8;
    state_error_partial<<<(unsigned)grid, kThreads, 0, s>>>(S, Sh, n_mats, mat_elems, partials,
                                                           err_per);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (err_total) {
    state_error_total<<<1, kThreads, 0, s>>>(partials, n_mats, err_total);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace tr
