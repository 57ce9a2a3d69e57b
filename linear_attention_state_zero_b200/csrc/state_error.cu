// state_error.cu -- ||S - S_hat||_F / ||S||_F per matrix and in total, with fp64
// accumulation of the fp32 states.  HBM-bound: each state is read once.
//   pass 1: each matrix is cut into `splits` contiguous pieces, one block per piece ->
//           (sum (S - S_hat)^2, sum S^2) of the piece into `partials`
//   pass 2: one block; thread t folds the pieces of matrices t, t + blockDim, ... in
//           piece order -> per-matrix ratio, then a fixed tree -> the total ratio
// Every sum runs in a fixed order, so results are bitwise reproducible.
#include <math.h>

#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

constexpr int kThreads = 256;
constexpr int kTotalThreads = 1024;

__device__ __forceinline__ double ratio_or_special(double num, double den) {
  if (den > 0.0) return sqrt(num / den);
  return num > 0.0 ? __longlong_as_double(0x7ff0000000000000ll) : 0.0;  // +inf or 0
}

template <int NT>
__device__ __forceinline__ void block_sum2(double &a, double &b) {
  __shared__ double sa[NT / 32], sb[NT / 32];
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
    a = (l < NT / 32) ? sa[l] : 0.0;
    b = (l < NT / 32) ? sb[l] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
    }
  }
}

// block b = (matrix b / splits, piece b % splits); pieces are `piece` elements long
// (a multiple of 4), the last one shorter
__global__ void __launch_bounds__(kThreads)
    state_error_partial(const float *__restrict__ S, const float *__restrict__ Sh, int64_t n_blocks,
                        int64_t mat_elems, int splits, int64_t piece,
                        double *__restrict__ partials) {
  pdl_trigger();
  pdl_wait();
  for (int64_t blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
    const int64_t m = blk / splits, j = blk % splits;
    const int64_t lo = j * piece;
    const int64_t hi = lo + piece < mat_elems ? lo + piece : mat_elems;
    const float *a = S + m * mat_elems;
    const float *b = Sh + m * mat_elems;
    double num = 0.0, den = 0.0;
    if ((mat_elems & 3) == 0) {
      const float4 *a4 = reinterpret_cast<const float4 *>(a);
      const float4 *b4 = reinterpret_cast<const float4 *>(b);
      for (int64_t i = lo / 4 + threadIdx.x; i < hi / 4; i += kThreads) {
        const float4 x = a4[i], y = b4[i];
        const double d0 = (double)x.x - y.x, d1 = (double)x.y - y.y, d2 = (double)x.z - y.z,
                     d3 = (double)x.w - y.w;
        num += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
        den += (double)x.x * x.x + (double)x.y * x.y + (double)x.z * x.z + (double)x.w * x.w;
      }
    } else {
      for (int64_t i = lo + threadIdx.x; i < hi; i += kThreads) {
        const double d = (double)a[i] - b[i];
        num += d * d;
        den += (double)a[i] * a[i];
      }
    }
    block_sum2<kThreads>(num, den);
    if (threadIdx.x == 0) {
      partials[2 * blk] = num;
      partials[2 * blk + 1] = den;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kTotalThreads)
    state_error_total(const double *__restrict__ partials, int64_t n_mats, int splits,
                      double *__restrict__ err_per, double *__restrict__ err_total) {
  pdl_trigger();
  pdl_wait();
  double num = 0.0, den = 0.0;
  for (int64_t m = threadIdx.x; m < n_mats; m += kTotalThreads) {
    double nm = 0.0, dm = 0.0;
    for (int j = 0; j < splits; ++j) {
      nm += partials[2 * (m * splits + j)];
      dm += partials[2 * (m * splits + j) + 1];
    }
    if (err_per) err_per[m] = ratio_or_special(nm, dm);
    num += nm;
    den += dm;
  }
  block_sum2<kTotalThreads>(num, den);
  if (threadIdx.x == 0 && err_total) *err_total = ratio_or_special(num, den);
}

}  // namespace

int state_error_splits(int64_t n_mats, int64_t mat_elems, int64_t max_pieces) {
  // pieces of >= 2048 elements (8 KB per array), at most 16 per matrix, and no more
  // pieces in all than `max_pieces`
  int64_t s = mat_elems / 2048;
  if (s > 16) s = 16;
  if (n_mats > 0 && s * n_mats > max_pieces) s = max_pieces / n_mats;
  return s < 1 ? 1 : (int)s;
}

cudaError_t launch_state_error(const float *S, const float *Sh, int64_t n_mats, int64_t mat_elems,
                               int splits, double *partials, double *err_per, double *err_total,
                               cudaStream_t s, bool pdl) {
  if (!err_per && !err_total) return cudaSuccess;
  if (n_mats > 0) {
    int64_t piece = (mat_elems + splits - 1) / splits;
    piece = (piece + 3) & ~static_cast<int64_t>(3);
    const int64_t n_blocks = n_mats * splits;
    const int64_t grid = n_blocks < 65535 * 8 ? n_blocks : 65535 * 8;
    cudaError_t e = launch_kernel(state_error_partial, dim3((unsigned)grid), dim3(kThreads), 0, s,
                                  pdl, S, Sh, n_blocks, mat_elems, splits, piece, partials);
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(state_error_total, dim3(1), dim3(kTotalThreads), 0, s, pdl,
                       (const double *)partials, n_mats, splits, err_per, err_total);
}

}  // namespace tr
