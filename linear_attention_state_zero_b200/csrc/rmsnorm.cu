// rmsnorm.cu -- x_hat = bf16(x / sqrt(mean(x^2) + eps) * gain), one warp per row.
// HBM-bound: reads the row once (bf16 or fp32, 16-byte vectors), writes bf16.  Widths
// 1024/2048/4096 keep the row in registers; other widths (multiples of 8) loop twice.
#include <cuda_bf16.h>

#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

constexpr int kWarps = 8;

template <bool IN_BF16>
__global__ void __launch_bounds__(kWarps * 32)
    rmsnorm_kernel(const void *__restrict__ x, const float *__restrict__ gain, int64_t rows,
                   int D, float eps, __nv_bfloat16 *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  pdl_trigger();
  pdl_wait();
  if (row >= rows) return;
  const int nvec = D / 8;  // 8 elements per vector step
  float ss = 0.f;
  // pass 1: sum of squares
  for (int v = lane; v < nvec; v += 32) {
    float f[8];
    if (IN_BF16) {
      const uint4 p = reinterpret_cast<const uint4 *>(
          reinterpret_cast<const __nv_bfloat16 *>(x) + row * D)[v];
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&p);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
      }
    } else {
      const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + row * D);
      float4 a = p[2 * v], b = p[2 * v + 1];
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
      f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)D + eps);
  // pass 2: scale and store (the row is still in L1/L2)
  for (int v = lane; v < nvec; v += 32) {
    float f[8];
    if (IN_BF16) {
      const uint4 p = reinterpret_cast<const uint4 *>(
          reinterpret_cast<const __nv_bfloat16 *>(x) + row * D)[v];
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&p);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
      }
    } else {
      const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + row * D);
      float4 a = p[2 * v], b = p[2 * v + 1];
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
      f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    float g[8];
    if (gain) {
      const float4 *gp = reinterpret_cast<const float4 *>(gain);
      float4 a = gp[2 * v], b = gp[2 * v + 1];
      g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
      g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = 1.f;
    }
    uint4 o;
    __nv_bfloat162 *oh = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      oh[i] = __floats2bfloat162_rn(f[2 * i] * r * g[2 * i], f[2 * i + 1] * r * g[2 * i + 1]);
    reinterpret_cast<uint4 *>(out + row * D)[v] = o;
  }
}

// Whole row in registers: NV vectors of 8 elements per lane (D = 256 NV), all loads issued
// before the reduction, one pass over HBM.
constexpr int kRegWarps = 4;  // small blocks: up to ~130 registers per thread, 3+ blocks per SM

template <bool IN_BF16, int NV>
__global__ void __launch_bounds__(kRegWarps * 32)
    rmsnorm_reg_kernel(const void *__restrict__ x, const float *__restrict__ gain, int64_t rows,
                       float eps, __nv_bfloat16 *__restrict__ out) {
  constexpr int D = 256 * NV;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kRegWarps + (threadIdx.x >> 5);
  pdl_trigger();
  pdl_wait();
  if (row >= rows) return;
  float f[NV][8];
  if (IN_BF16) {
    const uint4 *p = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(x) + row * D);
    uint4 u[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) u[j] = p[lane + 32 * j];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u[j]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h[i]);
        f[j][2 * i] = t.x;
        f[j][2 * i + 1] = t.y;
      }
    }
  } else {
    const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + row * D);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const float4 a = p[2 * (lane + 32 * j)], b = p[2 * (lane + 32 * j) + 1];
      f[j][0] = a.x; f[j][1] = a.y; f[j][2] = a.z; f[j][3] = a.w;
      f[j][4] = b.x; f[j][5] = b.y; f[j][6] = b.z; f[j][7] = b.w;
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[j][i], f[j][i], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)D + eps);
  uint4 *op = reinterpret_cast<uint4 *>(out + row * D);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    float g[8];
    if (gain) {
      const float4 *gp = reinterpret_cast<const float4 *>(gain);
      const float4 a = gp[2 * (lane + 32 * j)], b = gp[2 * (lane + 32 * j) + 1];
      g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
      g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = 1.f;
    }
    uint4 o;
    __nv_bfloat162 *oh = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      oh[i] = __floats2bfloat162_rn(f[j][2 * i] * r * g[2 * i], f[j][2 * i + 1] * r * g[2 * i + 1]);
    op[lane + 32 * j] = o;
  }
}

template <int NV>
cudaError_t launch_reg(const void *x, int x_is_bf16, const float *gain, int64_t rows, float eps,
                __nv_bfloat16 *o, cudaStream_t s, bool pdl) {
  const unsigned blocks = (unsigned)((rows + kRegWarps - 1) / kRegWarps);
  return x_is_bf16 ? launch_kernel(rmsnorm_reg_kernel<true, NV>, dim3(blocks), dim3(kRegWarps * 32), 0,
                                   s, pdl, x, gain, rows, eps, o)
                   : launch_kernel(rmsnorm_reg_kernel<false, NV>, dim3(blocks), dim3(kRegWarps * 32),
                                   0, s, pdl, x, gain, rows, eps, o);
}

}  // namespace

cudaError_t launch_rmsnorm(const void *x, int x_is_bf16, const float *gain, int64_t rows, int D,
                           float eps, void *out, cudaStream_t s, bool pdl) {
  if (rows <= 0) return cudaSuccess;
  const int64_t blocks = (rows + kWarps - 1) / kWarps;
  auto *o = reinterpret_cast<__nv_bfloat16 *>(out);
  switch (D) {  // common model widths: whole row in registers
    case 1024: return launch_reg<4>(x, x_is_bf16, gain, rows, eps, o, s, pdl);
    case 2048: return launch_reg<8>(x, x_is_bf16, gain, rows, eps, o, s, pdl);
    case 4096: return launch_reg<16>(x, x_is_bf16, gain, rows, eps, o, s, pdl);
    default: break;
  }
  return x_is_bf16 ? launch_kernel(rmsnorm_kernel<true>, dim3((unsigned)blocks), dim3(kWarps * 32), 0,
                                   s, pdl, x, gain, rows, D, eps, o)
                   : launch_kernel(rmsnorm_kernel<false>, dim3((unsigned)blocks), dim3(kWarps * 32),
                                   0, s, pdl, x, gain, rows, D, eps, o);
}

}  // namespace tr
