// gdn_extras.cu -- the optional Gated DeltaNet layer details around the scan
// (the pages give no layer internals; these are the public Gated DeltaNet layer's):
//   short_conv_kernel : causal depthwise convolution (width 2..4) + silu over the bf16
//                       q/k/v projections, zero history at each sequence start (the
//                       replay starts every state at zero, the convolution's included),
//                       then the per-head L2 norm of q and k; also writes each sequence's
//                       convolution state (its last width-1 inputs)
//   gated_norm_kernel : o <- bf16(RMSNorm_{d_v}(o) * gain * silu(z)) per token and head
// Both are HBM-bound streaming passes (each input row read once, each output row written
// once), 8-byte or 4-byte loads per lane, fp32 arithmetic.
#include <math.h>

#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float silu_f(float y) { return y / (1.f + exp_ftz(-y)); }

// sequence index of token t: the last s with cu[s] <= t (cu non-decreasing)
__device__ __forceinline__ int seq_of(const int32_t *__restrict__ cu, int n_seqs, int64_t t) {
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// VPL values per lane (4 for 128-wide segments, 2 for 64-wide)
template <int VPL>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16 *p, float (&v)[VPL]) {
  if constexpr (VPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
  } else {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(p);
    v[0] = __low2float(a); v[1] = __high2float(a);
  }
}

template <int VPL>
__device__ __forceinline__ void store_bf16(__nv_bfloat16 *p, const float (&v)[VPL]) {
  if constexpr (VPL == 4) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
  } else {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v[0], v[1]);
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Segments: H q heads (d_k wide), H k heads (d_k), H v heads (d_v); all one width D here
// (d_k = d_v = D, 64 or 128).  Work units 0 .. n_chunks*n_seg-1 are (32-token chunk,
// segment) pairs, segment fastest, so a block's warps read the same rows: the warp loads
// its taps once, keeps the last W-1 inputs in registers and streams the chunk's rows with
// kBatch loads in flight.  Units after that are (sequence, segment) pairs that write the
// convolution state.
constexpr int kTokChunk = 32;
constexpr int kBatch = 8;

template <int D, int W>
__global__ void __launch_bounds__(kThreads)
    short_conv_kernel(ShortConvLaunch p) {
  constexpr int VPL = D / 32;
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int seg0 = p.skip_q ? p.H : 0;
  const int n_seg = 3 * p.H - seg0;
  const int64_t n_chunks = (p.T + kTokChunk - 1) / kTokChunk;
  const int64_t n_conv = n_chunks * n_seg;
  const int64_t n_units = n_conv + (p.state ? (int64_t)p.n_seqs * n_seg : 0);
  const int64_t C = (int64_t)3 * p.H * D;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t u = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); u < n_units;
       u += warps) {
    if (u < n_conv) {
      const int seg = seg0 + (int)(u % n_seg);
      const int64_t t0 = (u / n_seg) * kTokChunk;
      const int64_t t1 = t0 + kTokChunk < p.T ? t0 + kTokChunk : p.T;
      const int c0 = seg * D + lane * VPL;  // first channel of this lane
      const bool qk = seg < 2 * p.H;
      float wv[VPL][W];
#pragma unroll
      for (int i = 0; i < VPL; ++i)
#pragma unroll
        for (int j = 0; j < W; ++j) wv[i][j] = p.w[(int64_t)(c0 + i) * W + j];
      int s = seq_of(p.cu_seqlens, p.n_seqs, t0);
      int64_t next = p.cu_seqlens[s + 1];  // first token after this sequence
      // history of t0: the W-1 inputs before it inside its sequence, oldest first
      const int64_t start = p.cu_seqlens[s];
      float hist[W - 1][VPL];
#pragma unroll
      for (int j = 0; j < W - 1; ++j) {
        const int64_t src = t0 - (W - 1) + j;
        if (src >= start) {
          load_bf16<VPL>(p.pre + src * p.ld + c0, hist[j]);
        } else {
#pragma unroll
          for (int i = 0; i < VPL; ++i) hist[j][i] = 0.f;
        }
      }
      for (int64_t tb = t0; tb < t1; tb += kBatch) {
        float xb[kBatch][VPL];
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
          if (tb + b < t1) load_bf16<VPL>(p.pre + (tb + b) * p.ld + c0, xb[b]);
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int64_t t = tb + b;
          if (t >= t1) break;
          if (t >= next) {  // a new sequence starts here (skipping empty ones): zero history
            while (t >= next) next = p.cu_seqlens[++s + 1];
#pragma unroll
            for (int j = 0; j < W - 1; ++j)
#pragma unroll
              for (int i = 0; i < VPL; ++i) hist[j][i] = 0.f;
          }
          float y[VPL];
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < W - 1; ++j) acc = fmaf(wv[i][j], hist[j][i], acc);
            y[i] = silu_f(fmaf(wv[i][W - 1], xb[b][i], acc));
          }
          if (qk) {  // q or k head: L2 norm over its D channels
            float ssq = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) ssq = fmaf(y[i], y[i], ssq);
            const float inv = rsqrtf(warp_sum(ssq) + p.norm_eps);
#pragma unroll
            for (int i = 0; i < VPL; ++i) y[i] *= inv;
          }
          store_bf16<VPL>(p.post + t * p.ld + c0, y);
#pragma unroll
          for (int j = 0; j + 1 < W - 1; ++j)
#pragma unroll
            for (int i = 0; i < VPL; ++i) hist[j][i] = hist[j + 1][i];
#pragma unroll
          for (int i = 0; i < VPL; ++i) hist[W - 2][i] = xb[b][i];
        }
      }
    } else {
      const int64_t r = u - n_conv;
      const int s = (int)(r / n_seg);
      const int seg = seg0 + (int)(r % n_seg);
      const int64_t start = p.cu_seqlens[s], end = p.cu_seqlens[s + 1];
      const int c0 = seg * D + lane * VPL;
#pragma unroll
      for (int i = 0; i < W - 1; ++i) {
        const int64_t t = end - (W - 1) + i;
        float x[VPL];
        if (t >= start) {
          load_bf16<VPL>(p.pre + t * p.ld + c0, x);
        } else {
#pragma unroll
          for (int u2 = 0; u2 < VPL; ++u2) x[u2] = 0.f;
        }
        store_bf16<VPL>(p.state + ((int64_t)s * (W - 1) + i) * C + c0, x);
      }
    }
  }
}

// Rows of (token, head) with kRows rows per warp in flight.
constexpr int kRows = 4;

template <int D>
__global__ void __launch_bounds__(kThreads)
    gated_norm_kernel(__nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ z,
                      const float *__restrict__ gain, int64_t n_rows, float eps) {
  constexpr int VPL = D / 32;
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  float g[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) g[i] = gain ? gain[lane * VPL + i] : 1.f;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t r0 = ((int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5)) * kRows;
       r0 < n_rows; r0 += warps * kRows) {
    float v[kRows][VPL], zz[kRows][VPL];
#pragma unroll
    for (int b = 0; b < kRows; ++b) {
      if (r0 + b < n_rows) {
        load_bf16<VPL>(o + (r0 + b) * D + lane * VPL, v[b]);
        load_bf16<VPL>(z + (r0 + b) * D + lane * VPL, zz[b]);
      }
    }
#pragma unroll
    for (int b = 0; b < kRows; ++b) {
      if (r0 + b >= n_rows) break;
      float ssq = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) ssq = fmaf(v[b][i], v[b][i], ssq);
      const float inv = rsqrtf(warp_sum(ssq) * (1.f / D) + eps);
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[b][i] = v[b][i] * inv * g[i] * silu_f(zz[b][i]);
      store_bf16<VPL>(o + (r0 + b) * D + lane * VPL, v[b]);
    }
  }
}

int grid_for(int64_t warp_items) {
  int64_t b = (warp_items + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t cap = (int64_t)device_sm_count() * 8;
  if (b > cap) b = cap;
  return b < 1 ? 1 : (int)b;
}

template <int D>
cudaError_t conv_dispatch_w(const ShortConvLaunch &p, int grid, cudaStream_t s, bool pdl) {
  switch (p.width) {
    case 2: return launch_kernel(short_conv_kernel<D, 2>, dim3(grid), dim3(kThreads), 0, s, pdl, p);
    case 3: return launch_kernel(short_conv_kernel<D, 3>, dim3(grid), dim3(kThreads), 0, s, pdl, p);
    case 4: return launch_kernel(short_conv_kernel<D, 4>, dim3(grid), dim3(kThreads), 0, s, pdl, p);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_short_conv(const ShortConvLaunch &p, cudaStream_t s, bool pdl) {
  if (p.dk != p.dv || (p.dk != 64 && p.dk != 128)) return cudaErrorInvalidValue;
  const int n_seg = 3 * p.H - (p.skip_q ? p.H : 0);
  const int64_t units = (p.T + kTokChunk - 1) / kTokChunk * n_seg +
                        (p.state ? (int64_t)p.n_seqs * n_seg : 0);
  if (units == 0) return cudaSuccess;
  const int grid = grid_for(units);
  return p.dk == 128 ? conv_dispatch_w<128>(p, grid, s, pdl) : conv_dispatch_w<64>(p, grid, s, pdl);
}

cudaError_t launch_gated_norm(__nv_bfloat16 *o, const __nv_bfloat16 *z, const float *gain,
                              int64_t T, int H, int dv, float eps, cudaStream_t s, bool pdl) {
  const int64_t rows = T * H;
  if (rows == 0) return cudaSuccess;
  const int grid = grid_for((rows + kRows - 1) / kRows);
  if (dv == 128)
    return launch_kernel(gated_norm_kernel<128>, dim3(grid), dim3(kThreads), 0, s, pdl, o, z, gain,
                         rows, eps);
  if (dv == 64)
    return launch_kernel(gated_norm_kernel<64>, dim3(grid), dim3(kThreads), 0, s, pdl, o, z, gain,
                         rows, eps);
  return cudaErrorInvalidValue;
}

}  // namespace tr
