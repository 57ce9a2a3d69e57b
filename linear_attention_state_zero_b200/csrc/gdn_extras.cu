// gdn_extras.cu -- the optional Gated DeltaNet layer details around the scan
// (the pages give no layer internals; these are the public Gated DeltaNet layer's):
//   short_conv_kernel : causal depthwise convolution (width 2..4) + silu over the bf16
//                       q/k/v projections, zero history at each sequence start (the
//                       replay starts every state at zero, the convolution's included),
//                       then the per-head L2 norm of q and k; also writes each sequence's
//                       convolution state (its last width-1 inputs)
//   gated_norm_kernel : o <- bf16(RMSNorm_{d_v}(o) * gain * silu(z)) per token and head
// Both are HBM-bound streaming passes (each input row read once, each output row written
// once), fp32 arithmetic.
#include <math.h>

#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

constexpr int kThreads = 256;

// silu with the fast division intrinsic (relative error ~1e-7, far below the bf16 output's
// 4e-3); where e^{-y} overflows the quotient is -0, the limit.
__device__ __forceinline__ float silu_f(float y) { return __fdividef(y, 1.f + exp_ftz(-y)); }

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

// 16-byte asynchronous global -> shared copy (cp.async, cache-global) and its group wait.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Segments: H q heads (d_k wide), H k heads (d_k), H v heads (d_v); all one width D here
// (d_k = d_v = D, 64 or 128).  A tile is kTileTok tokens x kTileSeg segments: the block
// copies its input rows (the tile's tokens and the W-1 before them) into shared memory with
// asynchronous 16-byte copies, so a whole tile's bytes are in flight at once; then warp w
// takes segment w % kTileSeg and half w / kTileSeg of the tokens, keeps its taps in
// registers and reads the window from shared memory.  Blocks after the tiles write the
// convolution state, one warp per (sequence, segment).
constexpr int kTileTok = 32;
constexpr int kTileSeg = 4;
constexpr int kHalfTok = kTileTok / 2;
constexpr int kGroup = 4;
static_assert(kHalfTok % kGroup == 0, "token groups tile a half");
static_assert(kThreads / 32 == 2 * kTileSeg, "two warps per tile segment");

template <int D, int W>
__global__ void __launch_bounds__(kThreads)
    short_conv_kernel(ShortConvLaunch p) {
  constexpr int VPL = D / 32;
  constexpr int ROWS = kTileTok + W - 1;
  constexpr int COLS = kTileSeg * D;
  __shared__ __align__(16) __nv_bfloat16 tile[ROWS][COLS];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg0 = p.skip_q ? p.H : 0;
  const int n_seg = 3 * p.H - seg0;
  const int seg_groups = (n_seg + kTileSeg - 1) / kTileSeg;
  const int64_t n_tiles = (p.T + kTileTok - 1) / kTileTok * seg_groups;
  const int64_t n_pairs = p.state ? (int64_t)p.n_seqs * n_seg : 0;
  const int64_t n_blocks = n_tiles + (n_pairs + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t C = (int64_t)3 * p.H * D;
  for (int64_t bt = blockIdx.x; bt < n_blocks; bt += gridDim.x) {
    if (bt < n_tiles) {
      const int sg = (int)(bt % seg_groups);
      const int64_t t0 = bt / seg_groups * kTileTok;
      const int seg_a = seg0 + sg * kTileSeg;
      const int nseg = n_seg - sg * kTileSeg < kTileSeg ? n_seg - sg * kTileSeg : kTileSeg;
      const int64_t rbase = t0 - (W - 1);  // token of shared row 0
      const int cpr = nseg * D / 8;        // 16-byte pieces per row
      for (int c = threadIdx.x; c < ROWS * cpr; c += kThreads) {
        const int r = c / cpr, q = c - r * cpr;
        const int64_t src = rbase + r;
        __nv_bfloat16 *dst = &tile[r][q * 8];
        if (src >= 0 && src < p.T)
          cp_async16(dst, p.pre + src * p.ld + (int64_t)seg_a * D + q * 8);
        else
          *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
      cp_async_wait_all();
      __syncthreads();
      const int sl = warp % kTileSeg;
      const int64_t ta = t0 + (warp / kTileSeg) * kHalfTok;
      const int64_t tz = ta + kHalfTok < p.T ? ta + kHalfTok : p.T;
      if (sl < nseg && ta < tz) {
        const int seg = seg_a + sl;
        const int c0 = seg * D + lane * VPL;  // first global channel of this lane
        const int cs = sl * D + lane * VPL;   // the same channel in the tile
        const bool qk = seg < 2 * p.H;
        float wv[VPL][W];
#pragma unroll
        for (int i = 0; i < VPL; ++i)
#pragma unroll
          for (int j = 0; j < W; ++j) wv[i][j] = p.w[(int64_t)(c0 + i) * W + j];
        int s = seq_of(p.cu_seqlens, p.n_seqs, ta);
        int64_t next = p.cu_seqlens[s + 1];  // first token after this sequence
        int64_t cur = p.cu_seqlens[s];       // first token of this sequence
        // kGroup tokens at a time: their windows, silu and norms are independent, so the
        // reductions interleave (rows past the tile's last token are zero-filled and only
        // computed, never stored)
        for (int64_t tg = ta; tg < tz; tg += kGroup) {
          int64_t first[kGroup];
#pragma unroll
          for (int b = 0; b < kGroup; ++b) {
            const int64_t t = tg + b;
            if (t < tz && t >= next) {  // a new sequence starts here (empty ones skipped)
              while (t >= next) next = p.cu_seqlens[++s + 1];
              cur = p.cu_seqlens[s];
            }
            first[b] = cur;
          }
          float y[kGroup][VPL], ssq[kGroup];
#pragma unroll
          for (int b = 0; b < kGroup; ++b) {
            const int64_t t = tg + b;
#pragma unroll
            for (int i = 0; i < VPL; ++i) y[b][i] = 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) {
              const int64_t src = t - (W - 1) + j;
              float x[VPL];
              load_bf16<VPL>(&tile[src - rbase][cs], x);
              const bool in = src >= first[b];
#pragma unroll
              for (int i = 0; i < VPL; ++i) y[b][i] = fmaf(wv[i][j], in ? x[i] : 0.f, y[b][i]);
            }
            ssq[b] = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
              y[b][i] = silu_f(y[b][i]);
              ssq[b] = fmaf(y[b][i], y[b][i], ssq[b]);
            }
          }
          if (qk) {  // q or k head: L2 norm over its D channels
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
              for (int b = 0; b < kGroup; ++b) ssq[b] += __shfl_xor_sync(0xffffffffu, ssq[b], o);
#pragma unroll
            for (int b = 0; b < kGroup; ++b) {
              const float inv = rsqrtf(ssq[b] + p.norm_eps);
#pragma unroll
              for (int i = 0; i < VPL; ++i) y[b][i] *= inv;
            }
          }
#pragma unroll
          for (int b = 0; b < kGroup; ++b)
            if (tg + b < tz) store_bf16<VPL>(p.post + (tg + b) * p.ld + c0, y[b]);
        }
      }
      __syncthreads();  // the next tile reuses the shared rows
    } else {
      const int64_t pair = (bt - n_tiles) * (kThreads / 32) + warp;
      if (pair < n_pairs) {
        const int s = (int)(pair / n_seg);
        const int seg = seg0 + (int)(pair % n_seg);
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
      } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i) v[b][i] = zz[b][i] = 0.f;
      }
    }
    float ssq[kRows];
#pragma unroll
    for (int b = 0; b < kRows; ++b) {
      ssq[b] = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) ssq[b] = fmaf(v[b][i], v[b][i], ssq[b]);
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1)
#pragma unroll
      for (int b = 0; b < kRows; ++b) ssq[b] += __shfl_xor_sync(0xffffffffu, ssq[b], o2);
#pragma unroll
    for (int b = 0; b < kRows; ++b) {
      const float inv = rsqrtf(ssq[b] * (1.f / D) + eps);
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[b][i] = v[b][i] * inv * g[i] * silu_f(zz[b][i]);
      if (r0 + b < n_rows) store_bf16<VPL>(o + (r0 + b) * D + lane * VPL, v[b]);
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
  const int64_t tiles = (p.T + kTileTok - 1) / kTileTok * ((n_seg + kTileSeg - 1) / kTileSeg);
  const int64_t pairs = p.state ? (int64_t)p.n_seqs * n_seg : 0;
  int64_t blocks = tiles + (pairs + kThreads / 32 - 1) / (kThreads / 32);
  if (blocks == 0) return cudaSuccess;
  const int64_t cap = (int64_t)device_sm_count() * 8;
  const int grid = (int)(blocks < cap ? blocks : cap);
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
