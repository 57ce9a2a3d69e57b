// scan_recurrent.cu -- token-sequential Gated DeltaNet scan in fp32 FMA (no
// tensor cores, no TF32): the fp32 test path of tr_gdn_scan, and the fallback
// for bf16 inputs when TR_SCAN_RECURRENT is set.
//
// Eq. (1) in the M = S^T layout, one token at a time:
//   w = k_t^T M                       (a row over the d_v columns)
//   M <- alpha_t M + k_t (beta_t (v_t - alpha_t w))^T
//      = alpha_t (M - beta_t k_t w) + beta_t k_t v_t^T
//   o_t = scale * M^T q_t
// Every column of M evolves independently (all M-dependent products act
// column-wise), so a block owns 32 columns of one (sequence, head): each warp
// 8 columns, each lane one column and a quarter of the d_k rows; the two
// d_k-reductions per token are 2-step shuffles.  Tokens are staged through
// shared memory 16 at a time.
#include <cuda_bf16.h>

#include "../../include/tr.h"
#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

template <typename T>
__device__ __forceinline__ float ldf(const T *p);
template <>
__device__ __forceinline__ float ldf<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void stf(T *p, float v);
template <>
__device__ __forceinline__ void stf<float>(float *p, float v) { *p = v; }
template <>
__device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
  *p = __float2bfloat16_rn(v);
}

template <int DK, typename T>
__global__ void __launch_bounds__(128) scan_recurrent_kernel(ScanLaunch p) {
  constexpr int R = DK / 4;   // d_k rows per lane
  constexpr int RP = R + 1;   // padded row-group stride (bank-conflict free)
  constexpr int TT = 16;      // tokens staged per tile
  __shared__ float ks[TT][4 * RP];
  __shared__ float qs[TT][4 * RP];
  __shared__ float vs[TT][32];
  __shared__ float las[TT], bes[TT];

  pdl_trigger();
  pdl_wait();
  const int sh = blockIdx.x;
  const int seq = sh / p.H, head = sh % p.H;
  const int col0 = blockIdx.y * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane >> 3, c = lane & 7;
  const int col = col0 + warp * 8 + c;
  const int64_t t0 = p.cu_seqlens[seq], t1 = p.cu_seqlens[seq + 1];
  const bool norm = (p.flags & TR_NORMALIZE_QK) != 0;
  const bool want_o = p.o != nullptr;
  const T *q = reinterpret_cast<const T *>(p.q);
  const T *k = reinterpret_cast<const T *>(p.k);
  const T *v = reinterpret_cast<const T *>(p.v);
  T *o = reinterpret_cast<T *>(p.o);

  const int64_t sbase = ((int64_t)seq * p.H + head) * (int64_t)DK * p.dv;
  float M[R];
#pragma unroll
  for (int i = 0; i < R; ++i) M[i] = p.S0 ? p.S0[sbase + (int64_t)(rg * R + i) * p.dv + col] : 0.f;

  for (int64_t tb = t0; tb < t1; tb += TT) {
    const int nt = (int)min((int64_t)TT, t1 - tb);
    __syncthreads();
    for (int idx = threadIdx.x; idx < TT * DK; idx += 128) {
      const int tt = idx / DK, d = idx % DK;
      float kv = 0.f, qv = 0.f;
      if (tt < nt) {
        const int64_t t = tb + tt;
        kv = ldf<T>(k + t * p.k_stride + (int64_t)head * DK + d);
        if (want_o) qv = ldf<T>(q + t * p.q_stride + (int64_t)head * DK + d);
      }
      const int pos = (d / R) * RP + (d % R);
      ks[tt][pos] = kv;
      qs[tt][pos] = qv;
    }
    for (int idx = threadIdx.x; idx < TT * 32; idx += 128) {
      const int tt = idx >> 5, j = idx & 31;
      vs[tt][j] = (tt < nt) ? ldf<T>(v + (tb + tt) * p.v_stride + (int64_t)head * p.dv + col0 + j)
                            : 0.f;
    }
    if (threadIdx.x < TT) {
      const int tt = threadIdx.x;
      las[tt] = (tt < nt) ? p.log_alpha[(tb + tt) * p.H + head] : 0.f;
      bes[tt] = (tt < nt) ? p.beta[(tb + tt) * p.H + head] : 0.f;
    }
    __syncthreads();
    if (norm) {
      // x / sqrt(sum x^2 + 1e-6) for every staged k and q row
      for (int tt = warp; tt < nt; tt += 4) {
        float sk = 0.f, sq = 0.f;
        for (int d = lane; d < DK; d += 32) {
          const int pos = (d / R) * RP + (d % R);
          sk = fmaf(ks[tt][pos], ks[tt][pos], sk);
          sq = fmaf(qs[tt][pos], qs[tt][pos], sq);
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) {
          sk += __shfl_xor_sync(0xffffffffu, sk, o2);
          sq += __shfl_xor_sync(0xffffffffu, sq, o2);
        }
        const float ik = rsqrtf(sk + 1e-6f), iq = rsqrtf(sq + 1e-6f);
        for (int d = lane; d < DK; d += 32) {
          const int pos = (d / R) * RP + (d % R);
          ks[tt][pos] *= ik;
          qs[tt][pos] *= iq;
        }
      }
      __syncthreads();
    }
    for (int tt = 0; tt < nt; ++tt) {
      const float *kr = &ks[tt][rg * RP];
      float w = 0.f;
#pragma unroll
      for (int i = 0; i < R; ++i) w = fmaf(kr[i], M[i], w);
      w += __shfl_xor_sync(0xffffffffu, w, 8);
      w += __shfl_xor_sync(0xffffffffu, w, 16);
      const float a = expf(las[tt]);
      const float u = bes[tt] * (vs[tt][warp * 8 + c] - a * w);
#pragma unroll
      for (int i = 0; i < R; ++i) M[i] = fmaf(a, M[i], kr[i] * u);
      if (want_o) {
        const float *qr = &qs[tt][rg * RP];
        float ov = 0.f;
#pragma unroll
        for (int i = 0; i < R; ++i) ov = fmaf(qr[i], M[i], ov);
        ov += __shfl_xor_sync(0xffffffffu, ov, 8);
        ov += __shfl_xor_sync(0xffffffffu, ov, 16);
        if (rg == 0) stf<T>(o + (tb + tt) * p.o_stride + (int64_t)head * p.dv + col, ov * p.scale);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) p.S_final[sbase + (int64_t)(rg * R + i) * p.dv + col] = M[i];
}

}  // namespace

cudaError_t launch_scan_recurrent(const ScanLaunch &p, cudaStream_t s) {
  if (p.n_seqs == 0) return cudaSuccess;
  dim3 grid((unsigned)(p.n_seqs * p.H), (unsigned)(p.dv / 32));
  const bool bf = p.dtype == TR_DTYPE_BF16;
  if (p.dk == 128) {
    return bf ? launch_kernel(scan_recurrent_kernel<128, __nv_bfloat16>, grid, dim3(128), 0, s, p.pdl, p)
              : launch_kernel(scan_recurrent_kernel<128, float>, grid, dim3(128), 0, s, p.pdl, p);
  }
  return bf ? launch_kernel(scan_recurrent_kernel<64, __nv_bfloat16>, grid, dim3(128), 0, s, p.pdl, p)
            : launch_kernel(scan_recurrent_kernel<64, float>, grid, dim3(128), 0, s, p.pdl, p);
}

}  // namespace tr
