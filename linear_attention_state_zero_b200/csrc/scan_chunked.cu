// scan_chunked.cu -- chunked Gated DeltaNet scan on the 5th-generation tensor cores.
//
// Eq. (1) (Tail-Replay reading notes, section 2.3) in the M = S^T layout,
//   M_t = alpha_t (M_{t-1} - beta_t k_t (k_t^T M_{t-1})) + beta_t k_t v_t^T,
// regrouped over chunks of C = 64 tokens (the WY / UT form of the delta rule,
// derived here from Eq. (1)).  Inside a chunk, with g_t = sum_{s<=t} log alpha_s,
// gamma_t = e^{g_t}, gamma'_t = e^{g_C - g_t} and the incoming state M_0:
//   A_ts = beta_t e^{g_t - g_s} k_t.k_s  (s < t),   T = (I + A)^{-1}
//   W = T diag(beta gamma) K,   U~ = T diag(beta) V
//   P_ts = e^{g_t - g_s} q_t.k_s  (s <= t)
//   chunk transition:  M_C = gamma_C M_0 + A_c M_0 + B_c
//       A_c = -K^T diag(gamma') W   (d_k x d_k),   B_c = K^T diag(gamma') U~
//   chunk readout:     O = R M_0 + O0,   R = diag(gamma) Q - P W,   O0 = P U~
// Nothing but the last two lines depends on M_0, so the work splits in two
// launches:
//
//   scan_prep_kernel  one CTA per (chunk, head), all chunks in parallel:
//     P1  [K; Q] K^T -> TMEM            (tcgen05, K-major operands)
//     A, P on CUDA cores; T = (I + A)^{-1} by forward substitution in fp32
//     P2  [-T''; T'] [V | K] -> -U~, W  (T' = T diag(beta gamma), T'' = T diag(beta))
//     P3  P W, P U~, K^T (gamma' W), K^T (gamma' U~) in one batch
//     -> workspace: A_c (bf16), R (bf16), B_c (fp32), O0 (fp32), gamma_C
//   scan_chain_kernel one CTA per (sequence, head, 64-column slice of d_v):
//     per chunk one tcgen05 round trip:  Z = A_c M_bf16,  O = R M_bf16  (TMEM),
//     then M <- gamma_C M + Z + B_c in fp32 registers (thread d owns row d),
//     o = O + O0.  Operands arrive by TMA, double-buffered one chunk ahead.
//
// Every M-dependent product acts column by column on d_v, so d_v splits into
// exact 64-column slices.  Tokens past the end of a sequence get beta = 0 and
// log alpha = 0: their rows of T are the identity and their W, U~ rows vanish.
#include <cuda_bf16.h>

#include "../../include/tr.h"
#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

constexpr int C = 64;      // chunk length
constexpr int DK = 128;    // key dimension handled here
constexpr int DVS = 64;    // d_v columns per chain CTA
constexpr int kThreads = 128;

// --------------------------------------------------------------- helpers
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int kk, uint32_t half_stride) {
  // K-major operand: 128-byte rows, 64-column halves `half_stride` bytes apart; K step kk
  // (16 elements) starts 32 bytes further inside the 128-byte swizzle atom.
  return sw128_desc(base + (uint32_t)(kk >> 2) * half_stride + (uint32_t)(kk & 3) * 32u, 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int kk, uint32_t lbo) {
  // MN-major operand: rows are the K dimension, 128-byte rows hold 64 M/N elements,
  // 64-element M/N blocks `lbo` bytes apart; K step kk = 16 rows = 2048 bytes.
  return sw128_desc(base + (uint32_t)kk * 2048u, lbo, 1024);
}

// 32 consecutive bf16 (v[i] * s) into row `row` of a 128-byte-row swizzled tile at col0.
__device__ __forceinline__ void store_row_bf16(uint8_t *tile, int row, int col0, const float *v,
                                               float s) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t off = sw128_offset((uint32_t)row, (uint32_t)(col0 + 8 * w) * 2u);
    st_shared_v4(smem_u32(tile + off), pack_bf16x2(v[8 * w + 0] * s, v[8 * w + 1] * s),
                 pack_bf16x2(v[8 * w + 2] * s, v[8 * w + 3] * s),
                 pack_bf16x2(v[8 * w + 4] * s, v[8 * w + 5] * s),
                 pack_bf16x2(v[8 * w + 6] * s, v[8 * w + 7] * s));
  }
}

// 8 consecutive bf16 of row `row` starting at column col0 (multiple of 8).
__device__ __forceinline__ void load_row8_bf16(const uint8_t *tile, int row, int col0, float *f) {
  const uint4 u = *reinterpret_cast<const uint4 *>(
      tile + sw128_offset((uint32_t)row, (uint32_t)col0 * 2u));
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  float a[16], b[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    a[i] = v[i];
    b[i] = v[16 + i];
  }
  tmem_st16(taddr, a);
  tmem_st16(taddr + 16, b);
}

// sum over sequences i < seq of ceil(len_i / C); every thread of the CTA gets the value
__device__ int chunk_base(const int32_t *cu, int seq, int *red) {
  int s = 0;
  for (int i = threadIdx.x; i < seq; i += blockDim.x) s += (cu[i + 1] - cu[i] + C - 1) / C;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  int t = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  __syncthreads();
  return t;
}

// L2-normalise one 128-element bf16 row of a KQ tile in place (TR_NORMALIZE_QK).
__device__ __forceinline__ void normalize_row(uint8_t *kq, int row) {
  float ss = 0.f;
  for (int c0 = 0; c0 < DK; c0 += 8) {
    float f[8];
    load_row8_bf16(kq + (c0 >> 6) * 16384, row, c0 & 63, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
  const float inv = rsqrtf(ss + 1e-6f);
  for (int c0 = 0; c0 < DK; c0 += 8) {
    float f[8];
    uint8_t *h = kq + (c0 >> 6) * 16384;
    load_row8_bf16(h, row, c0 & 63, f);
    const uint32_t off = sw128_offset((uint32_t)row, (uint32_t)(c0 & 63) * 2u);
    st_shared_v4(smem_u32(h + off), pack_bf16x2(f[0] * inv, f[1] * inv),
                 pack_bf16x2(f[2] * inv, f[3] * inv), pack_bf16x2(f[4] * inv, f[5] * inv),
                 pack_bf16x2(f[6] * inv, f[7] * inv));
  }
}

// workspace arrays (slot = (first chunk of the sequence + chunk) * H + head)
struct ScanWs {
  __nv_bfloat16 *A;  // [slots][128][128]  A_c = -K^T diag(gamma') W
  __nv_bfloat16 *R;  // [slots][64][128]   R = diag(gamma) Q - P W
  float *B;          // [slots][128][dv]   B_c = K^T diag(gamma') U~
  float *O;          // [slots][64][dv]    O0 = P U~
  float *G;          // [slots]            gamma_C
  int64_t slots;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int64_t count_slots(const ScanLaunch &p, int *max_chunks) {
  int64_t n = 0;
  int mx = 0;
  for (int i = 0; i < p.n_seqs; ++i) {
    const int c = (p.cu_seqlens_host[i + 1] - p.cu_seqlens_host[i] + C - 1) / C;
    n += c;
    mx = c > mx ? c : mx;
  }
  if (max_chunks) *max_chunks = mx;
  return n * p.H;
}

ScanWs ws_layout(const ScanLaunch &p, void *base, size_t *total) {
  ScanWs w{};
  w.slots = count_slots(p, nullptr);
  const size_t S = (size_t)w.slots;
  size_t off = 0;
  const size_t oA = off; off = align256(off + S * 128 * 128 * 2);
  const size_t oR = off; off = align256(off + S * 64 * 128 * 2);
  const size_t oB = off; off = align256(off + S * 128 * (size_t)p.dv * 4);
  const size_t oO = off; off = align256(off + S * 64 * (size_t)p.dv * 4);
  const size_t oG = off; off = align256(off + S * 4);
  if (total) *total = off;
  uint8_t *b = static_cast<uint8_t *>(base);
  if (b) {
    w.A = reinterpret_cast<__nv_bfloat16 *>(b + oA);
    w.R = reinterpret_cast<__nv_bfloat16 *>(b + oR);
    w.B = reinterpret_cast<float *>(b + oB);
    w.O = reinterpret_cast<float *>(b + oO);
    w.G = reinterpret_cast<float *>(b + oG);
  }
  return w;
}

// ============================================================ prep kernel
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t P_KQ = 0;        // [half][K rows 0-63 | Q rows 64-127]      32 KB
constexpr uint32_t P_V = 32768;     // [64-col block][64 t][128 B]              16 KB
constexpr uint32_t P_AP = 49152;    // 128 x 64: rows 0-63 zero, 64-127 = P     16 KB
constexpr uint32_t P_TS = 65536;    // 128 x 64: rows 0-63 = -T'', 64-127 = T'  16 KB
constexpr uint32_t P_W = 81920;     // [half][64 t][128 B]  W                   16 KB
constexpr uint32_t P_WG = 98304;    // gamma' W                                  16 KB
constexpr uint32_t P_UT = 114688;   // [block][64 t][128 B]  U~                 16 KB
constexpr uint32_t P_UG = 131072;   // gamma' U~                                 16 KB
constexpr uint32_t P_AS = 147456;   // 64 x 65 fp32: A
constexpr int AS_LD = 65;
constexpr uint32_t P_CTL = 164096;
constexpr size_t PREP_SMEM = P_CTL + 1024 + 1024;

struct PrepCtl {
  uint64_t tma_bar;
  uint64_t mma_bar;
  uint32_t tmem;
  int abort;
  float g[C];
  float beta[C];
  int red[4];
};

template <int DV>
__global__ void __launch_bounds__(kThreads, 1)
    scan_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, ScanLaunch p, ScanWs ws) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  PrepCtl *ctl = reinterpret_cast<PrepCtl *>(sm + P_CTL);
  float *As = reinterpret_cast<float *>(sm + P_AS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H;
  const int c = blockIdx.x;
  const int seq = blockIdx.y / H, head = blockIdx.y % H;
  const int t_begin = p.cu_seqlens[seq], t_end = p.cu_seqlens[seq + 1];
  if (c * C >= t_end - t_begin) return;  // uniform: this sequence has fewer chunks
  const int t0 = t_begin + c * C;
  const int nv = min(C, t_end - t0);
  const bool want_o = p.o != nullptr;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int cb = chunk_base(p.cu_seqlens, seq, ctl->red);
  const int64_t slot = ((int64_t)cb + c) * H + head;

  if (tid == 0) {
    mbar_init(smem_u32(&ctl->tma_bar), 1);
    mbar_init(smem_u32(&ctl->mma_bar), 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl->tmem), 512);
    tmem_relinquish();
  }
  for (int i = tid; i < 8192 / 16; i += kThreads) st_shared_v4(smem_u32(sm + P_AP) + 16 * i, 0, 0, 0, 0);
  if (!want_o)
    for (int i = tid; i < 2 * 8192 / 16; i += kThreads)
      st_shared_v4(smem_u32(sm + P_KQ + (i >> 9) * 16384 + 8192) + 16 * (i & 511), 0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const AbortFlag ab{&ctl->abort, p.err_word, ERRBIT_SCAN_TIMEOUT};
  const uint32_t kq_u = smem_u32(sm + P_KQ);

  if (tid == 0) {
    const uint32_t bar = smem_u32(&ctl->tma_bar);
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, 16384u + (want_o ? 16384u : 0u) + (uint32_t)DV * 128u);
    tma_load_2d(kq_u, &tm_k, head * DK, t0, bar);
    tma_load_2d(kq_u + 16384, &tm_k, head * DK + 64, t0, bar);
    if (want_o) {
      tma_load_2d(kq_u + 8192, &tm_q, head * DK, t0, bar);
      tma_load_2d(kq_u + 16384 + 8192, &tm_q, head * DK + 64, t0, bar);
    }
#pragma unroll
    for (int b = 0; b < DV / 64; ++b)
      tma_load_2d(smem_u32(sm + P_V) + 8192 * b, &tm_v, head * DV + 64 * b, t0, bar);
  }
  // gates: g = inclusive cumsum of log alpha over the chunk, beta; 0 past the end
  if (tid < C) {
    float la = 0.f, b = 0.f;
    if (tid < nv) {
      la = p.log_alpha[(size_t)(t0 + tid) * H + head];
      b = p.beta[(size_t)(t0 + tid) * H + head];
    }
    float s = la;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    ctl->g[tid] = s;
    ctl->beta[tid] = b;
  }
  __syncthreads();
  if (tid >= 32 && tid < C) ctl->g[tid] += ctl->g[31];
  const bool ok_tma = mbar_wait(smem_u32(&ctl->tma_bar), 0, ab);
  bool failed = __syncthreads_or(!ok_tma);
  const uint32_t mma_bar = smem_u32(&ctl->mma_bar);
  uint32_t mma_phase = 0;
  auto mma_wait = [&]() -> bool {
    const bool ok = mbar_wait(mma_bar, mma_phase, ab);
    mma_phase ^= 1u;
    if (__syncthreads_or(!ok)) return false;
    tc_fence_after();
    return true;
  };

  do {
    if (failed) break;
    if (p.flags & TR_NORMALIZE_QK) {
      if (tid < C || want_o) normalize_row(sm + P_KQ, tid);
      fence_proxy_async_smem();
      __syncthreads();
    }
    // P1: [K; Q] K^T -> S (cols 0-63)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk)
        tc_mma_bf16(tmem + 0, desc_k(kq_u, kk, 16384), desc_k(kq_u, kk, 16384),
                    idesc_bf16(128, 64, 0, 0), kk > 0);
      tc_commit(mma_bar);
    }
    if (!mma_wait()) { failed = true; break; }

    // A (strictly lower, fp32) from K K^T, P (lower incl. diagonal) from Q K^T
    {
      const int t = tid & 63;
      const float gt = ctl->g[t];
      float v[32];
      if (tid < C) {
        const float bt = ctl->beta[t];
        float *Arow = As + t * AS_LD;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(tmem + lane_base + 32 * hh, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int s = 32 * hh + i;
            Arow[s] = (s < t) ? bt * __expf(gt - ctl->g[s]) * v[i] : 0.f;
          }
        }
      } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(tmem + lane_base + 32 * hh, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int s = 32 * hh + i;
            v[i] = (s <= t) ? __expf(gt - ctl->g[s]) * v[i] : 0.f;
          }
          if (want_o) store_row_bf16(sm + P_AP, 64 + t, 32 * hh, v, 1.f);
        }
      }
    }
    __syncthreads();

    // T = (I + A)^{-1}: thread j builds column j row by row (forward substitution, fp32);
    // four partial sums keep the dependent FMA chains short.
    if (tid < C) {
      const int j = tid;
      float Tc[C];
#pragma unroll
      for (int i = 0; i < C; ++i) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        const float *Ar = As + i * AS_LD;
#pragma unroll
        for (int s = 0; s + 3 < i; s += 4) {
          a0 = fmaf(Ar[s], Tc[s], a0);
          a1 = fmaf(Ar[s + 1], Tc[s + 1], a1);
          a2 = fmaf(Ar[s + 2], Tc[s + 2], a2);
          a3 = fmaf(Ar[s + 3], Tc[s + 3], a3);
        }
#pragma unroll
        for (int s = i & ~3; s < i; ++s) a0 = fmaf(Ar[s], Tc[s], a0);
        const float acc = (a0 + a1) + (a2 + a3);
        Tc[i] = (i == j) ? 1.f : ((i < j) ? 0.f : -acc);
      }
      const float bj = ctl->beta[j];
      const float bgj = bj * __expf(ctl->g[j]);
      __nv_bfloat16 *ts = reinterpret_cast<__nv_bfloat16 *>(sm + P_TS);
#pragma unroll
      for (int i = 0; i < C; ++i) {
        ts[sw128_offset((uint32_t)i, (uint32_t)j * 2u) / 2] = __float2bfloat16_rn(-Tc[i] * bj);
        ts[sw128_offset((uint32_t)(64 + i), (uint32_t)j * 2u) / 2] =
            __float2bfloat16_rn(Tc[i] * bgj);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // P2: [-T''; T'] V -> cols [64, 64+DV) (lanes 0-63: -U~), [-T''; T'] K -> [192, 320) (lanes 64-127: W)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ts_u = smem_u32(sm + P_TS);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 64, desc_k(ts_u, kk, 0), desc_mn(smem_u32(sm + P_V), kk, 8192),
                    idesc_bf16(128, DV, 0, 1), kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 192, desc_k(ts_u, kk, 0), desc_mn(kq_u, kk, 16384),
                    idesc_bf16(128, 128, 0, 1), kk > 0);
      tc_commit(mma_bar);
    }
    if (!mma_wait()) { failed = true; break; }

    const float gC = ctl->g[C - 1];
    {
      float v[32];
      const int t = tid & 63;
      const float gp = __expf(gC - ctl->g[t]);
      if (tid >= C) {  // W row t -> W and gamma' W (natural [t][d] layout, 8 KB halves)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tmem_ld32(tmem + 192 + lane_base + 32 * q, v);
          tc_wait_ld();
          store_row_bf16(sm + P_W + (q >> 1) * 8192, t, 32 * (q & 1), v, 1.f);
          store_row_bf16(sm + P_WG + (q >> 1) * 8192, t, 32 * (q & 1), v, gp);
        }
      } else {  // -U~ row t -> U~ and gamma' U~
#pragma unroll
        for (int q = 0; q < DV / 32; ++q) {
          tmem_ld32(tmem + 64 + lane_base + 32 * q, v);
          tc_wait_ld();
          store_row_bf16(sm + P_UT + (q >> 1) * 8192, t, 32 * (q & 1), v, -1.f);
          store_row_bf16(sm + P_UG + (q >> 1) * 8192, t, 32 * (q & 1), v, -gp);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // one batch: P W -> [0,128), P U~ -> [128, 128+DV), A_c -> [256, 384), B_c -> [384, 384+DV)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ap_u = smem_u32(sm + P_AP), w_u = smem_u32(sm + P_W);
      const uint32_t ut_u = smem_u32(sm + P_UT), wg_u = smem_u32(sm + P_WG);
      const uint32_t ug_u = smem_u32(sm + P_UG);
      if (want_o) {
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(tmem + 0, desc_k(ap_u, kk, 0), desc_mn(w_u, kk, 8192),
                      idesc_bf16(128, 128, 0, 1), kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(tmem + 128, desc_k(ap_u, kk, 0), desc_mn(ut_u, kk, 8192),
                      idesc_bf16(128, DV, 0, 1), kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 256, desc_mn(kq_u, kk, 16384), desc_mn(wg_u, kk, 8192),
                    idesc_bf16(128, 128, 1, 1), kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 384, desc_mn(kq_u, kk, 16384), desc_mn(ug_u, kk, 8192),
                    idesc_bf16(128, DV, 1, 1), kk > 0);
      tc_commit(mma_bar);
    }
    if (!mma_wait()) { failed = true; break; }

    {
      float v[32];
      // A_c row d = -(K^T gamma' W)[d][:] (bf16), B_c row d (fp32): all 128 lanes
      const int d = tid;
      __nv_bfloat16 *Ad = ws.A + (size_t)slot * 128 * 128 + (size_t)d * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        tmem_ld32(tmem + 256 + lane_base + 32 * q, v);
        tc_wait_ld();
        uint4 *dst = reinterpret_cast<uint4 *>(Ad + 32 * q);
#pragma unroll
        for (int w = 0; w < 4; ++w)
          dst[w] = make_uint4(pack_bf16x2(-v[8 * w], -v[8 * w + 1]),
                              pack_bf16x2(-v[8 * w + 2], -v[8 * w + 3]),
                              pack_bf16x2(-v[8 * w + 4], -v[8 * w + 5]),
                              pack_bf16x2(-v[8 * w + 6], -v[8 * w + 7]));
      }
      float *Bd = ws.B + (size_t)slot * 128 * DV + (size_t)d * DV;
#pragma unroll
      for (int q = 0; q < DV / 32; ++q) {
        tmem_ld32(tmem + 384 + lane_base + 32 * q, v);
        tc_wait_ld();
        float4 *dst = reinterpret_cast<float4 *>(Bd + 32 * q);
#pragma unroll
        for (int w = 0; w < 8; ++w)
          dst[w] = make_float4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]);
      }
      if (want_o && tid >= C) {
        // R row t = gamma_t q_t - (P W)_t (bf16), O0 row t (fp32)
        const int t = tid - C;
        const float gam = __expf(ctl->g[t]);
        __nv_bfloat16 *Rt = ws.R + (size_t)slot * 64 * 128 + (size_t)t * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tmem_ld32(tmem + 0 + lane_base + 32 * q, v);
          tc_wait_ld();
          uint4 *dst = reinterpret_cast<uint4 *>(Rt + 32 * q);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            float f[8];
            load_row8_bf16(sm + P_KQ + (q >> 1) * 16384, 64 + t, 32 * (q & 1) + 8 * w, f);
            dst[w] = make_uint4(pack_bf16x2(gam * f[0] - v[8 * w], gam * f[1] - v[8 * w + 1]),
                                pack_bf16x2(gam * f[2] - v[8 * w + 2], gam * f[3] - v[8 * w + 3]),
                                pack_bf16x2(gam * f[4] - v[8 * w + 4], gam * f[5] - v[8 * w + 5]),
                                pack_bf16x2(gam * f[6] - v[8 * w + 6], gam * f[7] - v[8 * w + 7]));
          }
        }
        float *Ot = ws.O + (size_t)slot * 64 * DV + (size_t)t * DV;
#pragma unroll
        for (int q = 0; q < DV / 32; ++q) {
          tmem_ld32(tmem + 128 + lane_base + 32 * q, v);
          tc_wait_ld();
          float4 *dst = reinterpret_cast<float4 *>(Ot + 32 * q);
#pragma unroll
          for (int w = 0; w < 8; ++w)
            dst[w] = make_float4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]);
        }
      }
      if (tid == 0) ws.G[slot] = __expf(gC);
    }
  } while (false);

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =========================================================== chain kernel
constexpr uint32_t H_A = 0;          // 2 x 32 KB  A_c  [half][128 rows][128 B]
constexpr uint32_t H_R = 65536;      // 2 x 16 KB  R    [half][64 rows][128 B] (MMA rows 64-127 unused)
constexpr uint32_t H_B = 98304;      // 2 x 32 KB  B_c slice, fp32 [box][128 rows][32 floats]
constexpr uint32_t H_O = 163840;     // 2 x 16 KB  O0 slice,  fp32 [box][64 rows][32 floats]
constexpr uint32_t H_MB = 196608;    // 16 KB      bf16 state slice [d][64]
constexpr uint32_t H_CTL = 212992;
constexpr size_t CHAIN_SMEM = H_CTL + 1024 + 1024;

struct ChainCtl {
  uint64_t tma_bar[2];
  uint64_t mma_bar;
  uint32_t tmem;
  int abort;
  int red[4];
};

__device__ __forceinline__ void load_row32_f32(const uint8_t *tile, int row, float *f) {
  // one row (32 floats = 128 B) of a 128-byte-swizzled fp32 tile
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const float4 u = *reinterpret_cast<const float4 *>(
        tile + sw128_offset((uint32_t)row, (uint32_t)ch * 16u));
    f[4 * ch] = u.x; f[4 * ch + 1] = u.y; f[4 * ch + 2] = u.z; f[4 * ch + 3] = u.w;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    scan_chain_kernel(const __grid_constant__ CUtensorMap tm_A, const __grid_constant__ CUtensorMap tm_R,
                      const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_O,
                      ScanLaunch p, ScanWs ws) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  ChainCtl *ctl = reinterpret_cast<ChainCtl *>(sm + H_CTL);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int H = p.H;
  const int seq = blockIdx.x / H, head = blockIdx.x % H;
  const int slice = blockIdx.y;
  const int t_begin = p.cu_seqlens[seq], t_end = p.cu_seqlens[seq + 1];
  const int nch = (t_end - t_begin + C - 1) / C;
  const bool want_o = p.o != nullptr;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int cb = chunk_base(p.cu_seqlens, seq, ctl->red);

  if (tid == 0) {
    mbar_init(smem_u32(&ctl->tma_bar[0]), 1);
    mbar_init(smem_u32(&ctl->tma_bar[1]), 1);
    mbar_init(smem_u32(&ctl->mma_bar), 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl->tmem), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;  // Z: cols [0, 64), O: [64, 128)
  const AbortFlag ab{&ctl->abort, p.err_word, ERRBIT_SCAN_TIMEOUT};

  float Mr[DVS];
  bool m_zero = p.S0 == nullptr;
  const size_t s_base = ((size_t)seq * H + head) * DK * p.dv + (size_t)tid * p.dv + (size_t)slice * DVS;
  if (!m_zero) {
#pragma unroll
    for (int j = 0; j < DVS; j += 4) {
      const float4 a = *reinterpret_cast<const float4 *>(p.S0 + s_base + j);
      Mr[j] = a.x; Mr[j + 1] = a.y; Mr[j + 2] = a.z; Mr[j + 3] = a.w;
    }
    store_row_bf16(sm + H_MB, tid, 0, Mr, 1.f);
    store_row_bf16(sm + H_MB, tid, 32, Mr + 32, 1.f);
  } else {
#pragma unroll
    for (int j = 0; j < DVS; ++j) Mr[j] = 0.f;
  }

  const uint32_t tx = 32768u + 32768u + (want_o ? 16384u + 16384u : 0u);
  auto issue = [&](int c, int buf) {
    const int64_t slot = ((int64_t)cb + c) * H + head;
    const uint32_t bar = smem_u32(&ctl->tma_bar[buf]);
    mbar_arrive_expect_tx(bar, tx);
    const uint32_t a_u = smem_u32(sm + H_A + buf * 32768);
    tma_load_2d(a_u, &tm_A, 0, (int32_t)(slot * 128), bar);
    tma_load_2d(a_u + 16384, &tm_A, 64, (int32_t)(slot * 128), bar);
    const uint32_t b_u = smem_u32(sm + H_B + buf * 32768);
    tma_load_2d(b_u, &tm_B, slice * DVS, (int32_t)(slot * 128), bar);
    tma_load_2d(b_u + 16384, &tm_B, slice * DVS + 32, (int32_t)(slot * 128), bar);
    if (want_o) {
      const uint32_t r_u = smem_u32(sm + H_R + buf * 16384);
      tma_load_2d(r_u, &tm_R, 0, (int32_t)(slot * 64), bar);
      tma_load_2d(r_u + 8192, &tm_R, 64, (int32_t)(slot * 64), bar);
      const uint32_t o_u = smem_u32(sm + H_O + buf * 16384);
      tma_load_2d(o_u, &tm_O, slice * DVS, (int32_t)(slot * 64), bar);
      tma_load_2d(o_u + 8192, &tm_O, slice * DVS + 32, (int32_t)(slot * 64), bar);
    }
  };
  if (tid == 0) {
    fence_proxy_async_smem();
    if (nch > 0) issue(0, 0);
    if (nch > 1) issue(1, 1);
  }
  const uint32_t mma_bar = smem_u32(&ctl->mma_bar);
  uint32_t mma_phase = 0;
  bool failed = false;

  for (int c = 0; c < nch; ++c) {
    const int buf = c & 1;
    const int t0 = t_begin + c * C;
    const int64_t slot = ((int64_t)cb + c) * H + head;
    const float gC = ws.G[slot];
    const bool ok_tma = mbar_wait(smem_u32(&ctl->tma_bar[buf]), (uint32_t)(c >> 1) & 1u, ab);
    if (__syncthreads_or(!ok_tma)) { failed = true; break; }
    if (!m_zero) {
      if (tid == 0) {
        tc_fence_after();
        const uint32_t a_u = smem_u32(sm + H_A + buf * 32768);
        const uint32_t r_u = smem_u32(sm + H_R + buf * 16384);
        const uint32_t mb_u = smem_u32(sm + H_MB);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          tc_mma_bf16(tmem + 0, desc_k(a_u, kk, 16384), desc_mn(mb_u, kk, 8192),
                      idesc_bf16(128, DVS, 0, 1), kk > 0);
        if (want_o) {
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            tc_mma_bf16(tmem + 64, desc_k(r_u, kk, 8192), desc_mn(mb_u, kk, 8192),
                        idesc_bf16(128, DVS, 0, 1), kk > 0);
        }
        tc_commit(mma_bar);
      }
      const bool ok = mbar_wait(mma_bar, mma_phase, ab);
      mma_phase ^= 1u;
      if (__syncthreads_or(!ok)) { failed = true; break; }
      tc_fence_after();
    }
    // M <- gamma_C M + Z + B_c ; o = O + O0
    {
      const uint8_t *bt = sm + H_B + buf * 32768;
      float v[32], b[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (!m_zero) {
          tmem_ld32(tmem + 0 + lane_base + 32 * hh, v);
          tc_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        load_row32_f32(bt + hh * 16384, tid, b);
#pragma unroll
        for (int i = 0; i < 32; ++i) Mr[32 * hh + i] = fmaf(gC, Mr[32 * hh + i], v[i] + b[i]);
      }
      if (want_o && tid < C) {
        const int t = tid;
        const uint8_t *ot = sm + H_O + buf * 16384;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (!m_zero) {
            tmem_ld32(tmem + 64 + lane_base + 32 * hh, v);
            tc_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
          load_row32_f32(ot + hh * 8192, t, b);
          if (t0 + t < t_end) {
            uint4 *d4 = reinterpret_cast<uint4 *>(
                reinterpret_cast<__nv_bfloat16 *>(p.o) + (size_t)(t0 + t) * p.o_stride +
                (size_t)head * p.dv + slice * DVS + 32 * hh);
            const float sc = p.scale;
#pragma unroll
            for (int w = 0; w < 4; ++w)
              d4[w] = make_uint4(pack_bf16x2((v[8 * w] + b[8 * w]) * sc, (v[8 * w + 1] + b[8 * w + 1]) * sc),
                                 pack_bf16x2((v[8 * w + 2] + b[8 * w + 2]) * sc, (v[8 * w + 3] + b[8 * w + 3]) * sc),
                                 pack_bf16x2((v[8 * w + 4] + b[8 * w + 4]) * sc, (v[8 * w + 5] + b[8 * w + 5]) * sc),
                                 pack_bf16x2((v[8 * w + 6] + b[8 * w + 6]) * sc, (v[8 * w + 7] + b[8 * w + 7]) * sc));
          }
        }
      }
      store_row_bf16(sm + H_MB, tid, 0, Mr, 1.f);
      store_row_bf16(sm + H_MB, tid, 32, Mr + 32, 1.f);
      m_zero = false;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && c + 2 < nch) {
      fence_proxy_async_smem();
      issue(c + 2, buf);
    }
  }

  if (!failed) {
    float *dst = p.S_final + s_base;
#pragma unroll
    for (int j = 0; j < DVS; j += 4)
      *reinterpret_cast<float4 *>(dst + j) = make_float4(Mr[j], Mr[j + 1], Mr[j + 2], Mr[j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

bool make_tmap_f32_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                      std::string *err);

bool scan_chunked_supported(const ScanLaunch &p) {
  return p.dtype == TR_DTYPE_BF16 && p.dk == DK && (p.dv == 64 || p.dv == 128) &&
         (p.o == nullptr || p.o_stride % 8 == 0);
}

size_t scan_chunked_workspace(const ScanLaunch &p) {
  size_t total = 0;
  ws_layout(p, nullptr, &total);
  return total;
}

int scan_chunked_kernels() { return 2; }

cudaError_t launch_scan_chunked(const ScanLaunch &p, cudaStream_t s, std::string *err,
                                const std::function<cudaError_t()> &between) {
  if (p.n_seqs == 0) return cudaSuccess;
  size_t total = 0;
  ScanWs ws = ws_layout(p, p.ws, &total);
  if (total > p.ws_bytes || (total > 0 && !p.ws)) {
    if (err) *err = "scan workspace too small";
    return cudaErrorInvalidValue;
  }
  int max_chunks = 0;
  count_slots(p, &max_chunks);
  const uint64_t T = (uint64_t)(p.T > 0 ? p.T : 1);
  const uint64_t slots = (uint64_t)(ws.slots > 0 ? ws.slots : 1);
  CUtensorMap tq, tk, tv, tA, tR, tB, tO;
  const void *qb = p.q ? p.q : p.k;
  if (!make_tmap_bf16_2d(&tk, p.k, (uint64_t)p.H * DK, T, (uint64_t)p.k_stride * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&tq, qb, (uint64_t)p.H * DK, T,
                         (uint64_t)(p.q ? p.q_stride : p.k_stride) * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&tv, p.v, (uint64_t)p.H * p.dv, T, (uint64_t)p.v_stride * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&tA, ws.A, 128, slots * 128, 256, 64, 128, err) ||
      !make_tmap_bf16_2d(&tR, ws.R, 128, slots * 64, 256, 64, 64, err) ||
      !make_tmap_f32_2d(&tB, ws.B, (uint64_t)p.dv, slots * 128, (uint64_t)p.dv * 4, 32, 128, err) ||
      !make_tmap_f32_2d(&tO, ws.O, (uint64_t)p.dv, slots * 64, (uint64_t)p.dv * 4, 32, 64, err))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (max_chunks > 0) {
    dim3 pg((unsigned)max_chunks, (unsigned)(p.n_seqs * p.H));
    if (p.dv == 128) {
      e = cudaFuncSetAttribute(scan_prep_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)PREP_SMEM);
      if (e != cudaSuccess) return e;
      scan_prep_kernel<128><<<pg, kThreads, PREP_SMEM, s>>>(tq, tk, tv, p, ws);
    } else {
      e = cudaFuncSetAttribute(scan_prep_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)PREP_SMEM);
      if (e != cudaSuccess) return e;
      scan_prep_kernel<64><<<pg, kThreads, PREP_SMEM, s>>>(tq, tk, tv, p, ws);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (between) {
    e = between();
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(scan_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)CHAIN_SMEM);
  if (e != cudaSuccess) return e;
  dim3 cg((unsigned)(p.n_seqs * p.H), (unsigned)(p.dv / DVS));
  scan_chain_kernel<<<cg, kThreads, CHAIN_SMEM, s>>>(tA, tR, tB, tO, p, ws);
  return cudaGetLastError();
}

}  // namespace tr
