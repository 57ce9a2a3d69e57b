// scan_chunked.cu -- chunked Gated DeltaNet scan on the 5th-generation tensor cores.
//
// Eq. (1) (Tail-Replay reading notes, section 2.3) in the M = S^T layout,
//   M_t = alpha_t (M_{t-1} - beta_t k_t (k_t^T M_{t-1})) + beta_t k_t v_t^T,
// regrouped over chunks of C = 64 tokens (the WY / UT form of the delta rule, derived
// here from Eq. (1)).  Inside chunk c, with g_t = sum_{s<=t} log alpha_s, gamma_t = e^{g_t},
// gamma'_t = e^{g_C - g_t}, gamma_C = e^{g_C} and the state M_c at the chunk start:
//   A_ts = beta_t e^{g_t - g_s} k_t.k_s (s < t),  T = (I + A)^{-1}
//   W = T diag(beta gamma) K,  U~ = T diag(beta) V,  U_c = U~ - W M_c
//   P_ts = e^{g_t - g_s} q_t.k_s (s <= t)
//   output   O_c = diag(gamma) Q M_c + P U_c
//   state    M_{c+1} = gamma_C M_c + K^T diag(gamma') U_c
// Substituting M_{c+1} into U_{c+1} gives the look-ahead form the chain uses:
//   U_{c+1} = U~_{c+1} - gamma_C W_{c+1} M_c - Y_{c+1} U_c,   Y_{c+1} = W_{c+1} (diag(gamma'_c) K_c)^T
// so U_{c+1} needs M_c and U_c (not M_{c+1}): per chunk, one product of M_c and one of U_c
// give both the chunk's output and the next chunk's U, and the state update runs beside
// them.  Everything that does not depend on the state is computed first, for all chunks in
// parallel:
//
//   scan_prep_kernel   persistent over all (chunk, head) items (256 threads):
//     [Q; K] [K; K_prev]^T -> TMEM (tcgen05): P, A and Z = K_c (diag(gamma'_{c-1}) K_{c-1})^T
//     T = (I + A)^{-1} on CUDA cores (blocked forward substitution, fp32)
//     [T'; T''] [K | V | Z] -> W, U~, Y (T' = T diag(beta gamma), T'' = T diag(beta); T as a
//        bf16 hi + lo pair for U~)
//     -> workspace, by TMA stores: gamma Q, -gamma_C(prev) W, P, -Y, K (bf16), U~ (fp32),
//        gamma' and gamma_C
//   scan_chain_kernel  one CTA per (sequence, head, 64-column slice of d_v), sequential over
//     the sequence's chunks, longest sequences first:
//       D = [gamma Q_c; -gamma_C W_{c+1}] M_c + [P_c; -Y_{c+1}] U_c   (rows 0-63: O_c,
//                                                   rows 64-127: U_{c+1} - U~_{c+1})
//       dM = K_c^T (gamma' U_c),  M_{c+1} = gamma_C M_c + dM  (fp32 registers; gamma' U_c
//       as a bf16 hi + lo pair, so the state's update keeps fp32-level accuracy)
//     warp-specialised: a TMA producer, an MMA issuer, four state warps, four output warps.
//   scan_plan_kernel   (only for more than kParamSeqs sequences) chunk offsets per sequence
//     and the longest-first order; fewer sequences get both from the host in the launch.
//
// Every M-dependent product acts column by column on d_v, so d_v splits into exact
// 64-column slices.  Tokens past the end of a sequence get beta = 0 and log alpha = 0: their
// rows of T are the identity, their W, U~ and Y rows vanish, and so do their U rows.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <numeric>

#include "../../include/tr.h"
#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

constexpr int C = 64;      // chunk length
constexpr int DK = 128;    // key dimension handled here
constexpr int DVS = 64;    // d_v columns per chain CTA
constexpr int kParamSeqs = 64;   // up to this many sequences, the plan travels in the launch

// --------------------------------------------------------------- helpers
// Shared-memory descriptors are built once per operand (sw128_desc) and advanced per K
// step by adding to the 16-byte start-address field only.
//   K-major operand: 128-byte rows, 64-column halves `half_stride` bytes apart; K step kk
//   (16 elements) starts 32 bytes further inside the 128-byte swizzle atom.
//   MN-major operand: rows are the K dimension, 128-byte rows hold 64 M/N elements
//   (64-element blocks LBO bytes apart); K step kk = 16 rows = 2048 bytes.
__device__ __forceinline__ uint64_t kmaj(uint32_t base) { return sw128_desc(base, 16, 1024); }
__device__ __forceinline__ uint64_t mnmaj(uint32_t base, uint32_t lbo) {
  return sw128_desc(base, lbo, 1024);
}
__device__ __forceinline__ uint64_t desc_k(uint64_t d0, int kk, uint32_t half_stride) {
  return d0 + (((uint32_t)(kk >> 2) * half_stride + (uint32_t)(kk & 3) * 32u) >> 4);
}
__device__ __forceinline__ uint64_t desc_mn(uint64_t d0, int kk) {
  return d0 + (uint64_t)kk * 128u;
}

// Packed fp32 pairs (sm_100a f32x2 arithmetic): one instruction for two lanes, each lane
// rounded exactly as the scalar operation would be.
__device__ __forceinline__ uint64_t f32x2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t r, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
// (a0, a1) += (b0, b1)
__device__ __forceinline__ void add_f32x2(float &a0, float &a1, float b0, float b1) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f32x2_pack(a0, a1)), "l"(f32x2_pack(b0, b1)));
  f32x2_unpack(r, a0, a1);
}
// (d0, d1) = (a0, a1) - (b0, b1)
__device__ __forceinline__ void sub_f32x2(float &d0, float &d1, float a0, float a1, float b0,
                                          float b1) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f32x2_pack(a0, a1)), "l"(f32x2_pack(b0, b1)));
  f32x2_unpack(r, d0, d1);
}
// (d0, d1) = s (a0, a1)
__device__ __forceinline__ void mul_f32x2(float &d0, float &d1, float a0, float a1, float s) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f32x2_pack(a0, a1)), "l"(f32x2_pack(s, s)));
  f32x2_unpack(r, d0, d1);
}
// (m0, m1) = g (m0, m1) + (c0, c1), fused
__device__ __forceinline__ void fma_f32x2(float &m0, float &m1, float g, float c0, float c1) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(r)
      : "l"(f32x2_pack(g, g)), "l"(f32x2_pack(m0, m1)), "l"(f32x2_pack(c0, c1)));
  f32x2_unpack(r, m0, m1);
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

// 32 fp32 values (v[i] * s) as row `row` (128 bytes) of a 128-byte-row swizzled tile.
__device__ __forceinline__ void store_row32_f32(uint8_t *tile, int row, const float *v, float s) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    st_shared_v4(smem_u32(tile + sw128_offset((uint32_t)row, (uint32_t)ch * 16u)),
                 __float_as_uint(v[4 * ch] * s), __float_as_uint(v[4 * ch + 1] * s),
                 __float_as_uint(v[4 * ch + 2] * s), __float_as_uint(v[4 * ch + 3] * s));
}

// One row (32 floats = 128 B) of a 128-byte-swizzled fp32 tile.
__device__ __forceinline__ void load_row32_f32(const uint8_t *tile, int row, float *f) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const float4 u = *reinterpret_cast<const float4 *>(
        tile + sw128_offset((uint32_t)row, (uint32_t)ch * 16u));
    f[4 * ch] = u.x; f[4 * ch + 1] = u.y; f[4 * ch + 2] = u.z; f[4 * ch + 3] = u.w;
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

// hi + lo bf16 split of 32 values (v[i] * s; v[i] itself without kScale) into two
// 128-byte-row swizzled tiles.
template <bool kScale = true>
__device__ __forceinline__ void store_row_split(uint8_t *hi, uint8_t *lo, int row, int col0,
                                                const float *v, float s) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a = v[8 * w + 2 * i], b = v[8 * w + 2 * i + 1], ra, rb;
      if (kScale) mul_f32x2(a, b, a, b, s);
      const __nv_bfloat162 hh = __floats2bfloat162_rn(a, b);
      const float2 hf = __bfloat1622float2(hh);
      sub_f32x2(ra, rb, a, b, hf.x, hf.y);
      const __nv_bfloat162 ll = __floats2bfloat162_rn(ra, rb);
      h[i] = *reinterpret_cast<const uint32_t *>(&hh);
      l[i] = *reinterpret_cast<const uint32_t *>(&ll);
    }
    const uint32_t off = sw128_offset((uint32_t)row, (uint32_t)(col0 + 8 * w) * 2u);
    st_shared_v4(smem_u32(hi + off), h[0], h[1], h[2], h[3]);
    st_shared_v4(smem_u32(lo + off), l[0], l[1], l[2], l[3]);
  }
}

// Scale 32 bf16 of row `row`, columns col0..col0+31, of a swizzled tile in place.
__device__ __forceinline__ void scale_row32_bf16(uint8_t *tile, int row, int col0, float s) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float f[8];
    load_row8_bf16(tile, row, col0 + 8 * w, f);
    const uint32_t off = sw128_offset((uint32_t)row, (uint32_t)(col0 + 8 * w) * 2u);
    st_shared_v4(smem_u32(tile + off), pack_bf16x2(f[0] * s, f[1] * s),
                 pack_bf16x2(f[2] * s, f[3] * s), pack_bf16x2(f[4] * s, f[5] * s),
                 pack_bf16x2(f[6] * s, f[7] * s));
  }
}

// ------------------------------------------------------------------ plan
// cu_chunks[i] = sum_{j < i} ceil(len_j / C) (i = 0..n), and the sequences ordered by
// chunk count, longest first (ties by index).
struct ScanPlan {
  int32_t cu_chunks[kParamSeqs + 1];
  int32_t cu_tokens[kParamSeqs + 1];   // the sequences' token offsets (cu_seqlens)
  int32_t order[kParamSeqs];
  int in_params;     // 1: the arrays above hold the plan; 0: it is in the workspace
};

// workspace arrays (slot = (cu_chunks[seq] + chunk) * H + head)
struct ScanWs {
  __nv_bfloat16 *QW;  // [slots][128][128]: rows 0-63 gamma Q, rows 64-127 -gamma_C(prev) W
  __nv_bfloat16 *PY;  // [slots][128][64]:  rows 0-63 P, rows 64-127 -Y
  __nv_bfloat16 *KT;  // [slots][64][128]:  K (L2-normalised in place with TR_NORMALIZE_QK)
  float *UT;          // [slots][64][dv]:   U~
  float *GP;          // [slots][64]:       gamma'
  float *G;           // [slots][4]:        gamma_C (16 bytes per slot, for one bulk copy)
  int32_t *cu_chunks; // [n_seqs + 1]       (plan kernel output; unused with a launch plan)
  int32_t *order;     // [n_seqs]
  unsigned long long *flags;  // [slots]: the call's epoch once the slot is stored (fused launch)
  int64_t slots;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int64_t count_chunks(const ScanLaunch &p) {
  int64_t n = 0;
  for (int i = 0; i < p.n_seqs; ++i)
    n += (p.cu_seqlens_host[i + 1] - p.cu_seqlens_host[i] + C - 1) / C;
  return n;
}

ScanWs ws_layout(const ScanLaunch &p, void *base, size_t *total) {
  ScanWs w{};
  w.slots = count_chunks(p) * p.H;
  const size_t S = (size_t)w.slots;
  size_t off = 0;
  const size_t oQW = off; off = align256(off + S * 128 * 128 * 2);
  const size_t oPY = off; off = align256(off + S * 128 * 64 * 2);
  // K~ is kept only when the scan normalises k itself; otherwise the chain reads k
  const bool keep_kt = (p.flags & TR_NORMALIZE_QK) != 0;
  const size_t oKT = off; off = align256(off + (keep_kt ? S * 64 * 128 * 2 : 0));
  const size_t oUT = off; off = align256(off + S * 64 * (size_t)p.dv * 4);
  const size_t oGP = off; off = align256(off + S * 64 * 4);
  const size_t oG = off;  off = align256(off + S * 16);
  const size_t oCU = off; off = align256(off + (size_t)(p.n_seqs + 1) * 4);
  const size_t oOR = off; off = align256(off + (size_t)(p.n_seqs + 1) * 4);
  const size_t oFL = off; off = align256(off + S * 8);
  if (total) *total = off;
  uint8_t *b = static_cast<uint8_t *>(base);
  if (b) {
    w.QW = reinterpret_cast<__nv_bfloat16 *>(b + oQW);
    w.PY = reinterpret_cast<__nv_bfloat16 *>(b + oPY);
    w.KT = reinterpret_cast<__nv_bfloat16 *>(b + oKT);
    w.UT = reinterpret_cast<float *>(b + oUT);
    w.GP = reinterpret_cast<float *>(b + oGP);
    w.G = reinterpret_cast<float *>(b + oG);
    w.cu_chunks = reinterpret_cast<int32_t *>(b + oCU);
    w.order = reinterpret_cast<int32_t *>(b + oOR);
    w.flags = reinterpret_cast<unsigned long long *>(b + oFL);
  }
  return w;
}

constexpr int kPlanThreads = 1024;
constexpr int kSortMax = 4096;   // longest-first order for up to this many sequences

// One block: chunk offsets by a block-wide scan, then the longest-first order by a bitonic
// sort of (chunk count, index) keys in shared memory (the identity order beyond kSortMax).
__global__ void __launch_bounds__(kPlanThreads)
    scan_plan_kernel(const int32_t *cu_seqlens, int n_seqs, int32_t *cu_chunks, int32_t *order) {
  __shared__ unsigned long long keys[kSortMax];
  __shared__ int warp_sum[kPlanThreads / 32];
  __shared__ int carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();
  pdl_wait();
  if (tid == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < n_seqs; base += kPlanThreads) {
    const int i = base + tid;
    const int nch = i < n_seqs ? (cu_seqlens[i + 1] - cu_seqlens[i] + C - 1) / C : 0;
    int x = nch;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sum[lane] = w;   // inclusive over warps
    }
    __syncthreads();
    const int carry = carry_s;
    const int excl = carry + (warp > 0 ? warp_sum[warp - 1] : 0) + x - nch;
    if (i < n_seqs) {
      cu_chunks[i] = excl;
      if (n_seqs <= kSortMax)
        keys[i] = ((unsigned long long)(0x7fffffff - nch) << 32) | (unsigned)i;
    }
    __syncthreads();
    if (tid == 0) carry_s = carry + warp_sum[kPlanThreads / 32 - 1];
    __syncthreads();
  }
  if (tid == 0) cu_chunks[n_seqs] = carry_s;
  if (n_seqs > kSortMax) {
    for (int i = tid; i < n_seqs; i += kPlanThreads) order[i] = i;
    return;
  }
  int n2 = 1;
  while (n2 < n_seqs) n2 <<= 1;
  for (int i = n_seqs + tid; i < n2; i += kPlanThreads) keys[i] = ~0ull;
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n2; i += kPlanThreads) {
        const int l = i ^ j;
        if (l > i) {
          const unsigned long long a = keys[i], b = keys[l];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            keys[i] = b;
            keys[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < n_seqs; i += kPlanThreads) order[i] = (int32_t)(keys[i] & 0xffffffffu);
}

__device__ __forceinline__ const int32_t *plan_cu_chunks(const ScanPlan &pl, const ScanWs &ws) {
  return pl.in_params ? pl.cu_chunks : ws.cu_chunks;
}
__device__ __forceinline__ const int32_t *plan_order(const ScanPlan &pl, const ScanWs &ws) {
  return pl.in_params ? pl.order : ws.order;
}
__device__ __forceinline__ const int32_t *plan_cu_tokens(const ScanPlan &pl, const ScanLaunch &p) {
  return pl.in_params ? pl.cu_tokens : p.cu_seqlens;
}

// ============================================================ prep kernel
// 256 threads, persistent over work items (item = chunk_global * H + head, CTA b takes
// items b, b + grid, ...); the next item's tiles are prefetched by TMA into the other
// input stage.  Shared memory (bytes from a 1024-aligned base):
//   stage s (64 KB at s * 64 KB): half h (d_k columns 64h..64h+63) at + 32 KB h, bands of
//   64 rows x 128 B at + 8 KB b: b = 0 Q, 1 K, 2 K of the previous chunk, 3 V (d_v
//   columns 64h..).  After the item's products the Q band holds gamma Q and the
//   previous-K band -gamma_C(prev) W: they are stored from there, with the K band.
constexpr uint32_t P_STAGE = 65536;
constexpr uint32_t P_AF = 131072;         // A fp32 [64][68]
constexpr uint32_t P_TF = P_AF + 17408;   // T fp32 [64][68], then X fp32 [32][36]
constexpr uint32_t P_THI = 171008;        // [T'; T''] high bf16 parts [128][64] (then U~ staging)
constexpr uint32_t P_TLO = P_THI + 16384; // low parts
constexpr uint32_t P_P = P_TLO + 16384;   // P bf16 [64][64]
constexpr uint32_t P_Z = P_P + 8192;      // Z bf16 [64][64] (then -Y staging)
constexpr uint32_t P_END = P_Z + 8192;
constexpr int LDA = 68;                   // fp32 row stride of A and T (16-byte aligned rows)
constexpr int LDX = 36;
constexpr size_t PREP_SMEM = P_END + 1024;
constexpr int kPrepThreads = 256;
static_assert(P_TF + 17408 + 4608 <= P_THI, "prep shared-memory layout");
static_assert(P_THI % 1024 == 0 && P_P % 1024 == 0 && P_Z % 1024 == 0,
              "swizzled tiles are 1024-byte aligned");
static_assert(PREP_SMEM <= 232448, "prep shared memory");

struct PrepItem {
  int seq, c, head, t0, nv, has_prev;
  int64_t slot;
};

struct PrepCtl {
  uint64_t tma_bar[2];
  uint64_t mma_bar;     // group 1, then the first part of group 2 (thread 0, thread 64)
  uint64_t mma_bar2;    // the second part of group 2 (thread 64)
  uint64_t drain_bar, drain_bar2;
  uint32_t tmem;
  int abort;
  PrepItem cur, nxt;
  float g[C];      // inclusive cumsum of log alpha over the chunk
  __align__(16) float beta[C];
  __align__(16) float bg[C];     // beta * gamma
  float gp[C];     // gamma' = e^{g_C - g_t}
  __align__(16) float gpp[C];    // the previous chunk's gamma'
  float gq[C];     // gamma
  __align__(16) float igq[C];   // 1 / gamma (when the chunk's decay allows it: see p1)
  float gpv[C];    // the previous chunk's cumsum
  float gc_prev;   // the previous chunk's gamma_C (1 without one)
};

// The item's location given its sequence (cu_chunks[seq] <= chunk < cu_chunks[seq + 1]).
__device__ __forceinline__ PrepItem item_at(int64_t item, int seq, const ScanLaunch &p,
                                            const int32_t *cu_chunks, const int32_t *cu_tokens) {
  PrepItem it;
  const int chunk = (int)(item / p.H);
  it.seq = seq;
  it.c = chunk - cu_chunks[seq];
  it.head = (int)(item % p.H);
  it.t0 = cu_tokens[seq] + it.c * C;
  it.nv = min(C, cu_tokens[seq + 1] - it.t0);
  it.has_prev = it.c > 0;
  it.slot = item;
  return it;
}
// First item of a CTA: binary search for the last sequence whose first chunk is <= chunk
// and that owns chunks (sequences without tokens own none).
__device__ int seq_of_chunk(int chunk, int n_seqs, const int32_t *cu_chunks) {
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu_chunks[mid] <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}
// Later items: chunks only grow, so the sequence index only moves forward.
__device__ __forceinline__ int advance_seq(int seq, int chunk, const int32_t *cu_chunks) {
  while (cu_chunks[seq + 1] <= chunk) ++seq;
  return seq;
}

// L2-normalise one 128-element bf16 row of band `band` (row r) in place (TR_NORMALIZE_QK).
__device__ __forceinline__ void normalize_band_row(uint8_t *stage, int band, int r) {
  float ss = 0.f;
  for (int c0 = 0; c0 < DK; c0 += 8) {
    float f[8];
    load_row8_bf16(stage + (c0 >> 6) * 32768 + band * 8192, r, c0 & 63, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
  const float inv = rsqrtf(ss + 1e-6f);
  for (int c0 = 0; c0 < DK; c0 += 32)
    scale_row32_bf16(stage + (c0 >> 6) * 32768 + band * 8192, r, c0 & 63, inv);
}

// The maps both kernels' bodies read (prep: q, k, v in; workspace out; chain: workspace in,
// o out).
struct ScanMaps {
  CUtensorMap q, k, v, QW, PY, KT, UT, o;
};

// Publish item `slot` as complete for the chain running beside the prep (fused launch):
// its output stores have completed; the release store orders them before the flag.
__device__ __forceinline__ void publish_slot(const ScanWs &ws, int64_t slot, unsigned long long epoch) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(ws.flags + slot), "l"(epoch) : "memory");
}

// The items one prep CTA takes, in increasing order: first the shared rounds (items below
// shared_end, every `all` CTAs one each: item = cta, cta + all, ...), then, unless the CTA
// only helps in those rounds, the rest in its own stride (shared_end + own_first, + own_stride
// ...).  Without shared rounds this is one strided walk.
struct PrepSched {
  int64_t shared_end;   // items in the shared rounds (0: none)
  int cta, all;         // this CTA's place among the shared rounds' CTAs
  int64_t own_first;    // first item after the shared rounds, relative to shared_end (-1: none)
  int own_stride;
  __device__ __forceinline__ int64_t first(int64_t n_items) const {
    if (cta < shared_end) return cta;
    return own_first >= 0 ? shared_end + own_first : n_items;
  }
  __device__ __forceinline__ int64_t next(int64_t item, int64_t n_items) const {
    if (item < shared_end) {
      if (item + all < shared_end) return item + all;
      return own_first >= 0 ? shared_end + own_first : n_items;
    }
    return item + own_stride;
  }
};

// The prep work of one CTA (256 threads: warps 0-7) over the items of `sc`.  A CTA that
// allocates tensor memory again afterwards (a chain CTA of the fused launch) keeps its
// allocation permit (`last_alloc` false).  With `publish`, each item's
// flag is set once its stores have completed: by thread 0 right after it has issued the next
// item's first products (or after the loop, for the last item).
template <int DV>
__device__ __forceinline__ void prep_body(const ScanMaps &mp, const ScanLaunch &p, const ScanWs &ws,
                                          const ScanPlan &plan, const PrepSched &sc, bool publish,
                                          bool last_alloc = true) {
  const CUtensorMap &tm_q = mp.q, &tm_k = mp.k, &tm_v = mp.v, &tm_QW = mp.QW, &tm_PY = mp.PY,
                    &tm_KT = mp.KT, &tm_UT = mp.UT;
  extern __shared__ uint8_t smem_raw[];
  __shared__ PrepCtl ctl_s;
  PrepCtl *ctl = &ctl_s;
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  float *As = reinterpret_cast<float *>(sm + P_AF);
  float *Ts = reinterpret_cast<float *>(sm + P_TF);
  float *Xs = Ts + C * LDA;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, hsel = warp >> 2;   // TMEM lane quarter, column half
  const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
  const bool want_o = p.o != nullptr;
  const int64_t n_items = ws.slots;
  const int32_t *cu_chunks = plan_cu_chunks(plan, ws);
  const int32_t *cu_tokens = plan_cu_tokens(plan, p);

  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_QW);
    tma_prefetch_desc(&tm_PY);
    tma_prefetch_desc(&tm_KT);
    tma_prefetch_desc(&tm_UT);
    mbar_init(smem_u32(&ctl->tma_bar[0]), 1);
    mbar_init(smem_u32(&ctl->tma_bar[1]), 1);
    mbar_init(smem_u32(&ctl->mma_bar), 1);
    mbar_init(smem_u32(&ctl->mma_bar2), 1);
    mbar_init(smem_u32(&ctl->drain_bar), 1);
    mbar_init(smem_u32(&ctl->drain_bar2), 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl->tmem), 512);
    if (last_alloc) tmem_relinquish();
  }
  tc_fence_before();
  bar_sync_n(1, kPrepThreads);
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const AbortFlag ab{&ctl->abort, p.err_word, ERRBIT_SCAN_TIMEOUT, p.wait_ns};
  // TMEM is held: let the next kernel launch; then wait for the previous one's outputs
  pdl_trigger();
  pdl_wait();

  int fills[2] = {0, 0};   // TMA fills issued per stage (thread 0)
  int64_t prev_slot = -1;  // thread 0: the last item whose flag is not yet published
  auto issue = [&](const PrepItem &it, int buf) {
    const uint32_t bar = smem_u32(&ctl->tma_bar[buf]);
    const uint32_t st = smem_u32(sm + buf * P_STAGE);
    const uint32_t bytes = 16384u + (want_o ? 16384u : 0u) + (it.has_prev ? 16384u : 0u) +
                           (uint32_t)DV * 128u;
    mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int x = it.head * DK + 64 * h;
      if (want_o) tma_load_2d(st + h * 32768, &tm_q, x, it.t0, bar);
      tma_load_2d(st + h * 32768 + 8192, &tm_k, x, it.t0, bar);
      if (it.has_prev) tma_load_2d(st + h * 32768 + 16384, &tm_k, x, it.t0 - C, bar);
    }
#pragma unroll
    for (int h = 0; h < DV / 64; ++h)
      tma_load_2d(st + h * 32768 + 24576, &tm_v, it.head * DV + 64 * h, it.t0, bar);
    ++fills[buf];
  };
  // an item's gates, loaded into registers one item ahead: token tid (< 64) of the chunk,
  // and (threads 64..127) token tid - 64 of the previous chunk
  auto load_gates = [&](const PrepItem &it, float &la, float &b) {
    la = 0.f;
    b = 0.f;
    if (tid < C) {
      if (tid < it.nv) {
        la = p.log_alpha[(size_t)(it.t0 + tid) * p.H + it.head];
        b = p.beta[(size_t)(it.t0 + tid) * p.H + it.head];
      }
    } else if (tid < 2 * C && it.has_prev) {
      la = p.log_alpha[(size_t)(it.t0 - C + (tid - C)) * p.H + it.head];
    }
  };

  int64_t item = sc.first(n_items);
  int seq_cur = 0;   // threads 0 and 32: the sequence of the current item
  float la_next = 0.f, b_next = 0.f;
  if ((tid == 0 || tid == 32) && item < n_items) {
    seq_cur = seq_of_chunk((int)(item / p.H), p.n_seqs, cu_chunks);
    seq_cur = advance_seq(seq_cur, (int)(item / p.H), cu_chunks);
  }
  if (tid == 0 && item < n_items) {
    ctl->cur = item_at(item, seq_cur, p, cu_chunks, cu_tokens);
    fence_proxy_async_smem();
    issue(ctl->cur, 0);
  }
  bar_sync_n(1, kPrepThreads);
  if (item < n_items) load_gates(ctl->cur, la_next, b_next);

  const uint32_t mma_bar = smem_u32(&ctl->mma_bar);
  uint32_t mma_phase = 0;
  uint32_t mma2_phase = 0;
  bool mma_pending = false;   // threads 0, 64: products issued whose completion was not seen
  auto mma_wait = [&]() -> bool {
    const bool ok = mbar_wait(mma_bar, mma_phase, ab);
    mma_phase ^= 1u;
    if (tid == 0 && ok) mma_pending = false;
    if (bar_or_n(1, kPrepThreads, !ok)) return false;
    tc_fence_after();
    return true;
  };

  int n = 0;
  for (; item < n_items; item = sc.next(item, n_items), ++n) {
    const int buf = n & 1;
    uint8_t *ST = sm + buf * P_STAGE;
    const uint32_t st_u = smem_u32(ST);
    const PrepItem it = ctl->cur;
    const bool has_next = sc.next(item, n_items) < n_items;

    // gates: g = inclusive cumsum of log alpha (0 past the end), and the previous chunk's
    if (tid < 2 * C) {
      const float la = la_next, b = b_next;
      float s = la;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      if (tid < C) {
        ctl->g[tid] = s;
        ctl->beta[tid] = b;
      } else {
        ctl->gpv[tid - C] = s;
      }
    }
    bar_sync_n(1, kPrepThreads);
    if (tid >= 32 && tid < C) ctl->g[tid] += ctl->g[31];
    if (tid >= C + 32 && tid < 2 * C) ctl->gpv[tid - C] += ctl->gpv[31];
    bar_sync_n(1, kPrepThreads);
    if (tid < C) {
      const float gt = ctl->g[tid];
      ctl->gq[tid] = exp_ftz(gt);
      ctl->igq[tid] = exp_ftz(-gt);
      ctl->bg[tid] = ctl->beta[tid] * ctl->gq[tid];
      ctl->gp[tid] = exp_ftz(ctl->g[C - 1] - gt);
    } else if (tid < 2 * C) {
      ctl->gpp[tid - C] = it.has_prev ? exp_ftz(ctl->gpv[C - 1] - ctl->gpv[tid - C]) : 0.f;
    } else if (tid == 2 * C) {
      ctl->gc_prev = it.has_prev ? exp_ftz(ctl->gpv[C - 1]) : 1.f;
    }
    const bool ok_tma = mbar_wait(smem_u32(&ctl->tma_bar[buf]), (uint32_t)(n >> 1) & 1u, ab);
    if (bar_or_n(1, kPrepThreads, !ok_tma)) break;
    if (p.flags & TR_NORMALIZE_QK) {
      if (tid < C) normalize_band_row(ST, 1, tid);
      else if (tid < 2 * C && want_o) normalize_band_row(ST, 0, tid - C);
      else if (tid >= 2 * C && tid < 3 * C && it.has_prev) normalize_band_row(ST, 2, tid - 2 * C);
      fence_proxy_async_smem();
      bar_sync_n(1, kPrepThreads);
    }

    // group 1: [Q; K] [K; K_prev]^T -> TMEM cols [0, 128)
    if (tid == 0) {
      tc_fence_after();
      const uint64_t da = kmaj(st_u), db = kmaj(st_u + 8192);
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk)
        tc_mma_bf16(tmem, desc_k(da, kk, 32768), desc_k(db, kk, 32768),
                    idesc_bf16(128, 128, 0, 0), kk > 0);
      tc_commit(mma_bar);
      mma_pending = true;
      if (publish && prev_slot >= 0) {
        // the previous item's three store groups have completed: publish it for the chain
        bulk_wait<0>();
        publish_slot(ws, prev_slot, p.epoch);
        prev_slot = -1;
      } else {
        // the previous item's first store group (P, -Y) has read its staging: P and Z are
        // written below
        bulk_wait_read<2>();
      }
    } else if (tid == 32 && has_next) {
      // the next item's location, beside the products (its gates are loaded under the
      // inverse, its bands after group 2 is issued)
      const int64_t nx = sc.next(item, n_items);
      seq_cur = advance_seq(seq_cur, (int)(nx / p.H), cu_chunks);
      ctl->nxt = item_at(nx, seq_cur, p, cu_chunks, cu_tokens);
    }
    if (!mma_wait()) break;

    // P (rows 0-63, bf16), A (rows 64-127, fp32) and Z = K K~_prev^T (rows 64-127, bf16).
    // The decays e^{g_t - g_s} are gamma_t (1 / gamma_s) when the chunk's total decay keeps
    // 1 / gamma within fp32 (g_C > -80: then e^{-g} < 6e34): two exponentials per token
    // instead of one per pair; otherwise they are taken pair by pair.
    const bool factored = ctl->g[C - 1] > -80.f;
    {
      float v[32];
      // warps whose 32 columns all lie right of the diagonal (hsel 1, rows 0-31) write zeros
      const bool upper = hsel == 1 && (q4 & 1) == 0;
      if (q4 < 2) {
        if (want_o) {
          const int t = q4 * 32 + lane;
          if (upper) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          } else {
            tmem_ld32(tmem + lane_base + 32 * hsel, v);
            tc_wait_ld();
            if (factored) {
              const float et = ctl->gq[t];
              const float4 *ig = reinterpret_cast<const float4 *>(ctl->igq + 32 * hsel);
#pragma unroll
              for (int w = 0; w < 8; ++w) {
                const float4 q = ig[w];
                const float iq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int i = 4 * w + u, s = 32 * hsel + i;
                  v[i] = (s <= t) ? et * iq[u] * v[i] : 0.f;
                }
              }
            } else {
              const float gt = ctl->g[t];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int s = 32 * hsel + i;
                v[i] = (s <= t) ? exp_ftz(gt - ctl->g[s]) * v[i] : 0.f;
              }
            }
          }
          store_row_bf16(sm + P_P, t, 32 * hsel, v, 1.f);
        }
      } else {
        const int t = (q4 - 2) * 32 + lane;
        if (upper) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        } else {
          tmem_ld32(tmem + lane_base + 32 * hsel, v);
          tc_wait_ld();
          if (factored) {
            const float bet = ctl->beta[t] * ctl->gq[t];
            const float4 *ig = reinterpret_cast<const float4 *>(ctl->igq + 32 * hsel);
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              const float4 q = ig[w];
              const float iq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int i = 4 * w + u, s = 32 * hsel + i;
                v[i] = (s < t) ? bet * iq[u] * v[i] : 0.f;
              }
            }
          } else {
            const float gt = ctl->g[t], bt = ctl->beta[t];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int s = 32 * hsel + i;
              v[i] = (s < t) ? bt * exp_ftz(gt - ctl->g[s]) * v[i] : 0.f;
            }
          }
        }
        float4 *dst = reinterpret_cast<float4 *>(As + t * LDA + 32 * hsel);
#pragma unroll
        for (int w = 0; w < 8; ++w) dst[w] = make_float4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]);
        if (it.has_prev) {
          tmem_ld32(tmem + lane_base + 64 + 32 * hsel, v);
          tc_wait_ld();
          const float4 *gp4 = reinterpret_cast<const float4 *>(ctl->gpp + 32 * hsel);
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            const float4 g = gp4[w];
            v[4 * w] *= g.x;
            v[4 * w + 1] *= g.y;
            v[4 * w + 2] *= g.z;
            v[4 * w + 3] *= g.w;
          }
          store_row_bf16(sm + P_Z, t, 32 * hsel, v, 1.f);
        }
      }
    }
    bar_sync_n(1, kPrepThreads);
    // the next item's gates: their loads run under the inverse
    if (has_next) load_gates(ctl->nxt, la_next, b_next);

    // T = (I + A)^{-1}, blocked.  (a) the four 16 x 16 diagonal blocks by forward
    // substitution (thread = column, fp32 registers); (b) each 32 x 32 diagonal block from
    // its two 16-blocks: T21 = -T22 (A21 T11); (c) the 64 x 64 from the two 32-blocks the
    // same way.
    if (tid < C) {
      const int base = 16 * (tid >> 4), c = tid & 15;
      float Tc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 *Ar4 = reinterpret_cast<const float4 *>(As + (base + i) * LDA + base);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const int s = 4 * s4;
          if (s < i) {
            const float4 a = Ar4[s4];
            a0 = fmaf(a.x, Tc[s], a0);
            if (s + 1 < i) a1 = fmaf(a.y, Tc[s + 1], a1);
            if (s + 2 < i) a2 = fmaf(a.z, Tc[s + 2], a2);
            if (s + 3 < i) a3 = fmaf(a.w, Tc[s + 3], a3);
          }
        }
        Tc[i] = (i == c) ? 1.f : ((i < c) ? 0.f : -((a0 + a1) + (a2 + a3)));
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) Ts[(base + i) * LDA + base + c] = Tc[i];
    } else if (want_o) {
      // meanwhile the other warps scale Q by gamma in place (64 rows x 4 pieces of 32
      // columns; the Q band was group 1's operand only)
      for (int pc = tid - C; pc < 4 * C; pc += kPrepThreads - C) {
        const int r = pc & 63, q = pc >> 6;
        scale_row32_bf16(ST + (q >> 1) * 32768, r, 32 * (q & 1), ctl->gq[r]);
      }
    }
    bar_sync_n(1, kPrepThreads);
    const int mJ = tid >> 7, mr = (tid >> 3) & 15, mc = (tid & 7) * 2;
    {  // X16 = A21 T11 within 32-block J
      const float *Ar = As + (32 * mJ + 16 + mr) * LDA + 32 * mJ;
      float x0 = 0.f, x1 = 0.f;
#pragma unroll
      for (int s = 0; s < 16; s += 4) {
        const float4 a = *reinterpret_cast<const float4 *>(Ar + s);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 t = *reinterpret_cast<const float2 *>(Ts + (32 * mJ + s + u) * LDA + 32 * mJ + mc);
          x0 = fmaf(av[u], t.x, x0);
          x1 = fmaf(av[u], t.y, x1);
        }
      }
      *reinterpret_cast<float2 *>(Xs + (16 * mJ + mr) * LDX + mc) = make_float2(x0, x1);
      // the upper-right 16 x 16 of the 32-block is zero (T is lower triangular)
      *reinterpret_cast<float2 *>(Ts + (32 * mJ + mr) * LDA + 32 * mJ + 16 + mc) =
          make_float2(0.f, 0.f);
    }
    bar_sync_n(1, kPrepThreads);
    {  // T21 = -T22 X16 within block J (T22 lower triangular)
      const float *Tr = Ts + (32 * mJ + 16 + mr) * LDA + 32 * mJ + 16;
      float x0 = 0.f, x1 = 0.f;
#pragma unroll
      for (int s = 0; s < 16; s += 4) {
        const float4 a = *reinterpret_cast<const float4 *>(Tr + s);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 t = *reinterpret_cast<const float2 *>(Xs + (16 * mJ + s + u) * LDX + mc);
          x0 = fmaf(av[u], t.x, x0);
          x1 = fmaf(av[u], t.y, x1);
        }
      }
      *reinterpret_cast<float2 *>(Ts + (32 * mJ + 16 + mr) * LDA + 32 * mJ + mc) =
          make_float2(-x0, -x1);
    }
    bar_sync_n(1, kPrepThreads);
    if (tid < 128) {  // X = A21 T11 (32 x 32): thread -> rows r, r + 16, columns c0..c0+3
      // (two rows per thread: each T11 row read from shared memory serves 8 products; the
      // phase is bound by shared-memory bytes, not by threads)
      const int r = tid >> 3, c0 = (tid & 7) * 4;
      float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const float *Ar0 = As + (32 + r) * LDA, *Ar1 = As + (48 + r) * LDA;
#pragma unroll 2
      for (int s = 0; s < 32; s += 4) {
        const float4 a0 = *reinterpret_cast<const float4 *>(Ar0 + s);
        const float4 a1 = *reinterpret_cast<const float4 *>(Ar1 + s);
        const float av[2][4] = {{a0.x, a0.y, a0.z, a0.w}, {a1.x, a1.y, a1.z, a1.w}};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 t = *reinterpret_cast<const float4 *>(Ts + (s + u) * LDA + c0);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            x[h][0] = fmaf(av[h][u], t.x, x[h][0]); x[h][1] = fmaf(av[h][u], t.y, x[h][1]);
            x[h][2] = fmaf(av[h][u], t.z, x[h][2]); x[h][3] = fmaf(av[h][u], t.w, x[h][3]);
          }
        }
      }
      *reinterpret_cast<float4 *>(Xs + r * LDX + c0) = make_float4(x[0][0], x[0][1], x[0][2], x[0][3]);
      *reinterpret_cast<float4 *>(Xs + (r + 16) * LDX + c0) =
          make_float4(x[1][0], x[1][1], x[1][2], x[1][3]);
    }
    bar_sync_n(1, kPrepThreads);
    {  // T21 = -T22 X: thread -> row r, columns c0..c0+3; T22 is lower triangular, so
       // columns s > r of it contribute nothing (the warp's rows end at 4 warp + 3)
      const int r = tid >> 3, c0 = (tid & 7) * 4;
      float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
      const float *Tr = Ts + (32 + r) * LDA + 32;
#pragma unroll
      for (int s = 0; s < 32; s += 4) {
        if (s > 4 * warp + 3) break;
        const float4 a = *reinterpret_cast<const float4 *>(Tr + s);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 t = *reinterpret_cast<const float4 *>(Xs + (s + u) * LDX + c0);
          x0 = fmaf(av[u], t.x, x0); x1 = fmaf(av[u], t.y, x1);
          x2 = fmaf(av[u], t.z, x2); x3 = fmaf(av[u], t.w, x3);
        }
      }
      *reinterpret_cast<float4 *>(Ts + (32 + r) * LDA + c0) = make_float4(-x0, -x1, -x2, -x3);
    }
    // the previous item's second store group (U~) has read the T tiles written below
    if (tid == 0) bulk_wait_read<1>();
    bar_sync_n(1, kPrepThreads);
    {  // [T diag(beta gamma); T diag(beta)] as high + low bf16 parts; consecutive lanes take
       // consecutive rows (conflict-free reads of T and swizzled stores)
      const int rr = tid & 127, half = tid >> 7, t = rr & 63;
      const bool zero = t < 32 && half == 1;  // T is lower triangular: T12 = 0
      // the column scales, four per (broadcast) read
      const float4 *sc4 =
          reinterpret_cast<const float4 *>((rr < C ? ctl->bg : ctl->beta) + 32 * half);
      float v[32];
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float4 tv = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                               : *reinterpret_cast<const float4 *>(Ts + t * LDA + 32 * half + 4 * w);
        const float4 sv = sc4[w];
        v[4 * w] = tv.x * sv.x;
        v[4 * w + 1] = tv.y * sv.y;
        v[4 * w + 2] = tv.z * sv.z;
        v[4 * w + 3] = tv.w * sv.w;
      }
      store_row_split<false>(sm + P_THI, sm + P_TLO, rr, 32 * half, v, 1.f);
    }
    fence_proxy_async_smem();
    bar_sync_n(1, kPrepThreads);

    // group 2, issued by thread 64 in two parts: [T'; T''] K -> cols [128, 256) (rows 0-63:
    // W) and [T'; T''] Z -> [384, 448) (rows 0-63: Y), committed for the W / Y epilogue; then
    // [T'; T''] V (hi + lo) -> [256, 256 + DV) (rows 64-127: U~).  Thread 0 meanwhile
    // prefetches the next item into the other stage, once the previous item's output
    // stores have finished reading their staging there (issued an item ago: usually done).
    if (tid == 64) {
      tc_fence_after();
      const uint64_t th = kmaj(smem_u32(sm + P_THI)), tl = kmaj(smem_u32(sm + P_TLO));
      const uint64_t dk_ = mnmaj(st_u + 8192, 32768), dv_ = mnmaj(st_u + 24576, 32768);
      const uint64_t dz = mnmaj(smem_u32(sm + P_Z), 8192);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 128, desc_k(th, kk, 0), desc_mn(dk_, kk), idesc_bf16(128, 128, 0, 1), kk > 0);
      if (it.has_prev) {
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(tmem + 384, desc_k(th, kk, 0), desc_mn(dz, kk), idesc_bf16(128, 64, 0, 1), kk > 0);
      }
      tc_commit(mma_bar);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 256, desc_k(th, kk, 0), desc_mn(dv_, kk), idesc_bf16(128, DV, 0, 1), kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 256, desc_k(tl, kk, 0), desc_mn(dv_, kk), idesc_bf16(128, DV, 0, 1), 1u);
      tc_commit(smem_u32(&ctl->mma_bar2));
      mma_pending = true;
    } else if (tid == 0) {
      bulk_wait_read<0>();
      if (has_next) {
        fence_proxy_async_smem();
        issue(ctl->nxt, buf ^ 1);
      }
    }
    // lane quarters 0, 1 (W, Y) wait for the first part, quarters 2, 3 (U~) for the second
    const bool ok2 = mbar_wait(q4 < 2 ? mma_bar : smem_u32(&ctl->mma_bar2),
                               q4 < 2 ? mma_phase : mma2_phase, ab);
    mma_phase ^= 1u;
    mma2_phase ^= 1u;
    if (tid == 64 && ok2) mma_pending = false;
    if (ok2) {
      tc_fence_after();
      float v[32];
      if (q4 < 2) {
        const int t = q4 * 32 + lane;
        // -gamma_C(prev) W -> the previous-K band of half hsel (row t)
        const float s = -ctl->gc_prev;
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          tmem_ld32(tmem + 128 + lane_base + 64 * hsel + 32 * j, v);
          tc_wait_ld();
          store_row_bf16(ST + hsel * 32768 + 16384, t, 32 * j, v, s);
        }
        if (it.has_prev) {  // -Y -> the Z tile (consumed)
          tmem_ld32(tmem + 384 + lane_base + 32 * hsel, v);
          tc_wait_ld();
          store_row_bf16(sm + P_Z, t, 32 * hsel, v, -1.f);
        }
      } else {
        const int t = (q4 - 2) * 32 + lane;
        // U~ row t (fp32), columns (DV/2) hsel.. -> 32-column boxes over the T tiles
#pragma unroll 1
        for (int j = 0; j < DV / 64; ++j) {
          const int col = (DV / 2) * hsel + 32 * j;
          tmem_ld32(tmem + 256 + lane_base + col, v);
          tc_wait_ld();
          store_row32_f32(sm + P_THI + 8192 * (col >> 5), t, v, 1.f);
        }
      }
    }
    if (bar_or_n(1, kPrepThreads, !ok2)) break;
    fence_proxy_async_smem();
    tc_fence_before();
    bar_sync_n(1, kPrepThreads);
    if (tid == 0) {
      const int64_t slot = it.slot;
      const int32_t y128 = (int32_t)(slot * 128), y64 = (int32_t)(slot * 64);
      // three bulk groups, in the order their staging is written again by the next item:
      // P and -Y (p1), U~ (over the T tiles: p3), the stage's bands (the prefetch after it)
      if (want_o) tma_store_2d(&tm_PY, smem_u32(sm + P_P), 0, y128);
      if (it.has_prev) tma_store_2d(&tm_PY, smem_u32(sm + P_Z), 0, y128 + 64);
      bulk_commit();
#pragma unroll
      for (int b = 0; b < DV / 32; ++b)
        tma_store_2d(&tm_UT, smem_u32(sm + P_THI + 8192 * b), 32 * b, y64);
      bulk_commit();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (want_o) tma_store_2d(&tm_QW, st_u + h * 32768, 64 * h, y128);
        tma_store_2d(&tm_QW, st_u + h * 32768 + 16384, 64 * h, y128 + 64);
        if (p.flags & TR_NORMALIZE_QK) tma_store_2d(&tm_KT, st_u + h * 32768 + 8192, 64 * h, y64);
      }
      bulk_commit();
      ws.G[slot * 4] = exp_ftz(ctl->g[C - 1]);
      if (has_next) ctl->cur = ctl->nxt;
      if (publish) prev_slot = slot;   // published once its stores complete
    }
    if (tid < C) ws.GP[it.slot * C + tid] = ctl->gp[tid];
    bar_sync_n(1, kPrepThreads);
  }

  if (tid == 0) {
    // every output store has completed before the grid does (the chain reads them)
    bulk_wait<0>();
    if (publish && prev_slot >= 0 && item >= n_items) publish_slot(ws, prev_slot, p.epoch);
    if (item < n_items) {
      // left the loop at a wait that gave up: nothing issued may still be in flight when
      // the CTA releases its shared memory and TMEM
      for (int b = 0; b < 2; ++b)
        if (fills[b] > 0) mbar_wait_drain(smem_u32(&ctl->tma_bar[b]), (uint32_t)(fills[b] - 1) & 1u);
      if (mma_pending) {
        tc_commit(smem_u32(&ctl->drain_bar));
        mbar_wait_drain(smem_u32(&ctl->drain_bar), 0);
      }
    }
  }
  if (tid == 64 && item < n_items && mma_pending) {
    tc_commit(smem_u32(&ctl->drain_bar2));
    mbar_wait_drain(smem_u32(&ctl->drain_bar2), 0);
  }
  tc_fence_before();
  bar_sync_n(1, kPrepThreads);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DV>
__global__ void __launch_bounds__(kPrepThreads, 1)
    scan_prep_kernel(const __grid_constant__ ScanMaps mp, const __grid_constant__ ScanLaunch p,
                     const __grid_constant__ ScanWs ws, const __grid_constant__ ScanPlan plan) {
  prep_body<DV>(mp, p, ws, plan, PrepSched{0, 0, 1, (int64_t)blockIdx.x, (int)gridDim.x}, false);
}

// =========================================================== chain kernel
// One CTA per (sequence, head, 64-column slice of d_v), in longest-first order of the
// sequences; 384 threads:
//   warp 0      TMA producer: stage k (k = 0..n) holds chunk k-1's gamma Q, P, K~ and
//               gamma_C and chunk k's -gamma_C W, -Y and U~ slice (2 stages; the MMA
//               operands and the epilogue operands each with their own barriers)
//   warp 1      MMA issuer (one thread)
//   warps 2-5   state warps: thread (quarter q = warp % 4) owns row d = 32 q + lane of the
//               fp32 state slice M (64 columns in registers); M_{c+1} = gamma_C M_c + dM
//   warps 6, 7, 10, 11  U warps (TMEM lanes 64-127; 6, 7 columns 0-31, 10, 11 columns
//               32-63): U_{c+1} = U~_{c+1} + D rows 64-127, written as bf16 and
//               gamma' U_{c+1} as a bf16 hi + lo pair (shared memory)
//   warps 8, 9  O warps (TMEM lanes 0-63): the chunk's output rows, bf16, stored by TMA
//               (off the chain's critical path)
// The state and U warps signal the issuer warp by warp (mbarrier counts of 4), with no CTA
// barrier on the step's path.
// Per chunk c the issuer waits for M_c and U_c and issues
//   D[c % 2] = A1 M_c (8 MMAs; 16 with the state as a hi + lo pair) once M_c is ready, then,
//   once U_c is, dM = K^T [gamma' U_c hi | lo] (4 MMAs of N = 128), commit S;
//   D[c % 2] += A2 U_c (4), commit D (and the buffer's output barrier).  TMEM: D[2] at
//   columns 0 and 64, dM at 128 (hi) and 192 (lo).
constexpr uint32_t C_A1 = 0;        // [2 halves][128 rows][128 B]
constexpr uint32_t C_A2 = 32768;    // [128 rows][128 B]
constexpr uint32_t C_KT = 49152;    // [2 halves][64 rows][128 B]
constexpr uint32_t C_UT = 65536;    // [2 boxes][64 rows][32 fp32]
constexpr uint32_t C_GP = 81920;    // gamma' [64] fp32
constexpr uint32_t C_G = 82176;     // gamma_C (16 bytes)
constexpr uint32_t C_STAGE = 82944;
constexpr uint32_t C_MT = 2 * C_STAGE;          // M bf16 [128 d][64 cols] (high parts)
constexpr uint32_t C_MTL = C_MT + 16384;        // low parts (precise_state)
constexpr uint32_t C_UTL = C_MTL + 16384;       // U bf16 [64 t][64 cols]
constexpr uint32_t C_GUH = C_UTL + 8192;        // gamma' U, high bf16 parts
constexpr uint32_t C_GUL = C_GUH + 8192;        // low parts
constexpr size_t CHAIN_SMEM = C_GUL + 8192 + 1024;
static_assert(C_MT % 1024 == 0, "swizzled tiles are 1024-byte aligned");
constexpr int kChainThreads = 384;
static_assert(CHAIN_SMEM <= 232448, "chain shared memory");

struct ChainCtl {
  uint64_t full[2], empty[2];   // the stage's epilogue operands: landed / read
  uint64_t full_m[2], empty_m[2];   // its MMA operands: landed / read (the issuer's commit)
  uint64_t bar_s, bar_d, bar_m, bar_u, drain;
  uint64_t bar_dO[2];   // D[b] holds a finished chunk output (for the O warps)
  uint64_t bar_o[2];    // the O warps have read D[b]
  uint32_t tmem;
  int abort;
};

// Wait until the prep running beside this chain (fused launch) has published the slots a
// stage reads (`n` of them, 1 or 2): acquire loads of their flags, repeated (bounded like
// every other wait) until both carry this call's epoch, then a proxy fence that orders them
// before this thread's TMA loads of the slots' data.  (A generic fence instead of acquire
// loads made the chain slower: it waited for this thread's bulk copies in flight.)
__device__ bool wait_slots(const ScanWs &ws, const int64_t (&slot)[2], int n,
                           unsigned long long epoch, const AbortFlag &ab) {
  auto ready = [&]() {
    unsigned long long v[2] = {epoch, epoch};
    for (int i = 0; i < n; ++i)
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v[i]) : "l"(ws.flags + slot[i]) : "memory");
    return v[0] == epoch && v[1] == epoch;
  };
  if (!ready()) {
    const unsigned long long t0 = globaltimer_ns();
    for (int i = 0;; ++i) {
      __nanosleep(64);
      if (ready()) break;
      if ((i & 15) == 15) {
        if (*ab.flag) return false;
        if (globaltimer_ns() - t0 > ab.limit_ns) {
          *ab.flag = 1;
          if (ab.err_word) atomicOr(ab.err_word, ab.err_bit);
          return false;
        }
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// The chain of CTA `cta` (384 threads); with `wait_flags` each stage's slots are awaited
// first (their prep runs in the same launch).  SPL CTAs share one 64-column tile of d_v:
// with SPL = 2 each carries 32 of its state columns (the columns of M, U and the products
// are independent): the products still run over the whole tile (at the tensor pipe's
// per-instruction floor N = 32 and N = 64 cost the same), the other half's columns are
// zero, and each CTA's epilogues do half the work, on two U warps.
template <int SPL>
__device__ __forceinline__ void chain_body(const ScanMaps &mp, const ScanLaunch &p,
                                           const ScanWs &ws, const ScanPlan &plan, int cta,
                                           bool wait_flags) {
  static_assert(SPL == 1 || SPL == 2, "one or two CTAs per 64-column tile");
  constexpr int CN = DVS / SPL;     // state columns this CTA carries
  constexpr int NU = 4 / SPL;       // U warps
  const CUtensorMap &tm_QW = mp.QW, &tm_PY = mp.PY, &tm_KT = mp.KT, &tm_UT = mp.UT, &tm_o = mp.o,
                    &tm_k = mp.k;
  // K of a chunk: the prep's normalised copy, or the scan's own k input (no copy made)
  const bool kt_ws = (p.flags & TR_NORMALIZE_QK) != 0;
  extern __shared__ uint8_t smem_raw[];
  __shared__ ChainCtl ctl_s;
  ChainCtl *ctl = &ctl_s;
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = p.dv / DVS;
  const int H = p.H;
  const int per_head = NS * SPL;
  const int pos = cta / (H * per_head);
  const int head = (cta / per_head) % H, sub = cta % per_head;
  const int slice = sub / SPL, part = sub % SPL;
  const int c_lo = part * CN;       // this CTA's first column within the tile
  const bool want_o = p.o != nullptr;
  if (SPL > 1) {
    // the other half of the MMA operand tiles stays zero
    for (uint32_t o = 16u * (uint32_t)tid; o < C_GUL + 8192 - C_MT; o += 16u * kChainThreads)
      *reinterpret_cast<uint4 *>(sm + C_MT + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }

  if (tid == 0) {
    tma_prefetch_desc(&tm_QW);
    tma_prefetch_desc(&tm_PY);
    tma_prefetch_desc(&tm_KT);
    tma_prefetch_desc(&tm_UT);
    if (want_o) tma_prefetch_desc(&tm_o);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 4 + NU);   // each state warp and each U warp
      mbar_init(smem_u32(&ctl->full_m[s]), 1);
      mbar_init(smem_u32(&ctl->empty_m[s]), 1);
    }
    mbar_init(smem_u32(&ctl->bar_s), 1);
    mbar_init(smem_u32(&ctl->bar_d), 1);
    mbar_init(smem_u32(&ctl->bar_m), 4);        // each state warp
    mbar_init(smem_u32(&ctl->bar_u), NU);       // each U warp
    mbar_init(smem_u32(&ctl->drain), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->bar_dO[b]), 1);
      mbar_init(smem_u32(&ctl->bar_o[b]), 1);
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl->tmem), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const AbortFlag ab{&ctl->abort, p.err_word, ERRBIT_SCAN_TIMEOUT, p.wait_ns};
  // TMEM is held: let the next kernel launch; then wait for the previous one's outputs
  pdl_trigger();
  pdl_wait();

  const int seq = plan_order(plan, ws)[pos];
  const int cb = plan_cu_chunks(plan, ws)[seq];
  const int32_t *cu_tokens = plan_cu_tokens(plan, p);
  const int t_begin = cu_tokens[seq], t_end = cu_tokens[seq + 1];
  const int n = (t_end - t_begin + C - 1) / C;
  auto slot_of = [&](int c) -> int64_t { return ((int64_t)cb + c) * H + head; };
  const bool s0 = p.S0 != nullptr;
  const uint32_t mt_u = smem_u32(sm + C_MT), utl_u = smem_u32(sm + C_UTL);
  int last_k[2] = {-1, -1};   // producer: the last stage whose epilogue part was loaded
  int last_m[2] = {-1, -1};   // ... and whose MMA part was
  bool mma_pending = false;   // issuer: products issued whose completion was not seen

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    // A stage is refilled in two parts: the MMA operands (gamma Q, P, K~, -gamma_C W, -Y)
    // as soon as the issuer's products of its last use have completed, the epilogue
    // operands (gamma_C, the U~ slice, gamma') once the state and U warps have read them.
    // The first part's loads thus run under the last use's epilogues.
    if (lane == 0) {
      for (int k = 0; k <= n; ++k) {
        const int st = k & 1;
        const bool cur = k >= 1, nxt = k <= n - 1;
        const uint32_t bytes_m = (cur ? (want_o ? 16384u + 8192u : 0u) + 16384u : 0u) +
                                 (nxt ? 16384u + (k >= 1 ? 8192u : 0u) : 0u);
        const uint32_t bytes_e = (cur ? 16u : 0u) + (nxt ? 16384u / SPL + 256u : 0u);
        const int64_t sc = cur ? slot_of(k - 1) : 0, sn = nxt ? slot_of(k) : 0;
        const uint32_t par = (uint32_t)((k - 2) >> 1) & 1u;
        // the slots' flags first: their check runs while the stage is still in use
        if (wait_flags && (cur || nxt)) {
          const int64_t sl[2] = {cur ? sc : sn, sn};
          if (!wait_slots(ws, sl, (cur && nxt) ? 2 : 1, p.epoch, ab)) break;
        }
        if (k >= 2 && !mbar_wait(smem_u32(&ctl->empty_m[st]), par, ab)) break;
        const uint32_t bar_mm = smem_u32(&ctl->full_m[st]), bar = smem_u32(&ctl->full[st]);
        const uint32_t base = smem_u32(sm + st * C_STAGE);
        mbar_arrive_expect_tx(bar_mm, bytes_m);
        if (cur) {
          if (want_o) {
            tma_load_2d(base + C_A1, &tm_QW, 0, (int32_t)(sc * 128), bar_mm);
            tma_load_2d(base + C_A1 + 16384, &tm_QW, 64, (int32_t)(sc * 128), bar_mm);
            tma_load_2d(base + C_A2, &tm_PY, 0, (int32_t)(sc * 128), bar_mm);
          }
          if (kt_ws) {
            tma_load_2d(base + C_KT, &tm_KT, 0, (int32_t)(sc * 64), bar_mm);
            tma_load_2d(base + C_KT + 8192, &tm_KT, 64, (int32_t)(sc * 64), bar_mm);
          } else {
            // rows past the sequence's end are other tokens or zero fill: their U rows are 0
            const int32_t t0 = t_begin + C * (k - 1);
            tma_load_2d(base + C_KT, &tm_k, head * DK, t0, bar_mm);
            tma_load_2d(base + C_KT + 8192, &tm_k, head * DK + 64, t0, bar_mm);
          }
        }
        if (nxt) {
          tma_load_2d(base + C_A1 + 8192, &tm_QW, 0, (int32_t)(sn * 128 + 64), bar_mm);
          tma_load_2d(base + C_A1 + 16384 + 8192, &tm_QW, 64, (int32_t)(sn * 128 + 64), bar_mm);
          if (k >= 1)
            tma_load_2d(base + C_A2 + 8192, &tm_PY, 0, (int32_t)(sn * 128 + 64), bar_mm);
        }
        last_m[st] = k;
        if (k >= 2 && !mbar_wait(smem_u32(&ctl->empty[st]), par, ab)) break;
        mbar_arrive_expect_tx(bar, bytes_e);
        if (cur) bulk_load(base + C_G, ws.G + sc * 4, 16u, bar);
        if (nxt) {
          // the U~ columns this CTA carries (boxes of 32)
          for (int bx = c_lo / 32; bx < (c_lo + CN) / 32; ++bx)
            tma_load_2d(base + C_UT + 8192 * bx, &tm_UT, slice * DVS + 32 * bx, (int32_t)(sn * 64),
                        bar);
          bulk_load(base + C_GP, ws.GP + sn * C, 256u, bar);
        }
        last_k[st] = k;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      const uint32_t bar_s = smem_u32(&ctl->bar_s), bar_d = smem_u32(&ctl->bar_d);
      const uint64_t md = mnmaj(mt_u, 16384), ud = mnmaj(utl_u, 8192);
      const uint64_t mdl = mnmaj(smem_u32(sm + C_MTL), 16384);
      const bool lo2 = p.precise_state;
      const uint64_t gu = mnmaj(smem_u32(sm + C_GUH), 8192);   // [hi | lo] blocks, 8 KB apart
      const uint32_t id_s = idesc_bf16(128, 2 * DVS, 1, 1);
      const uint32_t id_mn = idesc_bf16(128, DVS, 0, 1);
      bool ok = mbar_wait(smem_u32(&ctl->full_m[0]), 0, ab);
      if (ok && s0) {
        // U_0 = U~_0 - W_0 M_0: D[1] rows 64-127 = -W_0 M_0
        ok = mbar_wait(smem_u32(&ctl->bar_m), 0, ab);
        if (ok) {
          tc_fence_after();
          const uint64_t a1 = kmaj(smem_u32(sm + C_A1));
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            tc_mma_bf16(tmem + 64, desc_k(a1, kk, 16384), desc_mn(md, kk), id_mn, kk > 0);
          if (lo2) {
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
              tc_mma_bf16(tmem + 64, desc_k(a1, kk, 16384), desc_mn(mdl, kk), id_mn, 1u);
          }
          tc_commit(bar_d);
          mma_pending = true;
        }
      }
      // stage 0's MMA operands (read by the products above, if any) may be refilled
      if (ok) {
        if (s0)
          tc_commit(smem_u32(&ctl->empty_m[0]));
        else
          mbar_arrive(smem_u32(&ctl->empty_m[0]));
      }
      for (int j = 0; ok && j < n; ++j) {
        const int k = j + 1, st = k & 1;
        const uint32_t base = smem_u32(sm + st * C_STAGE);
        const uint32_t dcol = tmem + 64 * (j & 1);
        const uint64_t a1 = kmaj(base + C_A1), a2 = kmaj(base + C_A2);
        const uint64_t kt = mnmaj(base + C_KT, 8192);
        // D = A1 M_j as soon as M_j is ready (it does not need U_j), once the O warps have
        // read D[j % 2]'s previous chunk
        if (!mbar_wait(smem_u32(&ctl->full_m[st]), (uint32_t)(k >> 1) & 1u, ab)) break;
        if (!mbar_wait(smem_u32(&ctl->bar_m), (uint32_t)j & 1u, ab)) break;
        if (want_o && j >= 2 &&
            !mbar_wait(smem_u32(&ctl->bar_o[j & 1]), (uint32_t)((j >> 1) - 1) & 1u, ab))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          tc_mma_bf16(dcol, desc_k(a1, kk, 16384), desc_mn(md, kk), id_mn, kk > 0);
        if (lo2) {
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            tc_mma_bf16(dcol, desc_k(a1, kk, 16384), desc_mn(mdl, kk), id_mn, 1u);
        }
        mma_pending = true;
        if (!mbar_wait(smem_u32(&ctl->bar_u), (uint32_t)j & 1u, ab)) break;
        tc_fence_after();
        // dM = K^T [gamma' U_hi | gamma' U_lo]: one N = 128 product, two 64-column results
        // the state warps add; then D += A2 U_j
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(tmem + 128, desc_mn(kt, kk), desc_mn(gu, kk), id_s, kk > 0);
        tc_commit(bar_s);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(dcol, desc_k(a2, kk, 0), desc_mn(ud, kk), id_mn, 1u);
        tc_commit(bar_d);
        tc_commit(smem_u32(&ctl->empty_m[st]));
        if (want_o) tc_commit(smem_u32(&ctl->bar_dO[j & 1]));
      }
      // the last step's products complete before the final barrier either way: the state
      // and output warps wait for them, or, after an abort, the drain below does
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------- state warps
    const int q = warp & 3, d = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    float M[CN];
    const size_t s_off =
        ((size_t)(seq * H + head) * DK + d) * p.dv + (size_t)slice * DVS + (size_t)c_lo;
    if (s0) {
#pragma unroll
      for (int j = 0; j < CN; j += 4) {
        const float4 a = *reinterpret_cast<const float4 *>(p.S0 + s_off + j);
        M[j] = a.x; M[j + 1] = a.y; M[j + 2] = a.z; M[j + 3] = a.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < CN; ++j) M[j] = 0.f;
    }
    bool failed = false;
    const bool lo2 = p.precise_state;
    auto store_state = [&]() {
#pragma unroll
      for (int h = 0; h < CN / 32; ++h) {
        if (lo2)
          store_row_split<false>(sm + C_MT, sm + C_MTL, d, c_lo + 32 * h, M + 32 * h, 1.f);
        else
          store_row_bf16(sm + C_MT, d, c_lo + 32 * h, M + 32 * h, 1.f);
      }
    };
    // each warp signals on its own (no CTA barrier on the step's path); a warp that gives
    // up a wait leaves, and the abort flag ends every other role's next wait
    if (n > 0) {
      store_state();
      fence_proxy_async_smem();
      __syncwarp();
      // (the test hook withholds this signal: every role's bounded wait then runs out)
      if (lane == 0 && !(p.flags & TR_SCAN_STALL_TEST)) mbar_arrive(smem_u32(&ctl->bar_m));
    }
    for (int j = 0; j < n; ++j) {
      const int k = j + 1, st = k & 1;
      // gamma_C first (it lands long before the product)
      bool got = mbar_wait(smem_u32(&ctl->full[st]), (uint32_t)(k >> 1) & 1u, ab);
      const float gC = got ? *reinterpret_cast<const float *>(sm + st * C_STAGE + C_G) : 0.f;
      got = got && mbar_wait(smem_u32(&ctl->bar_s), (uint32_t)j & 1u, ab);
      if (!__all_sync(0xffffffffu, got)) {
        failed = true;
        break;
      }
      tc_fence_after();
      float v0[32], v1[32];
#pragma unroll
      for (int h = 0; h < CN / 32; ++h) {
        tmem_ld32(tmem + 128 + lane_base + c_lo + 32 * h, v0);   // K^T (gamma' U_hi)
        tmem_ld32(tmem + 192 + lane_base + c_lo + 32 * h, v1);   // K^T (gamma' U_lo)
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          add_f32x2(v0[i], v0[i + 1], v1[i], v1[i + 1]);
          fma_f32x2(M[32 * h + i], M[32 * h + i + 1], gC, v0[i], v0[i + 1]);
        }
      }
      if (j + 1 < n) {
        store_state();
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (j + 1 < n) mbar_arrive(smem_u32(&ctl->bar_m));
        mbar_arrive(smem_u32(&ctl->empty[st]));   // gamma_C read
      }
    }
    if (!failed) {
      float *dst = p.S_final + s_off;
#pragma unroll
      for (int j = 0; j < CN; j += 4)
        *reinterpret_cast<float4 *>(dst + j) = make_float4(M[j], M[j + 1], M[j + 2], M[j + 3]);
    }
  } else if (SPL == 1 ? (warp < 8 || warp >= 10) : warp < 8) {
    // ------------------------------------------------------------- U warps
    // warps 6, 7 (columns 0-31) and 10, 11 (columns 32-63), TMEM lanes 64-127:
    // U_{c+1} = U~_{c+1} + D rows 64-127, written as bf16 (for A2 U) and gamma' U as a bf16
    // hi + lo pair (for dM); each warp then announces its part
    // with SPL = 2 warps 6 and 7 take this CTA's 32 columns; warps 10 and 11 have no role
    const int q = warp & 3, t = 32 * (q - 2) + lane, ch = SPL == 1 ? (warp >= 10 ? 1 : 0) : part;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    uint32_t d_phase = 0;
    if (n > 0) {
      bool ok = mbar_wait(smem_u32(&ctl->full[0]), 0, ab);
      if (ok && s0) {
        ok = mbar_wait(smem_u32(&ctl->bar_d), d_phase, ab);
        d_phase ^= 1u;
      }
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const float gp = reinterpret_cast<const float *>(sm + C_GP)[t];
        float u[32], v[32];
        if (s0) tmem_ld32(tmem + 64 + lane_base + 32 * ch, v);
        load_row32_f32(sm + C_UT + 8192 * ch, t, u);
        if (s0) {
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] += v[i];
        }
        store_row_bf16(sm + C_UTL, t, 32 * ch, u, 1.f);
        store_row_split(sm + C_GUH, sm + C_GUL, t, 32 * ch, u, gp);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&ctl->bar_u));
          // its own arrival, and the state warps' share: stage 0 holds no gamma_C
          for (int i = 0; i < 1 + 4 / NU; ++i) mbar_arrive(smem_u32(&ctl->empty[0]));
        }
        for (int j = 0; j < n; ++j) {
          const int k = j + 1, st = k & 1;
          // the stage's U~ row and gamma' first (they land long before the products)
          bool got = mbar_wait(smem_u32(&ctl->full[st]), (uint32_t)(k >> 1) & 1u, ab);
          float gq = 0.f;
          if (got && j + 1 < n) {
            gq = reinterpret_cast<const float *>(sm + st * C_STAGE + C_GP)[t];
            load_row32_f32(sm + st * C_STAGE + C_UT + 8192 * ch, t, u);
          }
          got = got && mbar_wait(smem_u32(&ctl->bar_d), d_phase, ab);
          if (!__all_sync(0xffffffffu, got)) break;
          d_phase ^= 1u;
          tc_fence_after();
          if (j + 1 < n) {
            tmem_ld32(tmem + 64 * (j & 1) + lane_base + 32 * ch, v);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 2) add_f32x2(u[i], u[i + 1], v[i], v[i + 1]);
            store_row_bf16(sm + C_UTL, t, 32 * ch, u, 1.f);
            store_row_split(sm + C_GUH, sm + C_GUL, t, 32 * ch, u, gq);
            fence_proxy_async_smem();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (j + 1 < n) mbar_arrive(smem_u32(&ctl->bar_u));
            mbar_arrive(smem_u32(&ctl->empty[st]));
          }
        }
      }
    }
  } else if (want_o && warp < 10) {
    // ------------------------------------------------------------- O warps
    // warps 8, 9 (TMEM lanes 0-63): O_c = D rows 0-63 (scaled, bf16).  Full chunks go out
    // by one TMA store from a double-buffered staging tile; the ragged last chunk by
    // per-row stores.  D[c % 2] is released to the issuer once read.
    const int q = warp & 3, t = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const float sc = p.scale;
    for (int j = 0; j < n; ++j) {
      // D[j % 2]'s (j / 2)-th use is complete (one barrier per buffer: these warps may
      // trail the chain by up to two chunks)
      const bool got = mbar_wait(smem_u32(&ctl->bar_dO[j & 1]), (uint32_t)(j >> 1) & 1u, ab);
      if (bar_or_n(4, 64, !got)) break;
      tc_fence_after();
      const uint32_t dcol = tmem + 64 * (j & 1) + lane_base;
      float v0[32], v1[32];
      tmem_ld32(dcol + c_lo, v0);
      if (SPL == 1) tmem_ld32(dcol + 32, v1);
      tc_wait_ld();
      // staging buffer j % 2 was last read by the store of chunk j - 2
      if (warp == 8 && lane == 0) bulk_wait_read<1>();
      tc_fence_before();
      bar_sync_n(4, 64);
      if (warp == 8 && lane == 0) mbar_arrive(smem_u32(&ctl->bar_o[j & 1]));
      const int tok0 = t_begin + C * j;
      if (SPL > 1) {
        // half a tile's columns: row stores (a tile store would cover the other CTA's half)
        if (tok0 + t < t_end) {
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.o) +
                                                 (size_t)(tok0 + t) * p.o_stride +
                                                 (size_t)head * p.dv + slice * DVS + c_lo);
#pragma unroll
          for (int w = 0; w < 4; ++w)
            dst[w] = make_uint4(pack_bf16x2(v0[8 * w] * sc, v0[8 * w + 1] * sc),
                                pack_bf16x2(v0[8 * w + 2] * sc, v0[8 * w + 3] * sc),
                                pack_bf16x2(v0[8 * w + 4] * sc, v0[8 * w + 5] * sc),
                                pack_bf16x2(v0[8 * w + 6] * sc, v0[8 * w + 7] * sc));
        }
      } else if (tok0 + C <= t_end) {
        uint8_t *stg = sm + C_MTL + 8192 * (j & 1);
        store_row_bf16(stg, t, 0, v0, sc);
        store_row_bf16(stg, t, 32, v1, sc);
        fence_proxy_async_smem();
        bar_sync_n(4, 64);
        if (warp == 8 && lane == 0) {
          tma_store_2d(&tm_o, smem_u32(stg), head * p.dv + slice * DVS, tok0);
          bulk_commit();
        }
      } else if (tok0 + t < t_end) {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.o) +
                                               (size_t)(tok0 + t) * p.o_stride +
                                               (size_t)head * p.dv + slice * DVS);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          dst[w] = make_uint4(pack_bf16x2(v0[8 * w] * sc, v0[8 * w + 1] * sc),
                              pack_bf16x2(v0[8 * w + 2] * sc, v0[8 * w + 3] * sc),
                              pack_bf16x2(v0[8 * w + 4] * sc, v0[8 * w + 5] * sc),
                              pack_bf16x2(v0[8 * w + 6] * sc, v0[8 * w + 7] * sc));
          dst[4 + w] = make_uint4(pack_bf16x2(v1[8 * w] * sc, v1[8 * w + 1] * sc),
                                  pack_bf16x2(v1[8 * w + 2] * sc, v1[8 * w + 3] * sc),
                                  pack_bf16x2(v1[8 * w + 4] * sc, v1[8 * w + 5] * sc),
                                  pack_bf16x2(v1[8 * w + 6] * sc, v1[8 * w + 7] * sc));
        }
      }
    }
    // the outputs are in global memory before the kernel ends
    if (warp == 8 && lane == 0) bulk_wait<0>();
  }

  // a CTA that gave up a wait leaves no copy or product in flight behind it
  __syncwarp();
  const bool aborted = *ab.flag != 0;
  if (warp == 0 && lane == 0 && aborted)
    for (int b = 0; b < 2; ++b) {
      if (last_m[b] >= 0) mbar_wait_drain(smem_u32(&ctl->full_m[b]), (uint32_t)(last_m[b] >> 1) & 1u);
      if (last_k[b] >= 0) mbar_wait_drain(smem_u32(&ctl->full[b]), (uint32_t)(last_k[b] >> 1) & 1u);
    }
  if (warp == 1 && lane == 0 && aborted && mma_pending) {
    tc_commit(smem_u32(&ctl->drain));
    mbar_wait_drain(smem_u32(&ctl->drain), 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void __launch_bounds__(kChainThreads, 1)
    scan_chain_kernel(const __grid_constant__ ScanMaps mp, const __grid_constant__ ScanLaunch p,
                      const __grid_constant__ ScanWs ws, const __grid_constant__ ScanPlan plan) {
  chain_body<1>(mp, p, ws, plan, blockIdx.x, false);
}

// ===================================================== prep beside chain
// For few chains (a long sequence's heads: the latency-bound case) the chains run in the
// same launch as the prep, on their own CTAs, each stage waiting for its slots' flags, so
// the chain starts with the first chunks instead of after the last.  When the prep is the
// longer part (many heads, long tails) the chain CTAs first help with it for a few rounds
// (the shared rounds: every CTA of the grid takes one item per round), then run their
// chains on the chunks those rounds prepared.  The launch is
// cooperative: every CTA is resident at once, so a chain never waits on a prep CTA that
// cannot be scheduled.  CTAs [0, n_chain) run chains, the rest (warps 0-7) the prep.
template <int DV, int SPL>
__global__ void __launch_bounds__(kChainThreads, 1)
    scan_fused_kernel(const __grid_constant__ ScanMaps mp, const __grid_constant__ ScanLaunch p,
                      const __grid_constant__ ScanWs ws, const __grid_constant__ ScanPlan plan,
                      int n_chain, int64_t shared_end) {
  const int b = (int)blockIdx.x, all = (int)gridDim.x;
  const bool chain = b < n_chain;
  // a chain CTA first takes its items of the shared rounds (when the prep is the longer
  // part: then the chain would only wait), then runs its chain (one call site of each body)
  if (threadIdx.x < kPrepThreads && (!chain || shared_end > 0))
    prep_body<DV>(mp, p, ws, plan,
                  PrepSched{shared_end, b, all, chain ? -1 : (int64_t)(b - n_chain),
                            all - n_chain},
                  true, !chain);
  if (chain) chain_body<SPL>(mp, p, ws, plan, b, true);
}

// Host-side plan for up to kParamSeqs sequences: chunk offsets and the longest-first order.
bool host_plan(const ScanLaunch &p, ScanPlan *pl) {
  pl->in_params = 0;
  if (p.n_seqs > kParamSeqs) return false;
  int acc = 0;
  int nch[kParamSeqs];
  for (int i = 0; i < p.n_seqs; ++i) {
    pl->cu_chunks[i] = acc;
    pl->cu_tokens[i] = p.cu_seqlens_host[i];
    nch[i] = (p.cu_seqlens_host[i + 1] - p.cu_seqlens_host[i] + C - 1) / C;
    acc += nch[i];
  }
  pl->cu_chunks[p.n_seqs] = acc;
  pl->cu_tokens[p.n_seqs] = p.cu_seqlens_host[p.n_seqs];
  std::iota(pl->order, pl->order + p.n_seqs, 0);
  std::stable_sort(pl->order, pl->order + p.n_seqs,
                   [&](int a, int b) { return nch[a] > nch[b]; });
  pl->in_params = 1;
  return true;
}

}  // namespace

bool make_tmap_f32_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                      std::string *err);

// The fused launch serves few chains (at most kFusedMaxChains CTAs, leaving most SMs to the
// prep) of a plan that travels in the launch.
constexpr int kFusedMaxChains = 96;
constexpr int kSplitMaxChains = 64;
int64_t fused_chains(const ScanLaunch &p) { return (int64_t)p.n_seqs * p.H * (p.dv / DVS); }
bool use_fused(const ScanLaunch &p, int sms) {
  const int64_t n = fused_chains(p);
  return p.n_seqs <= kParamSeqs && n > 0 && n <= kFusedMaxChains && sms - n >= 32 &&
         count_chunks(p) > 0;
}
constexpr size_t FUSED_SMEM = PREP_SMEM > CHAIN_SMEM ? PREP_SMEM : CHAIN_SMEM;

bool scan_chunked_supported(const ScanLaunch &p) {
  return p.dtype == TR_DTYPE_BF16 && p.dk == DK && (p.dv == 64 || p.dv == 128) &&
         (p.o == nullptr || p.o_stride % 8 == 0);
}

size_t scan_chunked_workspace(const ScanLaunch &p) {
  size_t total = 0;
  ws_layout(p, nullptr, &total);
  return total;
}

std::vector<const char *> scan_chunked_kernel_names(const ScanLaunch &p, bool with_readout) {
  (void)with_readout;   // the readout is part of the chain kernel
  if (use_fused(p, device_sm_count())) return {"scan_fused"};
  if (p.n_seqs > kParamSeqs) return {"scan_plan", "scan_prep", "scan_chain"};
  return {"scan_prep", "scan_chain"};
}

cudaError_t launch_scan_chunked(const ScanLaunch &p, cudaStream_t s, std::string *err,
                                const std::function<cudaError_t()> &between) {
  if (p.n_seqs == 0) return cudaSuccess;
  if (p.precise_state && p.o) {
    if (err) *err = "the precise-state chain produces no readout";
    return cudaErrorInvalidValue;
  }
  size_t total = 0;
  ScanWs ws = ws_layout(p, p.ws, &total);
  if (total > p.ws_bytes || (total > 0 && !p.ws)) {
    if (err) *err = "scan workspace too small";
    return cudaErrorInvalidValue;
  }
  const int64_t items = ws.slots;
  if (items * 128 > 0x7fffffffLL) {
    if (err) *err = "too many (chunk, head) work items";
    return cudaErrorInvalidValue;
  }
  const int64_t ctas = (int64_t)p.n_seqs * p.H * (p.dv / DVS);
  if (ctas > 0x7fffffffLL) {
    if (err) *err = "too many (sequence, head) pairs";
    return cudaErrorInvalidValue;
  }
  const uint64_t T = (uint64_t)(p.T > 0 ? p.T : 1);
  const uint64_t slots = (uint64_t)(items > 0 ? items : 1);
  ScanMaps mp;
  const void *qb = p.q ? p.q : p.k;
  if (!make_tmap_bf16_2d(&mp.k, p.k, (uint64_t)p.H * DK, T, (uint64_t)p.k_stride * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&mp.q, qb, (uint64_t)p.H * DK, T,
                         (uint64_t)(p.q ? p.q_stride : p.k_stride) * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&mp.v, p.v, (uint64_t)p.H * p.dv, T, (uint64_t)p.v_stride * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&mp.QW, ws.QW, 128, slots * 128, 256, 64, 64, err) ||
      !make_tmap_bf16_2d(&mp.PY, ws.PY, 64, slots * 128, 128, 64, 64, err) ||
      !make_tmap_bf16_2d(&mp.KT, (p.flags & TR_NORMALIZE_QK) ? (const void *)ws.KT : p.k, 128,
                         (p.flags & TR_NORMALIZE_QK) ? slots * 64 : 1, 256, 64, 64, err) ||
      !make_tmap_f32_2d(&mp.UT, ws.UT, (uint64_t)p.dv, slots * 64, (uint64_t)p.dv * 4, 32, 64, err))
    return cudaErrorInvalidValue;
  // the readout o [T, H d_v] (token stride o_stride), stored in 64 x 64 boxes
  if (p.o && !make_tmap_bf16_2d(&mp.o, p.o, (uint64_t)p.H * p.dv, T, (uint64_t)p.o_stride * 2,
                                64, C, err))
    return cudaErrorInvalidValue;
  if (!p.o) mp.o = mp.k;
  ScanPlan plan{};
  cudaError_t e;
  const int sms = device_sm_count();
  // the fused launch's ready flags carry a per-call epoch, which a captured graph would
  // replay unchanged: under stream capture the prep and the chain run as separate kernels
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const bool capturing = cudaStreamIsCapturing(s, &cs) == cudaSuccess &&
                         cs != cudaStreamCaptureStatusNone;
  if (!capturing && use_fused(p, sms)) {
    // chains and prep in one cooperative launch (all CTAs resident at once)
    ScanLaunch pf = p;
    static std::atomic<unsigned long long> epoch_counter{0};
    pf.epoch = ++epoch_counter;
    host_plan(pf, &plan);
    const int grid = sms;
    // Shared rounds R: the chains start after R item-rounds on all SMs, the prep then goes
    // on on the other SMs.  Costs in units of a chain step: a prep item about 5.3 steps
    // (measured: ~14.7k against ~2.8k cycles); R minimises the later of the two ends.
    // few chains: two CTAs per 64-column tile, each carrying 32 state columns (half the
    // epilogue work on the chain's critical path; the prep keeps at least 84 SMs)
    const bool split = !p.precise_state && 2 * fused_chains(p) <= kSplitMaxChains;
    const int64_t n_chain = fused_chains(p) * (split ? 2 : 1), pc = grid - n_chain;
    int64_t longest = 0;
    for (int i = 0; i < p.n_seqs; ++i)
      longest = std::max<int64_t>(longest, (p.cu_seqlens_host[i + 1] - p.cu_seqlens_host[i] + C - 1) / C);
    constexpr double kItem = 5.3, kStep = 1.0;
    int64_t best_r = 0;
    double best_t = 1e300;
    for (int64_t r = 0; r * grid <= items + grid; ++r) {
      const int64_t rest = std::max<int64_t>(0, items - r * grid);
      const double prep = kItem * (double)(r + (rest + pc - 1) / pc);
      const double chain = kItem * (double)(r + 1) + kStep * (double)(longest + 1);
      const double t = std::max(prep, chain);
      if (t < best_t - 1e-9) {
        best_t = t;
        best_r = r;
      }
    }
    const int64_t shared_end = std::min<int64_t>(best_r * grid, items);
    auto kern = pf.dv == 128 ? (split ? scan_fused_kernel<128, 2> : scan_fused_kernel<128, 1>)
                             : (split ? scan_fused_kernel<64, 2> : scan_fused_kernel<64, 1>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FUSED_SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kChainThreads);
    cfg.dynamicSmemBytes = FUSED_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pf.pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, mp, pf, ws, plan, (int)n_chain, shared_end);
    if (e == cudaSuccess || !pf.pdl) return e;
    // a runtime that will not combine a cooperative launch with programmatic serialization:
    // the same launch without the latter
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mp, pf, ws, plan, (int)n_chain, shared_end);
  }
  if (!host_plan(p, &plan)) {
    e = launch_kernel(scan_plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, p.pdl, p.cu_seqlens,
                      p.n_seqs, ws.cu_chunks, ws.order);
    if (e != cudaSuccess) return e;
    if (between) {
      e = between();
      if (e != cudaSuccess) return e;
    }
  }
  if (items > 0) {
    int64_t grid = sms;
    if (grid > items) grid = items;
    auto kern = p.dv == 128 ? scan_prep_kernel<128> : scan_prep_kernel<64>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREP_SMEM);
    if (e != cudaSuccess) return e;
    e = launch_kernel(kern, dim3((unsigned)grid), dim3(kPrepThreads), PREP_SMEM, s, p.pdl, mp, p,
                      ws, plan);
    if (e != cudaSuccess) return e;
  }
  if (between) {
    e = between();
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(scan_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)CHAIN_SMEM);
  if (e != cudaSuccess) return e;
  return launch_kernel(scan_chain_kernel, dim3((unsigned)ctas), dim3(kChainThreads), CHAIN_SMEM,
                       s, p.pdl, mp, p, ws, plan);
}

}  // namespace tr
