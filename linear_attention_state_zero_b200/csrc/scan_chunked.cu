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
// Nothing but the transition and the readout depends on M_0, so the work splits in
// three launches:
//
//   scan_prep_kernel   persistent over all (chunk, head) items, in parallel:
//     P1  [K; Q] K^T -> TMEM            (tcgen05, K-major operands)
//     A, P on CUDA cores; T = (I + A)^{-1} by blocked forward substitution in fp32
//     P2  [-T''; T'] [V | K] -> -U~, W  (T' = T diag(beta gamma), T'' = T diag(beta))
//     P3  P W, P U~, K^T (gamma' W), K^T (gamma' U~) in one batch
//     -> workspace, by TMA stores: A_c (bf16), R (bf16), B_c (fp32), O0 (fp32), gamma_C
//   scan_chain_kernel  one CTA per (sequence, head, 64-column slice of d_v), sequential
//     over the chunks: one tcgen05 product Z = A_c M_bf16 per chunk, then
//     M <- gamma_C M + Z + B_c in fp32 registers; the bf16 chunk-start states go to the
//     workspace.  Operands arrive by TMA, double-buffered one chunk ahead.
//   scan_out_kernel    one CTA per (chunk, head), in parallel: o = R M_c + O0.
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

// --------------------------------------------------------------- helpers
// Shared-memory descriptors are built once per operand (sw128_desc) and advanced
// per K step by adding to the 16-byte start-address field only.
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
  __nv_bfloat16 *M;  // [slots][128][dv]   bf16 state at the chunk start (chain -> readout)
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
  const size_t oM = off; off = align256(off + S * 128 * (size_t)p.dv * 2);
  if (total) *total = off;
  uint8_t *b = static_cast<uint8_t *>(base);
  if (b) {
    w.A = reinterpret_cast<__nv_bfloat16 *>(b + oA);
    w.R = reinterpret_cast<__nv_bfloat16 *>(b + oR);
    w.B = reinterpret_cast<float *>(b + oB);
    w.O = reinterpret_cast<float *>(b + oO);
    w.G = reinterpret_cast<float *>(b + oG);
    w.M = reinterpret_cast<__nv_bfloat16 *>(b + oM);
  }
  return w;
}

// ============================================================ prep kernel
// 256 threads, persistent over work items (slot order: chunk-major, head-minor), with
// the next items' K/Q/V tiles prefetched by TMA into a second buffer.
// shared memory (bytes from a 1024-aligned base):
constexpr uint32_t P_IN = 0;          // 2 x 48 KB: [KQ 32 KB: half x (K rows 0-63 | Q rows 64-127)][V 16 KB]
constexpr uint32_t P_IN_BYTES = 49152;
constexpr uint32_t P_AP = 98304;      // 128 x 64 bf16: rows 0-63 zero, 64-127 = P
constexpr uint32_t P_TSH = 114688;    // [-T''; T'] high bf16 parts   (after P2: gamma' U~ high)
constexpr uint32_t P_TSL = 131072;    // [-T''; T'] low bf16 parts    (after P2: gamma' U~ low)
constexpr uint32_t P_AW = 147456;     // A fp32 [64][68] during the inverse; then W (16 KB) + gamma' W
constexpr uint32_t P_TU = 180224;     // T fp32 [64][68] + X fp32 [32][36]; then U~ high + U~ low
constexpr uint32_t P_END = 212992;
constexpr int LDA = 68;               // fp32 row stride of A and T (16-byte aligned rows)
constexpr int LDX = 36;
constexpr size_t PREP_SMEM = P_END + 1024 + 1024;
constexpr int kPrepThreads = 256;
constexpr int kMaxSeqsChunked = 1024;

struct PrepCtl {
  uint64_t tma_bar[2];
  uint64_t mma_bar;
  uint32_t tmem;
  int abort;
  float g[C];      // inclusive cumsum of log alpha over the chunk
  float beta[C];
  float bg[C];     // beta * gamma
  int cu_chunks[kMaxSeqsChunked + 1];
  int cu_tok[kMaxSeqsChunked + 1];  // the sequence offsets (cu_seqlens)
};

// hi + lo bf16 split of 32 values (v[i] * s) into two 128-byte-row swizzled tiles.
__device__ __forceinline__ void store_row_split(uint8_t *hi, uint8_t *lo, int row, int col0,
                                                const float *v, float s) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = v[8 * w + 2 * i] * s, b = v[8 * w + 2 * i + 1] * s;
      const __nv_bfloat162 hh = __floats2bfloat162_rn(a, b);
      const float2 hf = __bfloat1622float2(hh);
      const __nv_bfloat162 ll = __floats2bfloat162_rn(a - hf.x, b - hf.y);
      h[i] = *reinterpret_cast<const uint32_t *>(&hh);
      l[i] = *reinterpret_cast<const uint32_t *>(&ll);
    }
    const uint32_t off = sw128_offset((uint32_t)row, (uint32_t)(col0 + 8 * w) * 2u);
    st_shared_v4(smem_u32(hi + off), h[0], h[1], h[2], h[3]);
    st_shared_v4(smem_u32(lo + off), l[0], l[1], l[2], l[3]);
  }
}

// Output staging after the last product of an item (every region below is free by then;
// each tile is 128-byte swizzled, one TMA box):
//   A_c  [2 halves][128 rows][64 bf16]  at P_TU
//   B_c  [DV/32 boxes][128 rows][32 fp32] at P_TSH (spans TSH, TSL, AW)
//   R    [2 halves][64 rows][64 bf16]   at P_AP
//   O0   [DV/32 boxes][64 rows][32 fp32] in the item's input buffer, over the K rows and V
//        (the Q rows stay intact: R reads them)
__device__ __forceinline__ uint32_t o0_box_offset(int b) {
  return b < 2 ? (uint32_t)b * 16384u : 32768u + (uint32_t)(b - 2) * 8192u;
}

// The prep work of one CTA: items first, then second, second + stride, ... (256 threads;
// every barrier is the named barrier 1 over those threads).
template <int DV>
__device__ __forceinline__ void prep_body(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                          const CUtensorMap &tm_v, const CUtensorMap &tm_A,
                                          const CUtensorMap &tm_B, const CUtensorMap &tm_R,
                                          const CUtensorMap &tm_O, const ScanLaunch &p,
                                          const ScanWs &ws, int total_chunks, int64_t first,
                                          int64_t second, int64_t stride) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ PrepCtl ctl_s;
  PrepCtl *ctl = &ctl_s;
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  float *As = reinterpret_cast<float *>(sm + P_AW);
  float *Ts = reinterpret_cast<float *>(sm + P_TU);
  float *Xs = Ts + C * LDA;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, hsel = warp >> 2;   // TMEM lane quarter, column half
  const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
  const int row = q4 * 32 + lane;              // TMEM lane = row of a 128-row result
  const int H = p.H;
  const bool want_o = p.o != nullptr;
  const int64_t n_items = (int64_t)total_chunks * H;

  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_A);
    tma_prefetch_desc(&tm_B);
    tma_prefetch_desc(&tm_R);
    tma_prefetch_desc(&tm_O);
    mbar_init(smem_u32(&ctl->tma_bar[0]), 1);
    mbar_init(smem_u32(&ctl->tma_bar[1]), 1);
    mbar_init(smem_u32(&ctl->mma_bar), 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl->tmem), 512);
    tmem_relinquish();
  }
  for (int i = tid; i < 8192 / 16; i += kPrepThreads) st_shared_v4(smem_u32(sm + P_AP) + 16 * i, 0, 0, 0, 0);
  if (!want_o)
    for (int i = tid; i < 4 * 8192 / 16; i += kPrepThreads) {
      const int blk = i >> 9;  // (buffer, half)
      st_shared_v4(smem_u32(sm + P_IN + (blk >> 1) * P_IN_BYTES + (blk & 1) * 16384 + 8192) +
                       16 * (i & 511), 0, 0, 0, 0);
    }
  tc_fence_before();
  bar_sync_n(1, kPrepThreads);
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const AbortFlag ab{&ctl->abort, p.err_word, ERRBIT_SCAN_TIMEOUT};
  // TMEM is held: let the next kernel launch; then wait for the previous one's outputs
  pdl_trigger();
  pdl_wait();
  // first chunk of every sequence
  if (tid == 0) {
    int acc = 0;
    for (int i = 0; i < p.n_seqs; ++i) {
      ctl->cu_chunks[i] = acc;
      acc += (p.cu_seqlens[i + 1] - p.cu_seqlens[i] + C - 1) / C;
    }
    ctl->cu_chunks[p.n_seqs] = acc;
  }
  for (int i = tid; i <= p.n_seqs; i += kPrepThreads) ctl->cu_tok[i] = p.cu_seqlens[i];
  bar_sync_n(1, kPrepThreads);

  // (sequence, chunk) of an item
  auto locate = [&](int64_t item, int &seq, int &cc) {
    const int chunk = (int)(item / H);
    int lo = 0, hi = p.n_seqs - 1;
    while (lo < hi) {  // last sequence whose first chunk is <= chunk
      const int mid = (lo + hi + 1) >> 1;
      if (ctl->cu_chunks[mid] <= chunk) lo = mid; else hi = mid - 1;
    }
    seq = lo;
    cc = chunk - ctl->cu_chunks[lo];
  };
  auto issue = [&](int64_t item, int buf) {
    int seq, cc;
    locate(item, seq, cc);
    const int head = (int)(item % H);
    const int t0 = ctl->cu_tok[seq] + cc * C;
    const uint32_t bar = smem_u32(&ctl->tma_bar[buf]);
    const uint32_t kq = smem_u32(sm + P_IN + buf * P_IN_BYTES);
    mbar_arrive_expect_tx(bar, 16384u + (want_o ? 16384u : 0u) + (uint32_t)DV * 128u);
    tma_load_2d(kq, &tm_k, head * DK, t0, bar);
    tma_load_2d(kq + 16384, &tm_k, head * DK + 64, t0, bar);
    if (want_o) {
      tma_load_2d(kq + 8192, &tm_q, head * DK, t0, bar);
      tma_load_2d(kq + 16384 + 8192, &tm_q, head * DK + 64, t0, bar);
    }
#pragma unroll
    for (int b = 0; b < DV / 64; ++b)
      tma_load_2d(kq + 32768 + 8192 * b, &tm_v, head * DV + 64 * b, t0, bar);
  };
  if (tid == 0) {
    fence_proxy_async_smem();
    if (first < n_items) issue(first, 0);
    if (second < n_items) issue(second, 1);
  }
  // log alpha and beta of an item's 64 tokens (thread tid < C: token tid; 0 past the end)
  auto load_gates = [&](int64_t it, float &la, float &b) {
    int sq, cq;
    locate(it, sq, cq);
    const int hd = (int)(it % H);
    const int tt = ctl->cu_tok[sq] + cq * C;
    la = 0.f;
    b = 0.f;
    if (tid < min(C, ctl->cu_tok[sq + 1] - tt)) {
      la = p.log_alpha[(size_t)(tt + tid) * H + hd];
      b = p.beta[(size_t)(tt + tid) * H + hd];
    }
  };
  // the next item's gates are loaded during the current item
  float la_next = 0.f, b_next = 0.f;
  if (tid < C && first < n_items) load_gates(first, la_next, b_next);
  auto next_item = [&](int64_t it) -> int64_t { return it == first ? second : it + stride; };
  const uint32_t mma_bar = smem_u32(&ctl->mma_bar);
  uint32_t mma_phase = 0;
  auto mma_wait = [&]() -> bool {
    const bool ok = mbar_wait(mma_bar, mma_phase, ab);
    mma_phase ^= 1u;
    if (bar_or_n(1, kPrepThreads, !ok)) return false;
    tc_fence_after();
    return true;
  };

  int n = 0;
  for (int64_t item = first; item < n_items; item = next_item(item), ++n) {
    const int buf = n & 1;
    uint8_t *KQ = sm + P_IN + buf * P_IN_BYTES;
    const uint32_t kq_u = smem_u32(KQ);
    const uint32_t v_u = kq_u + 32768;

    // gates: g = inclusive cumsum of log alpha (0 past the end), beta, beta * gamma
    if (tid < C) {
      const float la = la_next, b = b_next;
      if (next_item(item) < n_items) load_gates(next_item(item), la_next, b_next);
      float s = la;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      ctl->g[tid] = s;
      ctl->beta[tid] = b;
    }
    bar_sync_n(1, kPrepThreads);
    if (tid >= 32 && tid < C) ctl->g[tid] += ctl->g[31];
    bar_sync_n(1, kPrepThreads);
    if (tid < C) ctl->bg[tid] = ctl->beta[tid] * exp_ftz(ctl->g[tid]);
    const bool ok_tma = mbar_wait(smem_u32(&ctl->tma_bar[buf]), (uint32_t)(n >> 1) & 1u, ab);
    if (bar_or_n(1, kPrepThreads, !ok_tma)) break;
    if (p.flags & TR_NORMALIZE_QK) {
      if (tid < C || (tid < 2 * C && want_o)) normalize_row(KQ, tid);
      fence_proxy_async_smem();
      bar_sync_n(1, kPrepThreads);
    }

    // P1: [K; Q] K^T -> TMEM cols [0, 64)
    if (tid == 0) {
      tc_fence_after();
      const uint64_t dkq = kmaj(kq_u);
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk)
        tc_mma_bf16(tmem, desc_k(dkq, kk, 16384), desc_k(dkq, kk, 16384),
                    idesc_bf16(128, 64, 0, 0), kk > 0);
      tc_commit(mma_bar);
      // the previous item's output stores of R and B_c boxes 2, 3 must have read their
      // staging before the A/P phase overwrites it (all threads pass the barrier in
      // mma_wait after this); A_c and B_c boxes 0, 1 are waited for before the inverse
      bulk_wait_read<1>();
    }
    if (!mma_wait()) break;

    // A (strictly lower, fp32) and P (lower incl. diagonal, bf16); columns split by hsel
    {
      float v[32];
      tmem_ld32(tmem + lane_base + 32 * hsel, v);
      tc_wait_ld();
      const int t = row & 63;
      const float gt = ctl->g[t];
      if (row < C) {
        const float bt = ctl->beta[t];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int s = 32 * hsel + i;
          v[i] = (s < t) ? bt * exp_ftz(gt - ctl->g[s]) * v[i] : 0.f;
        }
        float4 *dst = reinterpret_cast<float4 *>(As + t * LDA + 32 * hsel);
#pragma unroll
        for (int w = 0; w < 8; ++w) dst[w] = make_float4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]);
      } else if (want_o) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int s = 32 * hsel + i;
          v[i] = (s <= t) ? exp_ftz(gt - ctl->g[s]) * v[i] : 0.f;
        }
        store_row_bf16(sm + P_AP, row, 32 * hsel, v, 1.f);
      }
    }
    if (tid == 0) {
      bulk_wait_read<0>();  // the staging of A_c, B_c boxes 0, 1 is free
      // the previous item's input buffer (its K/Q/V, then its O0 staging) is free now:
      // prefetch the next item into it (items 0 and 1 were loaded before the loop)
      if (n >= 1 && next_item(item) < n_items) {
        fence_proxy_async_smem();
        issue(next_item(item), buf ^ 1);
      }
    }
    bar_sync_n(1, kPrepThreads);

    // T = (I + A)^{-1}, blocked.  (a) the four 16 x 16 diagonal blocks by forward
    // substitution (thread = column, fp32 registers); (b) each 32 x 32 diagonal block from
    // its two 16-blocks: T21 = -T22 (A21 T11); (c) the 64 x 64 from the two 32-blocks the
    // same way.
    if (tid < C) {
      const int base = 16 * (tid >> 4), c = tid & 15;
      float Tc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // row i of the block's A (16-byte aligned), 4 at a time; entries at columns >= i
        // are zeros of the strictly lower A and are skipped
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
    }
    bar_sync_n(1, kPrepThreads);
    // (b) thread -> 32-block J, row r of its lower 16 x 16 block, columns c0, c0 + 1
    const int mJ = tid >> 7, mr = (tid >> 3) & 15, mc = (tid & 7) * 2;
    {  // X16 = A21 T11 within block J
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
      // the upper-right 16 x 16 of the 32-block is zero (T is lower triangular); nothing
      // in this step reads it
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
    {  // X = A21 T11 (32 x 32): thread -> row r, columns c0..c0+3
      const int r = tid >> 3, c0 = (tid & 7) * 4;
      float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
      const float *Ar = As + (32 + r) * LDA;
#pragma unroll 4
      for (int s = 0; s < 32; s += 4) {
        const float4 a = *reinterpret_cast<const float4 *>(Ar + s);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 t = *reinterpret_cast<const float4 *>(Ts + (s + u) * LDA + c0);
          x0 = fmaf(av[u], t.x, x0); x1 = fmaf(av[u], t.y, x1);
          x2 = fmaf(av[u], t.z, x2); x3 = fmaf(av[u], t.w, x3);
        }
      }
      *reinterpret_cast<float4 *>(Xs + r * LDX + c0) = make_float4(x0, x1, x2, x3);
    }
    bar_sync_n(1, kPrepThreads);
    {  // T21 = -T22 X
      const int r = tid >> 3, c0 = (tid & 7) * 4;
      float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
      const float *Tr = Ts + (32 + r) * LDA + 32;
#pragma unroll 4
      for (int s = 0; s < 32; s += 4) {
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
    bar_sync_n(1, kPrepThreads);
    {  // [-T diag(beta); T diag(beta gamma)] as high + low bf16 parts; consecutive lanes
       // take consecutive rows (conflict-free reads of T and swizzled stores)
      const int rr = tid & 127, half = tid >> 7, t = rr & 63;
      const bool zero = t < 32 && half == 1;  // T is lower triangular: T12 = 0
      float v[32];
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float4 tv = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                               : *reinterpret_cast<const float4 *>(Ts + t * LDA + 32 * half + 4 * w);
        const float te[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = 32 * half + 4 * w + u;
          v[4 * w + u] = (rr < C) ? -te[u] * ctl->beta[s] : te[u] * ctl->bg[s];
        }
      }
      store_row_split(sm + P_TSH, sm + P_TSL, rr, 32 * half, v, 1.f);
    }
    fence_proxy_async_smem();
    bar_sync_n(1, kPrepThreads);

    // P2: [-T''; T'] V -> cols [64, 64+DV) (lanes 0-63: -U~); [-T''; T'] K -> [192, 320) (lanes 64-127: W)
    if (tid == 0) {
      tc_fence_after();
      const uint64_t th = kmaj(smem_u32(sm + P_TSH)), tl = kmaj(smem_u32(sm + P_TSL));
      const uint64_t dv_ = mnmaj(v_u, 8192), dk_ = mnmaj(kq_u, 16384);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 64, desc_k(th, kk, 0), desc_mn(dv_, kk), idesc_bf16(128, DV, 0, 1), kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 64, desc_k(tl, kk, 0), desc_mn(dv_, kk), idesc_bf16(128, DV, 0, 1), 1u);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 192, desc_k(th, kk, 0), desc_mn(dk_, kk), idesc_bf16(128, 128, 0, 1), kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 192, desc_k(tl, kk, 0), desc_mn(dk_, kk), idesc_bf16(128, 128, 0, 1), 1u);
      tc_commit(mma_bar);
    }
    if (!mma_wait()) break;

    const float gC = ctl->g[C - 1];
    {
      float v[32];
      const int t = row & 63;
      const float gp = exp_ftz(gC - ctl->g[t]);
      if (row >= C) {  // W row t, columns 64*hsel..+63 -> W and gamma' W ([t][d], 8 KB halves)
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          tmem_ld32(tmem + 192 + lane_base + 64 * hsel + 32 * j, v);
          tc_wait_ld();
          store_row_bf16(sm + P_AW + hsel * 8192, t, 32 * j, v, 1.f);
          store_row_bf16(sm + P_AW + 16384 + hsel * 8192, t, 32 * j, v, gp);
        }
      } else {  // -U~ row t, columns (DV/2)*hsel.. -> U~ (hi, lo) and gamma' U~ (hi, lo)
#pragma unroll 1
        for (int j = 0; j < DV / 64; ++j) {
          const int col = (DV / 2) * hsel + 32 * j;
          tmem_ld32(tmem + 64 + lane_base + col, v);
          tc_wait_ld();
          const int blkoff = (col >> 6) * 8192, c0 = col & 63;
          store_row_split(sm + P_TU + blkoff, sm + P_TU + 16384 + blkoff, t, c0, v, -1.f);
          store_row_split(sm + P_TSH + blkoff, sm + P_TSL + blkoff, t, c0, v, -gp);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    bar_sync_n(1, kPrepThreads);

    // batch: P W -> [0,128), P U~ -> [128,128+DV), A_c -> [256,384), B_c -> [384,384+DV)
    if (tid == 0) {
      tc_fence_after();
      const uint64_t ap = kmaj(smem_u32(sm + P_AP));
      const uint32_t w_u = smem_u32(sm + P_AW), uh_u = smem_u32(sm + P_TU);
      const uint64_t w_d = mnmaj(w_u, 8192), wg_d = mnmaj(w_u + 16384, 8192);
      const uint64_t uh = mnmaj(uh_u, 8192), ul = mnmaj(uh_u + 16384, 8192);
      const uint64_t gh = mnmaj(smem_u32(sm + P_TSH), 8192), gl = mnmaj(smem_u32(sm + P_TSL), 8192);
      const uint64_t kt = mnmaj(kq_u, 16384);
      if (want_o) {
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(tmem + 0, desc_k(ap, kk, 0), desc_mn(w_d, kk), idesc_bf16(128, 128, 0, 1), kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(tmem + 128, desc_k(ap, kk, 0), desc_mn(uh, kk), idesc_bf16(128, DV, 0, 1), kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          tc_mma_bf16(tmem + 128, desc_k(ap, kk, 0), desc_mn(ul, kk), idesc_bf16(128, DV, 0, 1), 1u);
      }
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 256, desc_mn(kt, kk), desc_mn(wg_d, kk), idesc_bf16(128, 128, 1, 1), kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 384, desc_mn(kt, kk), desc_mn(gh, kk), idesc_bf16(128, DV, 1, 1), kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        tc_mma_bf16(tmem + 384, desc_mn(kt, kk), desc_mn(gl, kk), idesc_bf16(128, DV, 1, 1), 1u);
      tc_commit(mma_bar);
    }
    if (!mma_wait()) break;

    {
      float v[32];
      // A_c row d = -(K^T gamma' W)[d] (bf16), columns 64*hsel..+63
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        tmem_ld32(tmem + 256 + lane_base + 64 * hsel + 32 * j, v);
        tc_wait_ld();
        store_row_bf16(sm + P_TU + hsel * 16384, row, 32 * j, v, -1.f);
      }
      // B_c row d (fp32), columns (DV/2)*hsel.. (one 32-column box per 32 columns)
#pragma unroll 1
      for (int j = 0; j < DV / 64; ++j) {
        tmem_ld32(tmem + 384 + lane_base + (DV / 2) * hsel + 32 * j, v);
        tc_wait_ld();
        store_row32_f32(sm + P_TSH + 16384 * (((DV / 2) * hsel + 32 * j) >> 5), row, v, 1.f);
      }
      if (want_o && row >= C) {
        const int t = row - C;
        const float gam = exp_ftz(ctl->g[t]);
        // R row t = gamma_t q_t - (P W)_t (bf16), columns 64*hsel..+63
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          tmem_ld32(tmem + 0 + lane_base + 64 * hsel + 32 * j, v);
          tc_wait_ld();
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            float f[8];
            load_row8_bf16(KQ + hsel * 16384, 64 + t, 32 * j + 8 * w, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[8 * w + i] = gam * f[i] - v[8 * w + i];
          }
          store_row_bf16(sm + P_AP + hsel * 8192, t, 32 * j, v, 1.f);
        }
        // O0 row t (fp32), columns (DV/2)*hsel..
#pragma unroll 1
        for (int j = 0; j < DV / 64; ++j) {
          tmem_ld32(tmem + 128 + lane_base + (DV / 2) * hsel + 32 * j, v);
          tc_wait_ld();
          store_row32_f32(KQ + o0_box_offset(((DV / 2) * hsel + 32 * j) >> 5), t, v, 1.f);
        }
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    bar_sync_n(1, kPrepThreads);
    if (tid == 0) {
      const int64_t slot = item;
      // three bulk groups, in the order the staging tiles are needed again:
      //   1. O0 (this item's input buffer: the prefetch below refills it)
      //   2. R (P_AP) and B_c boxes 2, 3 (P_AW): the next item's A/P phase writes there
      //   3. A_c (P_TU) and B_c boxes 0, 1 (P_TSH, P_TSL): its inverse and split write there
      if (want_o) {
#pragma unroll
        for (int b = 0; b < DV / 32; ++b)
          tma_store_2d(&tm_O, smem_u32(KQ + o0_box_offset(b)), 32 * b, (int32_t)(slot * 64));
      }
      bulk_commit();
      if (want_o) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tma_store_2d(&tm_R, smem_u32(sm + P_AP + h * 8192), 64 * h, (int32_t)(slot * 64));
      }
#pragma unroll
      for (int b = 2; b < DV / 32; ++b)
        tma_store_2d(&tm_B, smem_u32(sm + P_TSH + 16384 * b), 32 * b, (int32_t)(slot * 128));
      bulk_commit();
#pragma unroll
      for (int h = 0; h < 2; ++h)
        tma_store_2d(&tm_A, smem_u32(sm + P_TU + h * 16384), 64 * h, (int32_t)(slot * 128));
#pragma unroll
      for (int b = 0; b < 2; ++b)
        tma_store_2d(&tm_B, smem_u32(sm + P_TSH + 16384 * b), 32 * b, (int32_t)(slot * 128));
      bulk_commit();
      ws.G[slot] = exp_ftz(gC);
    }
  }

  if (tid == 0) bulk_wait<0>();
  tc_fence_before();
  bar_sync_n(1, kPrepThreads);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DV>
__global__ void __launch_bounds__(kPrepThreads, 1)
    scan_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_A,
                     const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_R,
                     const __grid_constant__ CUtensorMap tm_O, const __grid_constant__ ScanLaunch p,
                     const __grid_constant__ ScanWs ws, int total_chunks) {
  prep_body<DV>(tm_q, tm_k, tm_v, tm_A, tm_B, tm_R, tm_O, p, ws, total_chunks, blockIdx.x,
                (int64_t)blockIdx.x + gridDim.x, gridDim.x);
}

// =========================================================== chain kernel
// One CTA per (sequence, head, 64-column slice of d_v), 288 threads.  Warps 0-7:
// thread (quarter q4 = warp % 4, column group cg = warp / 4) owns row d = 32 q4 + lane
// of the fp32 state slice and its columns kCols cg .. +kCols-1 (the per-chunk update is
// latency-bound: 16 state warps with half the columns each measured no faster).  Warp 8
// only refills the TMA ring (a tensor load can stall its issuing thread while many are in flight, so the
// state-owning threads never issue them).  Per chunk: one tcgen05 product
// Z = A_c M (M in bf16 in shared memory, 8 MMAs of K = 16), then
// M <- gamma_C M + Z + B_c in registers.  A_c and the B_c slice arrive through a
// 2-stage TMA ring; all gamma_C of the sequence are read into shared memory at the
// start.  The bf16 state at the start of every chunk (double buffered by chunk
// parity) is the operand of the next product and goes to the workspace, for the
// readout kernel, by a TMA store.
constexpr int kStages = 2;
constexpr uint32_t H_STAGE = 65536;             // A_c [half][128 rows][128 B] + B_c [box][128][32 fp32]
constexpr uint32_t H_MB = kStages * H_STAGE;    // 2 x bf16 state slice [128 d][128 B]

struct ChainCtl {
  alignas(16) float g4[kStages][4];  // the 16-byte aligned group of G holding the stage's gamma_C
  uint64_t tma_bar[kStages];
  uint64_t empty_bar[kStages];  // stage consumed (arrived by thread 0 after the barrier)
  uint64_t bar_z;
  uint32_t tmem;
  int abort;
};
constexpr uint32_t H_CTL = H_MB + 2 * 16384;    // the control block, in dynamic shared memory
constexpr size_t CHAIN_SMEM = H_CTL + sizeof(ChainCtl) + 1024;

__device__ __forceinline__ void load_row32_f32(const uint8_t *tile, int row, float *f) {
  // one row (32 floats = 128 B) of a 128-byte-swizzled fp32 tile
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const float4 u = *reinterpret_cast<const float4 *>(
        tile + sw128_offset((uint32_t)row, (uint32_t)ch * 16u));
    f[4 * ch] = u.x; f[4 * ch + 1] = u.y; f[4 * ch + 2] = u.z; f[4 * ch + 3] = u.w;
  }
}

constexpr int kStateWarps = 8;
constexpr int kChainThreads = 32 * (kStateWarps + 1);
constexpr int kCols = DVS * 4 / kStateWarps;  // state columns per thread
static_assert(kCols == 32, "state columns per thread");



// The chain of one (sequence * H + head, slice) task (kChainThreads threads).  The
// loads of chunk c (A_c, the B_c slice and gamma_C, into stage c % kStages) are issued
// by the producer warp.
__device__ __forceinline__ void chain_body(const CUtensorMap &tm_A, const CUtensorMap &tm_B,
                                           const CUtensorMap &tm_M, const ScanLaunch &p,
                                           const ScanWs &ws, int seqhead, int slice) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int red[32];  // one entry per warp (chunk_base)
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  ChainCtl *ctl = reinterpret_cast<ChainCtl *>(sm + H_CTL);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, cg = warp >> 2;
  const int d = q4 * 32 + lane;
  const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
  const int H = p.H, DV = p.dv;
  const int seq = seqhead / H, head = seqhead % H;
  const int col = slice * DVS + kCols * cg;   // this thread's first d_v column

  if (tid == 0) {
    tma_prefetch_desc(&tm_A);
    tma_prefetch_desc(&tm_B);
    tma_prefetch_desc(&tm_M);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctl->tma_bar[s]), 1);
      mbar_init(smem_u32(&ctl->empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&ctl->bar_z), 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl->tmem), 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM is held: let the next kernel launch; then wait for the previous one's outputs
  pdl_trigger();
  pdl_wait();
  const int t_begin = p.cu_seqlens[seq], t_end = p.cu_seqlens[seq + 1];
  const int nch = (t_end - t_begin + C - 1) / C;
  const int cb = chunk_base(p.cu_seqlens, seq, red);
  auto slot_of = [&](int c) -> int64_t { return ((int64_t)cb + c) * H + head; };
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const AbortFlag ab{&ctl->abort, p.err_word, ERRBIT_SCAN_TIMEOUT};
  // bf16 state copy par (chunk parity) -> workspace slot of chunk c, by one TMA store
  auto store_mc = [&](int c, int par) {
    tma_store_2d(&tm_M, smem_u32(sm + H_MB + 16384 * par), slice * DVS, (int32_t)(slot_of(c) * 128));
    bulk_commit();
  };

  float Mr[kCols];
  const bool m_zero = p.S0 == nullptr;
  const bool producer = warp == kStateWarps;
  const size_t s_off = ((size_t)seq * H + head) * DK * DV + (size_t)d * DV + col;
  if (!m_zero && !producer) {
#pragma unroll
    for (int j = 0; j < kCols; j += 4) {
      const float4 a = *reinterpret_cast<const float4 *>(p.S0 + s_off + j);
      Mr[j] = a.x; Mr[j + 1] = a.y; Mr[j + 2] = a.z; Mr[j + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kCols; ++j) Mr[j] = 0.f;
  }
  auto store_state = [&](uint8_t *tile) { store_row_bf16(tile, d, kCols * cg, Mr, 1.f); };
  if (nch > 0 && !producer) store_state(sm + H_MB);

  auto issue_tma = [&](int c) {
    const int st = c % kStages;
    const int64_t slot = slot_of(c);
    const uint32_t bar = smem_u32(&ctl->tma_bar[st]);
    const uint32_t a_u = smem_u32(sm + st * H_STAGE);
    mbar_arrive_expect_tx(bar, 65536u + 16u);
    tma_load_2d(a_u, &tm_A, 0, (int32_t)(slot * 128), bar);
    tma_load_2d(a_u + 16384, &tm_A, 64, (int32_t)(slot * 128), bar);
    tma_load_2d(a_u + 32768, &tm_B, slice * DVS, (int32_t)(slot * 128), bar);
    tma_load_2d(a_u + 49152, &tm_B, slice * DVS + 32, (int32_t)(slot * 128), bar);
    // gamma_C: the 16-byte group of G that holds it (G is padded to 256 bytes)
    bulk_load(smem_u32(&ctl->g4[st][0]), ws.G + (slot & ~(int64_t)3), 16u, bar);
  };

  auto issue_mma = [&](int c) -> bool {
    const int st = c % kStages;
    if (!mbar_wait(smem_u32(&ctl->tma_bar[st]), (uint32_t)(c / kStages) & 1u, ab)) return false;
    tc_fence_after();
    const uint64_t ad = kmaj(smem_u32(sm + st * H_STAGE));
    const uint64_t md = mnmaj(smem_u32(sm + H_MB + 16384 * (c & 1)), 16384);
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk)
      tc_mma_bf16(tmem, desc_k(ad, kk, 16384), desc_mn(md, kk), idesc_bf16(128, DVS, 0, 1), kk > 0);
    tc_commit(smem_u32(&ctl->bar_z));
    return true;
  };

  bool failed = false;
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0 && nch > 0) store_mc(0, 0);

  if (producer) {
    // fill stage c % kStages with chunk c once chunk c - kStages has consumed it
    if (lane == 0) {
      for (int c = 0; c < nch; ++c) {
        const int st = c % kStages;
        if (c >= kStages &&
            !mbar_wait(smem_u32(&ctl->empty_bar[st]), (uint32_t)((c - kStages) / kStages) & 1u, ab))
          break;
        issue_tma(c);
      }
    }
  } else {
    if (tid == 0 && !m_zero && nch > 0 && !issue_mma(0)) failed = true;
    bool mma_for_c = !m_zero;
    uint32_t z_phase = 0;
    for (int c = 0; c < nch; ++c) {
      const int st = c % kStages;
      float v[kCols], b[kCols];
      if (mma_for_c) {
        if (!mbar_wait(smem_u32(&ctl->bar_z), z_phase, ab)) failed = true;
        z_phase ^= 1u;
        tc_fence_after();
        tmem_ld32(tmem + lane_base + kCols * cg, v);
      } else {
#pragma unroll
        for (int j = 0; j < kCols; ++j) v[j] = 0.f;
      }
      // the stage's B_c has landed (its A_c did, for the product); read this thread's
      // columns of row d from the 32-column box that holds them
      if (!mbar_wait(smem_u32(&ctl->tma_bar[st]), (uint32_t)(c / kStages) & 1u, ab)) failed = true;
      {
        const int c0 = kCols * cg;
        const uint8_t *bt = sm + st * H_STAGE + 32768 + (c0 >> 5) * 16384;
#pragma unroll
        for (int ch = 0; ch < kCols / 4; ++ch) {
          const float4 u = *reinterpret_cast<const float4 *>(
              bt + sw128_offset((uint32_t)d, (uint32_t)(((c0 & 31) >> 2) + ch) * 16u));
          b[4 * ch] = u.x; b[4 * ch + 1] = u.y; b[4 * ch + 2] = u.z; b[4 * ch + 3] = u.w;
        }
      }
      if (mma_for_c) tc_wait_ld();
      const float gC = ctl->g4[st][slot_of(c) & 3];
      // M <- gamma_C M + A_c M + B_c (fp32); bf16 copy for the next product and the readout
#pragma unroll
      for (int j = 0; j < kCols; ++j) Mr[j] = fmaf(gC, Mr[j], v[j] + b[j]);
      if (c + 1 < nch) store_state(sm + H_MB + 16384 * ((c + 1) & 1));
      fence_proxy_async_smem();
      tc_fence_before();
      // copy (c + 1) & 1 was last stored to global two chunks ago: that store must have
      // finished reading it before anyone rewrites it (after the barrier below)
      if (tid == 0) bulk_wait_read<0>();
      // named barrier over the state-owning threads, voting on `failed` so that all of
      // them leave the loop together
      uint32_t any_failed;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
          "bar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(any_failed)
          : "r"((uint32_t)(failed || *ab.flag)), "n"(32 * kStateWarps)
          : "memory");
      if (any_failed) { failed = true; break; }
      if (tid == 0) {
        // chunk c's stage is consumed: its product completed and its B_c rows were read
        mbar_arrive(smem_u32(&ctl->empty_bar[st]));
        if (c + 1 < nch) {
          tc_fence_after();
          if (!issue_mma(c + 1)) failed = true;
          store_mc(c + 1, (c + 1) & 1);
        }
      }
      mma_for_c = true;
    }
  }

  if (tid == 0) bulk_wait<0>();
  if (!failed && !producer) {
    float *dst = p.S_final + s_off;
#pragma unroll
    for (int j = 0; j < kCols; j += 4)
      *reinterpret_cast<float4 *>(dst + j) = make_float4(Mr[j], Mr[j + 1], Mr[j + 2], Mr[j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

__global__ void __launch_bounds__(kChainThreads, 1)
    scan_chain_kernel(const __grid_constant__ CUtensorMap tm_A, const __grid_constant__ CUtensorMap tm_B,
                      const __grid_constant__ CUtensorMap tm_M, const __grid_constant__ ScanLaunch p,
                      const __grid_constant__ ScanWs ws) {
  chain_body(tm_A, tm_B, tm_M, p, ws, blockIdx.x, blockIdx.y);
}

// ========================================================= readout kernel
// o_c = R_c M_c + O0_c for every (chunk, head) in parallel: one tcgen05 product
// ([R; unused rows] (128 x 128) times the bf16 chunk-start state M_c (128 x DV)),
// plus the fp32 O0, scaled and stored as bf16.  128 threads; thread t < 64 owns
// token row t.
constexpr uint32_t O_R = 0;          // [half][128 rows][128 B]: rows 0-63 = R
constexpr uint32_t O_M = 32768;      // [DV/64 blocks][128 d][128 B]: M_c
constexpr uint32_t O_O = 65536;      // [DV/32 boxes][64 rows][32 fp32]: O0
constexpr size_t OUT_SMEM = O_O + 32768 + 1024;

template <int DV>
__global__ void __launch_bounds__(128)
    scan_out_kernel(const __grid_constant__ CUtensorMap tm_R, const __grid_constant__ CUtensorMap tm_M,
                    const __grid_constant__ CUtensorMap tm_O, ScanLaunch p, ScanWs ws,
                    int total_chunks) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_t, bar_m;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  __shared__ int cu_chunks[kMaxSeqsChunked + 1];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H;
  const int64_t item = blockIdx.x;
  const int chunk = (int)(item / H), head = (int)(item % H);
  if (tid == 0) {
    tma_prefetch_desc(&tm_R);
    tma_prefetch_desc(&tm_M);
    tma_prefetch_desc(&tm_O);
    mbar_init(smem_u32(&bar_t), 1);
    mbar_init(smem_u32(&bar_m), 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_s), DV);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM is held: let the next kernel launch; then wait for the previous one's outputs
  pdl_trigger();
  pdl_wait();
  if (tid == 0) {
    int acc = 0;
    for (int i = 0; i < p.n_seqs; ++i) {
      cu_chunks[i] = acc;
      acc += (p.cu_seqlens[i + 1] - p.cu_seqlens[i] + C - 1) / C;
    }
    cu_chunks[p.n_seqs] = acc;
  }
  __syncthreads();
  const uint32_t tmem = tmem_s;
  const AbortFlag ab{&abort_s, p.err_word, ERRBIT_SCAN_TIMEOUT};
  int lo = 0, hi = p.n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu_chunks[mid] <= chunk) lo = mid; else hi = mid - 1;
  }
  const int seq = lo;
  const int t0 = p.cu_seqlens[seq] + (chunk - cu_chunks[seq]) * C;
  const int nv = min(C, p.cu_seqlens[seq + 1] - t0);
  if (tid == 0) {
    const uint32_t r_u = smem_u32(sm + O_R), m_u = smem_u32(sm + O_M);
    mbar_arrive_expect_tx(smem_u32(&bar_t), 16384u + (uint32_t)DV * 256u + (uint32_t)DV * 256u);
#pragma unroll
    for (int b = 0; b < DV / 32; ++b)
      tma_load_2d(smem_u32(sm + O_O) + 8192 * b, &tm_O, 32 * b, (int32_t)(item * 64), smem_u32(&bar_t));
    tma_load_2d(r_u, &tm_R, 0, (int32_t)(item * 64), smem_u32(&bar_t));
    tma_load_2d(r_u + 16384, &tm_R, 64, (int32_t)(item * 64), smem_u32(&bar_t));
#pragma unroll
    for (int b = 0; b < DV / 64; ++b)
      tma_load_2d(m_u + 16384 * b, &tm_M, 64 * b, (int32_t)(item * 128), smem_u32(&bar_t));
  }
  bool ok = mbar_wait(smem_u32(&bar_t), 0, ab);
  if (tid == 0 && ok) {
    tc_fence_after();
    const uint64_t rd = kmaj(smem_u32(sm + O_R)), md = mnmaj(smem_u32(sm + O_M), 16384);
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk)
      tc_mma_bf16(tmem, desc_k(rd, kk, 16384), desc_mn(md, kk), idesc_bf16(128, DV, 0, 1), kk > 0);
    tc_commit(smem_u32(&bar_m));
  }
  ok = ok && mbar_wait(smem_u32(&bar_m), 0, ab);
  if (__syncthreads_or(!ok)) {
    // a wait ran out: leave the outputs alone
  } else {
    tc_fence_after();
    if (tid < C) {
      const float sc = p.scale;
#pragma unroll 1
      for (int j = 0; j < DV / 32; ++j) {
        float v[32], b[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * j, v);
        load_row32_f32(sm + O_O + 8192 * j, tid, b);
        tc_wait_ld();
        if (tid < nv) {
          uint4 *d4 = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.o) +
                                                (size_t)(t0 + tid) * p.o_stride + (size_t)head * DV + 32 * j);
#pragma unroll
          for (int w = 0; w < 4; ++w)
            d4[w] = make_uint4(pack_bf16x2((v[8 * w] + b[8 * w]) * sc, (v[8 * w + 1] + b[8 * w + 1]) * sc),
                               pack_bf16x2((v[8 * w + 2] + b[8 * w + 2]) * sc, (v[8 * w + 3] + b[8 * w + 3]) * sc),
                               pack_bf16x2((v[8 * w + 4] + b[8 * w + 4]) * sc, (v[8 * w + 5] + b[8 * w + 5]) * sc),
                               pack_bf16x2((v[8 * w + 6] + b[8 * w + 6]) * sc, (v[8 * w + 7] + b[8 * w + 7]) * sc));
        }
      }
    }
  }
  (void)lane;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, DV);
  }
}

}  // namespace

bool make_tmap_f32_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                      std::string *err);

bool scan_chunked_supported(const ScanLaunch &p) {
  return p.dtype == TR_DTYPE_BF16 && p.dk == DK && (p.dv == 64 || p.dv == 128) &&
         p.n_seqs <= kMaxSeqsChunked && (p.o == nullptr || p.o_stride % 8 == 0);
}

size_t scan_chunked_workspace(const ScanLaunch &p) {
  size_t total = 0;
  ws_layout(p, nullptr, &total);
  return total;
}

std::vector<const char *> scan_chunked_kernel_names(const ScanLaunch &p, bool with_readout) {
  (void)p;
  if (with_readout) return {"scan_prep", "scan_chain", "scan_out"};
  return {"scan_prep", "scan_chain"};
}

cudaError_t launch_scan_chunked(const ScanLaunch &p, cudaStream_t s, std::string *err,
                                const std::function<cudaError_t()> &between) {
  if (p.n_seqs == 0) return cudaSuccess;
  size_t total = 0;
  ScanWs ws = ws_layout(p, p.ws, &total);
  if (total > p.ws_bytes || (total > 0 && !p.ws)) {
    if (err) *err = "scan workspace too small";
    return cudaErrorInvalidValue;
  }
  const int64_t items = ws.slots;
  const int total_chunks = (int)(items / p.H);
  if (items > 0x7fffffffLL) {
    if (err) *err = "too many (chunk, head) work items";
    return cudaErrorInvalidValue;
  }
  const uint64_t T = (uint64_t)(p.T > 0 ? p.T : 1);
  const uint64_t slots = (uint64_t)(items > 0 ? items : 1);
  CUtensorMap tq, tk, tv, tA, tR;
  const void *qb = p.q ? p.q : p.k;
  if (!make_tmap_bf16_2d(&tk, p.k, (uint64_t)p.H * DK, T, (uint64_t)p.k_stride * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&tq, qb, (uint64_t)p.H * DK, T,
                         (uint64_t)(p.q ? p.q_stride : p.k_stride) * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&tv, p.v, (uint64_t)p.H * p.dv, T, (uint64_t)p.v_stride * 2, 64, C, err) ||
      !make_tmap_bf16_2d(&tA, ws.A, 128, slots * 128, 256, 64, 128, err) ||
      !make_tmap_bf16_2d(&tR, ws.R, 128, slots * 64, 256, 64, 64, err))
    return cudaErrorInvalidValue;
  CUtensorMap tB, tM, tO;
  if (!make_tmap_f32_2d(&tB, ws.B, (uint64_t)p.dv, slots * 128, (uint64_t)p.dv * 4, 32, 128, err) ||
      !make_tmap_bf16_2d(&tM, ws.M, (uint64_t)p.dv, slots * 128, (uint64_t)p.dv * 2, 64, 128, err) ||
      !make_tmap_f32_2d(&tO, ws.O, (uint64_t)p.dv, slots * 64, (uint64_t)p.dv * 4, 32, 64, err))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (items > 0) {
    int64_t grid = device_sm_count();
    if (grid > items) grid = items;
    if (p.dv == 128) {
      e = cudaFuncSetAttribute(scan_prep_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)PREP_SMEM);
      if (e != cudaSuccess) return e;
      e = launch_kernel(scan_prep_kernel<128>, dim3((unsigned)grid), dim3(kPrepThreads), PREP_SMEM,
                        s, p.pdl, tq, tk, tv, tA, tB, tR, tO, p, ws, total_chunks);
    } else {
      e = cudaFuncSetAttribute(scan_prep_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)PREP_SMEM);
      if (e != cudaSuccess) return e;
      e = launch_kernel(scan_prep_kernel<64>, dim3((unsigned)grid), dim3(kPrepThreads), PREP_SMEM,
                        s, p.pdl, tq, tk, tv, tA, tB, tR, tO, p, ws, total_chunks);
    }
    if (e != cudaSuccess) return e;
  }
  if (between) {
    e = between();
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(scan_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)CHAIN_SMEM);
  if (e != cudaSuccess) return e;
  e = launch_kernel(scan_chain_kernel, dim3((unsigned)(p.n_seqs * p.H), (unsigned)(p.dv / DVS)),
                    dim3(kChainThreads), CHAIN_SMEM, s, p.pdl, tA, tB, tM, p, ws);
  if (e != cudaSuccess || !p.o || items == 0) return e;
  if (between) {
    e = between();
    if (e != cudaSuccess) return e;
  }
  if (p.dv == 128) {
    e = cudaFuncSetAttribute(scan_out_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)OUT_SMEM);
    if (e != cudaSuccess) return e;
    return launch_kernel(scan_out_kernel<128>, dim3((unsigned)items), dim3(128), OUT_SMEM, s, p.pdl,
                         tR, tM, tO, p, ws, total_chunks);
  } else {
    e = cudaFuncSetAttribute(scan_out_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)OUT_SMEM);
    if (e != cudaSuccess) return e;
    return launch_kernel(scan_out_kernel<64>, dim3((unsigned)items), dim3(128), OUT_SMEM, s, p.pdl,
                         tR, tM, tO, p, ws, total_chunks);
  }
}

}  // namespace tr
