// gemm_tc.cu -- the two projection GEMMs of an LA layer on the 5th-generation
// tensor cores (tcgen05 + TMEM), fed by TMA:
//
//   input projection  : [q|k|v|a_alpha|a_beta] = x_hat W_in^T, with the per-head
//                       L2 norm of q and k, -softplus / sigmoid gates, bf16 q/k/v
//   output projection : x <- x + o W_o^T (fp32 residual stream)
//   FFN gate/up       : h = bf16(silu(x_hat W_gate^T) * (x_hat W_up^T)); a 256-column
//                       tile holds 128 gate and the same 128 up columns (two B loads)
//
// C[M, N] = A[M, K] * B[N, K]^T, A and B bf16 with K contiguous (K-major).
// One persistent CTA per SM walks the output tiles (128 x BN).  Warp roles:
//   warp 0     TMA producer: 4-6 stage ring of (A 128x64, B BNx64) bf16 tiles,
//              128-byte swizzled, one mbarrier pair per stage
//   warp 1     TMEM owner + MMA issuer: one thread issues tcgen05.mma
//              (M=128, N=BN, K=16) into a double-buffered fp32 accumulator in
//              TMEM and commits each stage back to the producer
//   warps 2-9  epilogue: two warps per 32-lane quarter of the accumulator, each taking
//              half of the tile's columns: tcgen05.ld, fused activation/residual,
//              stores; overlaps the next tile's MMAs
// Every mbarrier wait is bounded (see tr_ptx.cuh); a timeout ends all roles of
// the CTA, frees its TMEM and raises the library's error word.
//
// Pair variant (the input projection): a cluster of two CTAs on two SMs computes a
// 256 x BN tile with tcgen05.mma.cta_group::2.  Each CTA loads its own 128 rows of A and
// its own BN / 2 rows of B (plain TMA loads, no multicast) into its shared memory, and
// those loads complete on the leader CTA's barrier; the leader's single thread issues the
// products (M = 256), whose completion is committed to both CTAs' barriers; each CTA's
// epilogue reads its 128 accumulator rows out of its own TMEM.  Per SM and k-block that
// is 32 KB of operands instead of 48 KB for a 128 x 256 tile: the L2-to-SM traffic that
// bounds the single-CTA tile drops by a third.
#include <cuda_bf16.h>

#include "tr_internal.h"
#include "tr_ptx.cuh"

namespace tr {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;

enum { EPI_INPROJ = 0, EPI_RESID = 1, EPI_SWIGLU = 2 };

template <int BN>
struct Cfg {
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  // as many stages as fit next to the control block (at most 6)
  static constexpr int STAGES = (200 * 1024 / STAGE_BYTES) < 6 ? (200 * 1024 / STAGE_BYTES) : 6;
  static constexpr uint32_t TMEM_COLS = BN <= 128 ? 2 * BN : 512;  // double buffer, power of 2
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
};

struct Ctl {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16 *dst, const float (&v)[32], float s) {
  uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int w = 0; w < 4; ++w)
    d[w] = make_uint4(pack_bf16x2(v[8 * w + 0] * s, v[8 * w + 1] * s),
                      pack_bf16x2(v[8 * w + 2] * s, v[8 * w + 3] * s),
                      pack_bf16x2(v[8 * w + 4] * s, v[8 * w + 5] * s),
                      pack_bf16x2(v[8 * w + 6] * s, v[8 * w + 7] * s));
}

// softplus(a) = max(a, 0) + ln(1 + e^{-|a|}) (no overflow for any a); when e^{-|a|} is
// below fp32 resolution the log term is dropped, an absolute error below 6e-8.
__device__ __forceinline__ float softplus_f(float a) {
  return fmaxf(a, 0.f) + log_ftz(1.f + exp_ftz(-fabsf(a)));
}
__device__ __forceinline__ float sigmoid_f(float a) { return 1.f / (1.f + exp_ftz(-a)); }

// Input-projection epilogue for tile columns [lo, hi) of one 128 x BN tile (lo, hi multiples
// of d_k); this thread owns `row`.
template <int BN>
__device__ __forceinline__ void epi_inproj(const InProjEpi &ep, uint32_t tbase, int n0, int N,
                                           int row, int M, int lo, int hi) {
  const int dk = ep.dk;
  const int nq = 2 * ep.H * dk;          // q and k features
  const int nv = nq + ep.H * ep.dv;      // end of the v features
  const int nz = nv + (ep.z ? ep.H * ep.dv : 0);  // end of the z features
  // the folded RMSNorm's 1/rms of this row (1 without it)
  float rs = 1.f;
  if (ep.ssq_part && row < M) {
    float ss = 0.f;
    for (int i = 0; i < ep.n_part; ++i) ss += ep.ssq_part[(int64_t)i * ep.part_ld + row];
    rs = rsqrtf(ss * ep.inv_d + ep.rms_eps);
  }
  for (int blk = lo / dk; blk < hi / dk; ++blk) {
    const int c0 = n0 + blk * dk;  // GEMM column
    if (c0 >= N) break;
    const int g0 = c0 + ep.col_offset;  // feature index in W_in
    const uint32_t tb = tbase + (uint32_t)(c0 - n0);
    if (g0 < nq) {
      // one q or k head: L2 norm over its d_k features (two passes over TMEM); raw when
      // a convolution comes first
      float inv = 1.f;
      if (!ep.raw_qk) {
        float ssq = 0.f;
        for (int j = 0; j < dk / 32; ++j) {
          float v[32];
          tmem_ld32(tb + 32 * j, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v[i] *= rs;
            ssq = fmaf(v[i], v[i], ssq);
          }
        }
        inv = rsqrtf(ssq + ep.norm_eps);
      }
      for (int j = 0; j < dk / 32; ++j) {
        float v[32];
        tmem_ld32(tb + 32 * j, v);
        tc_wait_ld();
        if (row < M) store_bf16x32(ep.qkv + (int64_t)row * ep.ldq + g0 + 32 * j, v, rs * inv);
      }
    } else {
      for (int j = 0; j < dk / 32; ++j) {
        const int c = c0 + 32 * j;
        if (c >= N) break;
        const int g = g0 + 32 * j;
        float v[32];
        tmem_ld32(tb + 32 * j, v);
        tc_wait_ld();
        if (row >= M) continue;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= rs;
        if (g + 32 <= nv) {
          store_bf16x32(ep.qkv + (int64_t)row * ep.ldq + g, v, 1.f);
        } else if (g + 32 <= nz) {
          store_bf16x32(ep.z + (int64_t)row * ep.H * ep.dv + (g - nv), v, 1.f);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int gi = g + i - nz;
            if (c + i >= N) break;
            if (gi < ep.H) {
              const float a = v[i] + (ep.dt_bias ? ep.dt_bias[gi] : 0.f);
              const float A = ep.A_log ? exp_ftz(ep.A_log[gi]) : 1.f;
              ep.log_alpha[(int64_t)row * ep.H + gi] = -A * softplus_f(a);
            } else if (gi < 2 * ep.H)
              ep.beta[(int64_t)row * ep.H + (gi - ep.H)] = sigmoid_f(v[i]);
          }
        }
      }
    }
  }
}

// 32 residual values of `row` at column c: fp32, or bf16 widened
struct Res32 {
  uint4 u[8];
};
__device__ __forceinline__ void load_res32(const ResidEpi &ep, int64_t row, int c, Res32 &r) {
  if (ep.res_is_bf16) {
    const uint4 *src = reinterpret_cast<const uint4 *>(
        reinterpret_cast<const __nv_bfloat16 *>(ep.x_res) + row * ep.ld + c);
#pragma unroll
    for (int w = 0; w < 4; ++w) r.u[w] = src[w];
  } else {
    const uint4 *src = reinterpret_cast<const uint4 *>(
        reinterpret_cast<const float *>(ep.x_res) + row * ep.ld + c);
#pragma unroll
    for (int w = 0; w < 8; ++w) r.u[w] = src[w];
  }
}
__device__ __forceinline__ void res32_to_f32(const ResidEpi &ep, const Res32 &r, float (&f)[32]) {
  if (ep.res_is_bf16) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r.u[w]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h[i]);
        f[8 * w + 2 * i] = t.x;
        f[8 * w + 2 * i + 1] = t.y;
      }
    }
  } else {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      f[4 * w] = __uint_as_float(r.u[w].x);
      f[4 * w + 1] = __uint_as_float(r.u[w].y);
      f[4 * w + 2] = __uint_as_float(r.u[w].z);
      f[4 * w + 3] = __uint_as_float(r.u[w].w);
    }
  }
}

// Output-projection epilogue for tile columns [lo, hi) of one 128 x BN tile (multiples of
// 32); this thread owns `row`.  The residual of the next 32 columns is requested before
// the current ones are added, so one global-load latency is in flight behind every TMEM
// load.
template <int BN>
__device__ __forceinline__ void epi_resid(const ResidEpi &ep, uint32_t tbase, int n0, int N,
                                          int row, int M, int lo, int hi) {
  const bool live = row < M;
  Res32 cur, nxt;
  float ss = 0.f;   // the folded RMSNorm's partial sum of squares of this row
  if (live && n0 + lo < N) load_res32(ep, row, n0 + lo, cur);
#pragma unroll 1
  for (int j = lo / 32; j < hi / 32; ++j) {
    const int c = n0 + 32 * j;
    if (c >= N) break;
    if (live && j + 1 < hi / 32 && c + 32 < N) load_res32(ep, row, c + 32, nxt);
    float v[32];
    tmem_ld32(tbase + 32 * j, v);
    tc_wait_ld();
    if (live) {
      float r[32];
      res32_to_f32(ep, cur, r);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] += r[i];
      float4 *out = reinterpret_cast<float4 *>(ep.x_out + (int64_t)row * ep.ld + c);
#pragma unroll
      for (int w = 0; w < 8; ++w)
        out[w] = make_float4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]);
      if (ep.xhat_out) {
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
        if (ep.gain) {
          const float4 *gp = reinterpret_cast<const float4 *>(ep.gain + c);
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            const float4 g = gp[w];
            v[4 * w] *= g.x;
            v[4 * w + 1] *= g.y;
            v[4 * w + 2] *= g.z;
            v[4 * w + 3] *= g.w;
          }
        }
        store_bf16x32(ep.xhat_out + (int64_t)row * ep.ld + c, v, 1.f);
      }
    }
    cur = nxt;
  }
  // one partial per (row, column group), written even when the group holds no column
  if (ep.xhat_out && live) ep.ssq_part[(int64_t)((n0 + lo) / (BN / 2)) * ep.part_ld + row] = ss;
}

// FFN epilogue for one tile of 128 gate (TMEM columns 0-127) and 128 up columns
// (128-255): half `half` of the warps takes outputs 64 half .. +63.
__device__ __forceinline__ void epi_swiglu(const SwigluEpi &ep, uint32_t tbase, int n0, int row,
                                           int M, int half) {
#pragma unroll 1
  for (int j = 0; j < 2; ++j) {
    const int c = 64 * half + 32 * j;  // output column within the tile
    float g[32], u[32];
    tmem_ld32(tbase + c, g);
    tmem_ld32(tbase + 128 + c, u);
    tc_wait_ld();
    if (row >= M) continue;
#pragma unroll
    for (int i = 0; i < 32; ++i) g[i] = g[i] / (1.f + exp_ftz(-g[i])) * u[i];
    store_bf16x32(ep.h + (int64_t)row * ep.ld + n0 + c, g, 1.f);
  }
}

// Work units: tiles [0, whole) run whole; each later tile (a partial last wave) runs as two
// units of BN / 2 columns (half the B bytes per k-block, so the last wave ends sooner).
__device__ __forceinline__ void unit_tile(int u, int whole, int &tile, int &half) {
  if (u < whole) {
    tile = u;
    half = -1;
  } else {
    tile = whole + (u - whole) / 2;
    half = (u - whole) % 2;
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB2, int M, int N, int K,
                        InProjEpi ip, ResidEpi rs, SwigluEpi sw, int whole,
                        unsigned *err_word) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  Ctl *ctl = reinterpret_cast<Ctl *>(smem + C::STAGES * C::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (M + BM - 1) / BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int n_total = m_tiles * n_tiles;
  // units: the whole tiles, then two half-width units per remaining tile (whole == n_total:
  // none split; the half units load B through tmB2, whose box is BN / 2 rows)
  const int n_units = whole + 2 * (n_total - whole);
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->tfull[b]), 1);
      mbar_init(smem_u32(&ctl->tempty[b]), kEpiWarps);
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (EPI == EPI_SWIGLU) tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const AbortFlag ab{&ctl->abort, err_word, ERRBIT_GEMM_TIMEOUT};
  // TMEM is held: the next kernel may start launching; the inputs are the previous
  // kernel's outputs, so wait for it before the first load
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        int t, hf;
        unit_tile(u, whole, t, hf);
        const int tm = t % m_tiles, tn = t / m_tiles;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(smem_u32(&ctl->empty[stage]), ph ^ 1u, ab)) goto producer_done;
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t fb = smem_u32(&ctl->full[stage]);
          mbar_arrive_expect_tx(fb, hf < 0 ? C::STAGE_BYTES : C::A_BYTES + C::B_BYTES / 2);
          tma_load_2d(sa, &tmA, kb * BK, tm * BM, fb);
          if (EPI == EPI_SWIGLU) {  // gate rows, then the same up rows
            tma_load_2d(sa + C::A_BYTES, &tmB, kb * BK, tn * (BN / 2), fb);
            tma_load_2d(sa + C::A_BYTES + C::B_BYTES / 2, &tmB2, kb * BK, tn * (BN / 2), fb);
          } else if (hf < 0) {
            tma_load_2d(sa + C::A_BYTES, &tmB, kb * BK, tn * BN, fb);
          } else {
            tma_load_2d(sa + C::A_BYTES, &tmB2, kb * BK, tn * BN + hf * (BN / 2), fb);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_full = idesc_bf16(BM, BN, 0, 0);
      constexpr uint32_t idesc_half = idesc_bf16(BM, BN / 2, 0, 0);
      int stage = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int un = blockIdx.x; un < n_units; un += gridDim.x, ++it) {
        int t, hf;
        unit_tile(un, whole, t, hf);
        (void)t;
        const uint32_t idesc = hf < 0 ? idesc_full : idesc_half;
        const int b = it & 1;
        const uint32_t u = (uint32_t)(it >> 1);
        if (!mbar_wait(smem_u32(&ctl->tempty[b]), (u & 1u) ^ 1u, ab)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(smem_u32(&ctl->full[stage]), ph, ab)) goto mma_done;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          // descriptors built once per stage; K step kk adds 32 bytes (2 units of 16)
          const uint64_t ad0 = sw128_desc(sa, 16, 1024);
          const uint64_t bd0 = sw128_desc(sa + C::A_BYTES, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_bf16(d, ad0 + 2u * kk, bd0 + 2u * kk, idesc, (kb | kk) ? 1u : 0u);
          tc_commit(smem_u32(&ctl->empty[stage]));
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        tc_commit(smem_u32(&ctl->tfull[b]));
      }
    mma_done:;
    }
  } else {
    const int q4 = warp & 3;  // TMEM lanes this warp may read: 32*q4 .. 32*q4+31
    const int half = (warp - 2) >> 2;  // which half of the tile's columns
    static_assert(BN % 64 == 0, "half tiles of whole 32-column groups");
    const int lo = half * (BN / 2), hi = lo + BN / 2;
    int it = 0;
    for (int un = blockIdx.x; un < n_units; un += gridDim.x, ++it) {
      int t, hf;
      unit_tile(un, whole, t, hf);
      const int b = it & 1;
      const uint32_t u = (uint32_t)(it >> 1);
      if (!mbar_wait(smem_u32(&ctl->tfull[b]), u & 1u, ab)) break;
      tc_fence_after();
      const int tm = t % m_tiles, tn = t / m_tiles;
      const int row = tm * BM + q4 * 32 + lane;
      const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(b * BN);
      // a half unit's BN / 2 columns sit at the accumulator's start: the warps of the first
      // column half take them all, the others have none
      const int n0 = tn * BN + (hf < 0 ? 0 : hf * (BN / 2));
      const bool any = hf < 0 || half == 0;
      const int ulo = hf < 0 ? lo : 0, uhi = hf < 0 ? hi : BN / 2;
      if (!any) {
      } else if (EPI == EPI_INPROJ)
        epi_inproj<BN>(ip, tbase, n0, N, row, M, ulo, uhi);
      else if (EPI == EPI_SWIGLU)
        epi_swiglu(sw, tbase, tn * (BN / 2), row, M, half);
      else
        epi_resid<BN>(rs, tbase, n0, N, row, M, ulo, uhi);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->tempty[b]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA pairs
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of `addr` (a shared::cta address) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Arrive on an mbarrier of either CTA of the cluster (a shared::cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
// Tiled TMA load into this CTA's shared memory whose transaction count completes on an
// mbarrier of either CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *tm, int32_t x,
                                                 int32_t y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.cta_group::2"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
// D[tmem] (+)= A * B^T over the pair: M = 256 (128 rows of A in each CTA), N columns (N / 2
// rows of B in each CTA), operands at the same shared-memory offsets in both CTAs.
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at shared offset `bar` in both CTAs of the pair when every
// product issued so far by this thread is done.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

template <int BN>
struct PairCfg {
  static constexpr uint32_t A_BYTES = BM * BK * 2;            // this CTA's 128 rows
  static constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;      // this CTA's BN / 2 rows
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024 / STAGE_BYTES) < 8 ? (200 * 1024 / STAGE_BYTES) : 8;
  static constexpr uint32_t TMEM_COLS = BN <= 128 ? 2 * BN : 512;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
};

// Units as in the single-CTA kernel, over pair tiles (256 x BN); a half unit is 256 x BN / 2.
template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, int M, int N, int K,
                     InProjEpi ip, ResidEpi rs, int whole, unsigned *err_word) {
  using C = PairCfg<BN>;
  static_assert(EPI != EPI_SWIGLU, "the pair kernel has no SwiGLU operand split");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  Ctl *ctl = reinterpret_cast<Ctl *>(smem + C::STAGES * C::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int m_tiles = (M + 2 * BM - 1) / (2 * BM);
  const int n_tiles = (N + BN - 1) / BN;
  const int n_total = m_tiles * n_tiles;
  const int n_units = whole + 2 * (n_total - whole);
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);    // the leader's: its expect-tx arrival
      mbar_init(smem_u32(&ctl->empty[s]), 1);   // the leader's commit, in both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->tfull[b]), 1);                // the leader's commit
      mbar_init(smem_u32(&ctl->tempty[b]), 2 * kEpiWarps);   // both CTAs' epilogue warps
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ctl->tmem_base)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  // both CTAs' barriers are initialised before either CTA's loads or arrivals reach them
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const AbortFlag ab{&ctl->abort, err_word, ERRBIT_GEMM_TIMEOUT};
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      for (int u = pair; u < n_units; u += n_pairs) {
        int t, hf;
        unit_tile(u, whole, t, hf);
        const int tm = t % m_tiles, tn = t / m_tiles;
        const int row_a = tm * 2 * BM + (int)rank * BM;
        // this CTA's rows of B: half of the tile's (or of the half unit's) columns
        const int row_b = hf < 0 ? tn * BN + (int)rank * (BN / 2)
                                 : tn * BN + hf * (BN / 2) + (int)rank * (BN / 4);
        const uint32_t pair_bytes = 2u * (hf < 0 ? C::STAGE_BYTES : C::A_BYTES + C::B_BYTES / 2);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(smem_u32(&ctl->empty[stage]), ph ^ 1u, ab)) goto producer_done;
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t fb = cluster_map(smem_u32(&ctl->full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&ctl->full[stage]), pair_bytes);
          tma_load_2d_pair(sa, &tmA, kb * BK, row_a, fb);
          tma_load_2d_pair(sa + C::A_BYTES, hf < 0 ? &tmB : &tmB2, kb * BK, row_b, fb);
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t idesc_full = idesc_bf16(2 * BM, BN, 0, 0);
      constexpr uint32_t idesc_half = idesc_bf16(2 * BM, BN / 2, 0, 0);
      int stage = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int un = pair; un < n_units; un += n_pairs, ++it) {
        int t, hf;
        unit_tile(un, whole, t, hf);
        (void)t;
        const uint32_t idesc = hf < 0 ? idesc_full : idesc_half;
        const int b = it & 1;
        const uint32_t u = (uint32_t)(it >> 1);
        if (!mbar_wait(smem_u32(&ctl->tempty[b]), (u & 1u) ^ 1u, ab)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(smem_u32(&ctl->full[stage]), ph, ab)) goto mma_done;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint64_t ad0 = sw128_desc(sa, 16, 1024);
          const uint64_t bd0 = sw128_desc(sa + C::A_BYTES, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_pair(d, ad0 + 2u * kk, bd0 + 2u * kk, idesc, (kb | kk) ? 1u : 0u);
          tc_commit_pair(smem_u32(&ctl->empty[stage]));
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        tc_commit_pair(smem_u32(&ctl->tfull[b]));
      }
    mma_done:;
    }
  } else {
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;
    static_assert(BN % 64 == 0, "half tiles of whole 32-column groups");
    const int lo = half * (BN / 2), hi = lo + BN / 2;
    const uint32_t tempty0 = cluster_map(smem_u32(&ctl->tempty[0]), 0);
    const uint32_t tempty1 = cluster_map(smem_u32(&ctl->tempty[1]), 0);
    int it = 0;
    for (int un = pair; un < n_units; un += n_pairs, ++it) {
      int t, hf;
      unit_tile(un, whole, t, hf);
      const int b = it & 1;
      const uint32_t u = (uint32_t)(it >> 1);
      if (!mbar_wait(smem_u32(&ctl->tfull[b]), u & 1u, ab)) break;
      tc_fence_after();
      const int tm = t % m_tiles, tn = t / m_tiles;
      const int row = tm * 2 * BM + (int)rank * BM + q4 * 32 + lane;
      const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(b * BN);
      const int n0 = tn * BN + (hf < 0 ? 0 : hf * (BN / 2));
      const bool any = hf < 0 || half == 0;
      const int ulo = hf < 0 ? lo : 0, uhi = hf < 0 ? hi : BN / 2;
      if (!any) {
      } else if (EPI == EPI_INPROJ)
        epi_inproj<BN>(ip, tbase, n0, N, row, M, ulo, uhi);
      else
        epi_resid<BN>(rs, tbase, n0, N, row, M, ulo, uhi);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(b ? tempty1 : tempty0);
    }
  }

  // no CTA leaves while its peer may still signal its barriers or read its operands
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS));
  }
}

// N counts the tile's output columns; for the FFN gate/up product N = 2 d_ff, B = W_gate
// and B2 = W_up ([d_ff, K] each).
template <int BN, int EPI>
cudaError_t launch(const void *A, int64_t lda, const void *B, const void *B2, int M, int N, int K,
                   const InProjEpi &ip, const ResidEpi &rs, const SwigluEpi &sw,
                   unsigned *err_word, cudaStream_t s, bool pdl, std::string *err) {
  using C = Cfg<BN>;
  if (M <= 0 || N <= 0) return cudaSuccess;
  CUtensorMap ta, tb, tb2;
  if (EPI == EPI_SWIGLU) {
    if (!make_tmap_bf16_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK, BM, err) ||
        !make_tmap_bf16_2d(&tb, B, (uint64_t)K, (uint64_t)(N / 2), (uint64_t)K * 2, BK, BN / 2,
                           err) ||
        !make_tmap_bf16_2d(&tb2, B2, (uint64_t)K, (uint64_t)(N / 2), (uint64_t)K * 2, BK, BN / 2,
                           err))
      return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_bf16_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK, BM, err) ||
        !make_tmap_bf16_2d(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN, err))
      return cudaErrorInvalidValue;
    tb2 = tb;
    // the half-width tail units load BN / 2 rows of B
    if (EPI == EPI_INPROJ &&
        !make_tmap_bf16_2d(&tb2, B, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN / 2, err))
      return cudaErrorInvalidValue;
  }
  auto kern = gemm_bf16_tn_kernel<BN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  int grid = device_sm_count();
  if (grid > tiles) grid = tiles;
  // the input projection's partial last wave: its tiles split into two half-width units
  // when twice as many still fit in one round
  int whole = tiles;
  if (EPI == EPI_INPROJ && grid > 0) {
    const int rest = tiles % grid;
    if (tiles > grid && rest > 0 && 2 * rest <= grid) whole = tiles - rest;
  }
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kThreads), C::SMEM, s, pdl, ta, tb, tb2, M,
                       N, K, ip, rs, sw, whole, err_word);
}

// The pair kernel: clusters of two CTAs, as many as can be resident at once (each needs two
// SMs of one TPC); tiles of 256 x BN, a partial last round as 256 x BN / 2 half units.
template <int BN, int EPI>
cudaError_t launch_pair(const void *A, int64_t lda, const void *B, int M, int N, int K,
                        const InProjEpi &ip, const ResidEpi &rs, unsigned *err_word,
                        cudaStream_t s, bool pdl, std::string *err) {
  using C = PairCfg<BN>;
  if (M <= 0 || N <= 0) return cudaSuccess;
  CUtensorMap ta, tb, tb2;
  if (!make_tmap_bf16_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK, BM, err) ||
      !make_tmap_bf16_2d(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN / 2, err) ||
      !make_tmap_bf16_2d(&tb2, B, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN / 4, err))
    return cudaErrorInvalidValue;
  auto kern = gemm_pair_kernel<BN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  // resident pairs (queried once per device; the SM count halved if the query fails)
  constexpr int kDevices = 64;
  static int resident[kDevices] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  int pairs = device_sm_count() / 2;
  if (dev >= 0 && dev < kDevices) {
    if (resident[dev] == 0) {
      cfg.gridDim = dim3((unsigned)(2 * pairs));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0)
        resident[dev] = n;
      else
        resident[dev] = pairs;
      cudaGetLastError();
    }
    pairs = resident[dev] < pairs ? resident[dev] : pairs;
  }
  const int tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + BN - 1) / BN);
  if (pairs > tiles) pairs = tiles;
  int whole = tiles;
  const int rest = tiles % pairs;
  if (tiles > pairs && rest > 0 && 2 * rest <= pairs) whole = tiles - rest;
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, tb2, M, N, K, ip, rs, whole, err_word);
}

}  // namespace

// The residual GEMM's tiles (launch<192, EPI_RESID>) are 192 columns wide, each half taken
// by its own epilogue warps: one partial sum of squares per row and half tile, the last
// tile's halves included even where they hold no column
int resid_ssq_partials(int N) { return 2 * ((N + 191) / 192); }

cudaError_t launch_gemm_inproj(const void *A, const void *B, int M, int N, int K,
                               const InProjEpi &ep, unsigned *err_word, cudaStream_t s,
                               bool pdl, std::string *err) {
  ResidEpi none{};
  SwigluEpi no_sw{};
  // more than one 128-row tile: 256-row tiles on CTA pairs
  if (M > BM) return launch_pair<256, EPI_INPROJ>(A, K, B, M, N, K, ep, none, err_word, s, pdl, err);
  return launch<256, EPI_INPROJ>(A, K, B, nullptr, M, N, K, ep, none, no_sw, err_word, s, pdl, err);
}

cudaError_t launch_gemm_resid(const void *A, int64_t lda, const void *B, int M, int N, int K,
                              const ResidEpi &ep, unsigned *err_word, cudaStream_t s, bool pdl,
                              std::string *err) {
  InProjEpi none{};
  // 192-column tiles: the output is narrow (d_model), so 128 x 256 tiles would leave SMs
  // idle and N = 128 MMAs are issue-bound; d_model 2048 gives 11 x 13 = 143 tiles, one wave
  SwigluEpi no_sw{};
  return launch<192, EPI_RESID>(A, lda, B, nullptr, M, N, K, none, ep, no_sw, err_word, s, pdl, err);
}

cudaError_t launch_gemm_swiglu(const void *A, const void *W_gate, const void *W_up, int M, int d_ff,
                               int K, const SwigluEpi &ep, unsigned *err_word, cudaStream_t s,
                               bool pdl, std::string *err) {
  InProjEpi no_ip{};
  ResidEpi no_rs{};
  return launch<256, EPI_SWIGLU>(A, K, W_gate, W_up, M, 2 * d_ff, K, no_ip, no_rs, ep, err_word, s,
                                 pdl, err);
}

}  // namespace tr
