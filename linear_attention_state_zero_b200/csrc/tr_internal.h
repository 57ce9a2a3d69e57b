// tr_internal.h -- host-side interfaces between the C ABI layer (tr_api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <functional>
#include <string>
#include <vector>

namespace tr {

// Device error word bits (OR-ed into the library's error word by the kernels).
enum : unsigned {
  ERRBIT_GEMM_TIMEOUT = 1u,
  ERRBIT_SCAN_TIMEOUT = 2u,
};

// Epilogue of the input projection: per-head L2 norm of q and k, bf16 q/k/v,
// gate activations in fp32.
struct InProjEpi {
  __nv_bfloat16 *qkv;  // [M, ldq] bf16
  int64_t ldq;         // 2 H d_k + H d_v
  float *log_alpha;    // [M, H]
  float *beta;         // [M, H]
  int H, dk, dv;
  int col_offset;      // W_in row that is GEMM column 0 (H d_k when q is skipped)
  float norm_eps;
  // optional Gated DeltaNet details (all zero / NULL: not used)
  int raw_qk;             // q, k stored without the L2 norm (a convolution follows)
  __nv_bfloat16 *z;       // [M, H d_v] bf16: the output gate's input, W_in rows after v
  const float *A_log;     // [H]: log alpha = -exp(A_log) softplus(a + dt_bias)
  const float *dt_bias;   // [H]
  // RMSNorm folded in (NULL: not used): A is bf16(x * gain) without the 1/rms factor, and
  // every output of row r is first multiplied by 1/sqrt(ss_r / d_model + rms_eps), ss_r the
  // sum of the row's n_part partial sums ssq_part[i * part_ld + r], added in order of i
  const float *ssq_part;
  int n_part;
  int64_t part_ld;
  float inv_d, rms_eps;
};

// Short causal depthwise convolution + silu over the bf16 q/k/v projections (zero history
// per sequence), then the per-head L2 norm of q and k, written as bf16 to `post`.
struct ShortConvLaunch {
  const __nv_bfloat16 *pre;  // [T, ld] bf16 (channels from col0 are read)
  __nv_bfloat16 *post;       // [T, ld] bf16
  int64_t ld;                // 2 H d_k + H d_v
  const float *w;            // [2 H d_k + H d_v, width] fp32
  int width;                 // 2..4
  const int32_t *cu_seqlens; // device [n_seqs + 1]
  int n_seqs;
  int64_t T;
  int H, dk, dv;
  int skip_q;                // q channels neither read nor written
  float norm_eps;
  __nv_bfloat16 *state;      // [n_seqs, width - 1, 2 H d_k + H d_v] bf16, or NULL
};

// Epilogue of the output projection: x_out = x_res + acc (fp32 out).
struct ResidEpi {
  const void *x_res;   // [M, ld] bf16 or fp32
  int res_is_bf16;
  float *x_out;        // [M, ld] fp32
  int64_t ld;
  // the next layer's RMSNorm, folded in (NULL: not used): bf16(x_out * gain) to xhat_out
  // [M, ld] and, per row, one partial sum of x_out^2 per column group (each half of a
  // 192-column tile; groups past N hold 0), group i to ssq_part[i * part_ld + row]
  __nv_bfloat16 *xhat_out;
  const float *gain;   // [ld] (NULL: 1)
  float *ssq_part;
  int64_t part_ld;
};

// Number of per-row partial sums of squares the residual GEMM writes for N columns.
int resid_ssq_partials(int N);

// Epilogue of the FFN's gate/up projection: h = bf16(silu(gate) * up).
struct SwigluEpi {
  __nv_bfloat16 *h;    // [M, ld] bf16
  int64_t ld;          // d_ff
};

struct ScanLaunch {
  int n_seqs, H, dk, dv;
  int64_t T;
  int dtype;           // TR_DTYPE_*
  unsigned flags;
  float scale;
  int64_t q_stride, k_stride, v_stride, o_stride;  // elements per token
  const void *q, *k, *v;
  const float *log_alpha, *beta;
  const int32_t *cu_seqlens;
  const int32_t *cu_seqlens_host;
  const float *S0;
  void *o;
  float *S_final;
  unsigned *err_word;
  void *ws;            // scan workspace (chunked kernels), ws_bytes long
  size_t ws_bytes;
  bool pdl;            // launch with programmatic dependent launch
  unsigned long long wait_ns;  // bounded-wait limit of the chunked kernels
  bool precise_state;  // chunked chain: the state enters its products as a bf16 hi + lo pair
  unsigned long long epoch;    // per-call tag of the chunked scan's ready flags (set at launch)
};

// The bounded-wait limit the scan kernels get (tr_set_wait_limit_ns; 4 s by default).
unsigned long long scan_wait_limit_ns();

int device_sm_count();

// Launch `kern` on `s`; with `pdl` the launch carries programmatic stream serialization
// (the kernel may start before its predecessor in the stream completes and must call
// pdl_wait() before touching global data).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Set the thread-local message tr_last_error() returns (cleared for TR_OK) and
// return `status`; printf-style.
int record_error(int status, const char *fmt, ...);

// 2D bf16 tensor map, 128-byte swizzle: `outer` rows of `inner` elements with
// `row_stride_bytes` between rows; box = box_inner x box_outer elements.
bool make_tmap_bf16_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                       std::string *err);

// C[M, N] = A[M, K] * B[N, K]^T with the input-projection epilogue.
cudaError_t launch_gemm_inproj(const void *A, const void *B, int M, int N, int K,
                               const InProjEpi &ep, unsigned *err_word, cudaStream_t s,
                               bool pdl, std::string *err);
// C[M, N] = A[M, K] * B[N, K]^T with the residual epilogue; A rows lda elements apart.
cudaError_t launch_gemm_resid(const void *A, int64_t lda, const void *B, int M, int N, int K,
                              const ResidEpi &ep, unsigned *err_word, cudaStream_t s, bool pdl,
                              std::string *err);

// h[M, d_ff] = bf16(silu(A W_gate^T) * (A W_up^T)), W_gate and W_up [d_ff, K] (d_ff a
// multiple of 128).
cudaError_t launch_gemm_swiglu(const void *A, const void *W_gate, const void *W_up, int M, int d_ff,
                               int K, const SwigluEpi &ep, unsigned *err_word, cudaStream_t s,
                               bool pdl, std::string *err);

cudaError_t launch_short_conv(const ShortConvLaunch &p, cudaStream_t s, bool pdl);

// o <- bf16(o / sqrt(mean_{d_v} o^2 + eps) * gain * silu(z)) per token and head, in place.
cudaError_t launch_gated_norm(__nv_bfloat16 *o, const __nv_bfloat16 *z, const float *gain,
                              int64_t T, int H, int dv, float eps, cudaStream_t s, bool pdl);

cudaError_t launch_rmsnorm(const void *x, int x_is_bf16, const float *gain, int64_t rows, int D,
                           float eps, void *out, cudaStream_t s, bool pdl);

// 2D fp32 tensor map, 128-byte swizzle (box_inner * 4 must be <= 128).
bool make_tmap_f32_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                      std::string *err);

cudaError_t launch_scan_recurrent(const ScanLaunch &p, cudaStream_t s);
// Two or three launches (prep, chain, and the readout when o is requested); `between`
// runs after every launch but the last.
cudaError_t launch_scan_chunked(const ScanLaunch &p, cudaStream_t s, std::string *err,
                                const std::function<cudaError_t()> &between);
bool scan_chunked_supported(const ScanLaunch &p);
size_t scan_chunked_workspace(const ScanLaunch &p);  // needs p.cu_seqlens_host, H, dv
// the kernels one call launches, in order
std::vector<const char *> scan_chunked_kernel_names(const ScanLaunch &p, bool with_readout);

// Pieces per matrix of the state error's first pass (partials holds 2 doubles per piece;
// at most max_pieces pieces in all).
int state_error_splits(int64_t n_mats, int64_t mat_elems, int64_t max_pieces);
cudaError_t launch_state_error(const float *S, const float *Sh, int64_t n_mats, int64_t mat_elems,
                               int splits, double *partials, double *err_per, double *err_total,
                               cudaStream_t s, bool pdl);

}  // namespace tr
