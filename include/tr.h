/*
 * tr.h -- C ABI of libtr.so, the B200 (sm_100a) hot path of Tail-Replay:
 * zero-initialised replay of the last k = ceil(r*m) tokens of a matched prefix
 * through each group's Gated DeltaNet (linear-attention, LA) layers, rebuilding
 * the recurrent states S_hat_m.
 *
 * Sources (web pages on the Tail-Replay paper, arXiv 2608.30310):
 *   RN = "Tail-Replay reading notes" (cc.laoqi.cc): section 2.1 (cache record,
 *        k = ceil(r m)), section 2.2 (the four-step hit path and its worked
 *        example), section 2.3 (Eq. (1), the error identity), section 2.4
 *        (per-group exact entry points), section 2.5 (tail-FFN skip).
 *   GS = "Tail-Replay technical summary" (gist.science), "Key Mechanisms":
 *        fetch the last k cached FA output hiddens, zero the replay state,
 *        replay Eq. (1), independently per group.
 *
 * Conventions for every call
 *   - Ownership: the caller owns every buffer.  Array arguments are DEVICE
 *     pointers unless the name ends in _host.  Nothing here allocates device
 *     memory: scratch space is the caller's workspace `ws` of at least the size
 *     the matching *_workspace_size() returns (256-byte aligned).
 *   - Asynchrony: work is enqueued on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and the call returns after enqueue.
 *     Device-side failures (a bounded wait that ran out) are reported by
 *     tr_check().
 *   - Errors: every call returns a tr_status; TR_OK is 0.  On failure nothing
 *     was enqueued (argument errors are found before any launch) and
 *     tr_last_error() returns a thread-local message.  No call exits, traps or
 *     prints.
 *   - Layouts are row-major and packed unless a stride argument says otherwise.
 *     bf16 means IEEE bfloat16 (round-to-nearest-even on every store); all
 *     recurrent state is fp32.
 *   - State layout: the pages leave the axis order open (RN section 2.3, remark
 *     after Eq. (1)).  States are stored as M = S^T, a d_k x d_v matrix per
 *     (sequence, head), so that Eq. (1) reads M_i = T_i M_{i-1} + beta_i k_i v_i^T
 *     with T_i = alpha_i (I - beta_i k_i k_i^T) acting from the left.
 */
#ifndef TAIL_REPLAY_TR_H
#define TAIL_REPLAY_TR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int tr_status;
enum {
  TR_OK = 0,
  TR_ERR_INVALID_ARG = 1,   /* NULL where a buffer is required, negative size, bad flag */
  TR_ERR_SHAPE = 2,         /* sizes inconsistent (e.g. cu_seqlens_host[N] != total_tokens) */
  TR_ERR_DTYPE = 3,         /* unknown dtype code */
  TR_ERR_ALIGNMENT = 4,     /* a pointer or row stride is not 16-byte aligned */
  TR_ERR_UNSUPPORTED = 5,   /* a size outside what the kernels implement (see each call) */
  TR_ERR_WORKSPACE = 6,     /* ws NULL or smaller than *_workspace_size() */
  TR_ERR_CUDA = 7,          /* a CUDA runtime call or launch failed */
  TR_ERR_TIMEOUT = 8        /* reported by tr_check(): a device-side bounded wait ran out */
};

/* element types */
enum { TR_DTYPE_F32 = 0, TR_DTYPE_BF16 = 1 };

/* flags */
enum {
  TR_NORMALIZE_QK = 1u,      /* tr_gdn_scan: L2-normalise q and k per head in the kernel */
  TR_SKIP_LAST_OUTPUT = 2u,  /* tr_replay_group(s): skip the last LA layer's readout, q
                                projection and output projection (its output rebuilds no
                                state; RN section 2.5 makes the same point for the tail FFN) */
  TR_SCAN_RECURRENT = 4u,    /* force the token-sequential scan kernel (test path) */
  TR_SKIP_LAST_FFN = 8u      /* tr_replay_group(s): do not run the last LA layer's FFN
                                sublayer (RN section 2.5, tail-FFN skip: the next group
                                starts from its own cached FA output, so that FFN output
                                rebuilds no state); x_out is then the residual after the
                                last LA sublayer */,
  TR_OUTPUT_GATE = 16u,      /* tr_replay_group(s): every layer's W_in carries H d_v more
                                rows (z, after v) and the readout goes through the gated
                                RMSNorm before the output projection (see below) */
  TR_SCAN_STALL_TEST = 256u  /* tr_gdn_scan, test hook: the chunked chain kernel never
                                announces its first state, so its bounded waits run out
                                (after tr_set_wait_limit_ns) and the call ends with
                                TR_ERR_TIMEOUT at tr_check; outputs undefined */
};

/* Human-readable message for the last failing call on this host thread. */
const char *tr_last_error(void);

/* Library build string (compiler, target). */
const char *tr_version(void);

/*
 * Tail length (RN section 2.1, symbol table; worked example RN section 2.2):
 * k = ceil(r * m) for r = r_num / r_den, in exact integer arithmetic, clamped to
 * [0, m].  Returns -1 if r_den <= 0 or m < 0.  Host-only, no device work.
 * The tail is rows m-k .. m-1 (0-based) of the cached hiddens, positions
 * m-k+1 .. m (1-based).
 */
int64_t tr_tail_len(int64_t m, int64_t r_num, int64_t r_den);

/*
 * ---------------------------------------------------------------- tr_gdn_scan
 * The Gated DeltaNet recurrence, Eq. (1) of RN section 2.3, over a packed batch
 * of sequences, per head, from S0 (zero start when S0 is NULL -- RN section 2.2
 * step 2, GS "Key Mechanisms"):
 *
 *   M_t = alpha_t (M_{t-1} - beta_t k_t (k_t^T M_{t-1})) + beta_t k_t v_t^T,
 *   o_t = scale * M_t^T q_t   (readout after the update; the pages do not define
 *                              the readout, this is the reading used)
 *   S_final = M at the last token of each sequence (S0, or 0, for empty ones).
 *
 * Arguments (T = total_tokens, N = n_seqs, H = n_heads):
 *   q, k      [T, H, d_k] elements of `dtype`, token stride q_stride/k_stride
 *             elements (0 = H*d_k).  q may be NULL when o is NULL.
 *   v         [T, H, d_v], token stride v_stride (0 = H*d_v).
 *   log_alpha [T, H] fp32, log of the decay alpha in (0, 1] (so <= 0).  Values
 *             are not checked on the device.
 *   beta      [T, H] fp32.
 *   cu_seqlens      [N+1] int32 device offsets, cu[0] = 0, cu[N] = T, nondecreasing.
 *   cu_seqlens_host the same N+1 values in host memory (validation and the
 *                   workspace size); must equal the device copy.
 *   S0        [N, H, d_k, d_v] fp32 or NULL (zero start).
 *   o         [T, H, d_v] of `dtype`, or NULL to skip the readout.
 *   S_final   [N, H, d_k, d_v] fp32, required.  Must not alias S0.
 *   scale     readout scale (1.0 in every workload here).
 *   flags     TR_NORMALIZE_QK, TR_SCAN_RECURRENT, TR_SCAN_STALL_TEST (test hook).
 * Supported: d_k, d_v in {64, 128}; dtype TR_DTYPE_BF16 (the chunked tensor-core
 * scan when d_k = 128 and N <= 1024, else the token-sequential kernel) or
 * TR_DTYPE_F32 (token-sequential fp32 FMA kernel, the test path);
 * 16-byte aligned q/k/v/o with strides that keep every row 16-byte aligned.
 * Workspace: tr_gdn_scan_workspace_size(args) bytes.
 */
typedef struct tr_scan_args {
  int32_t n_seqs, n_heads, d_k, d_v;
  int64_t total_tokens;
  int32_t dtype;
  uint32_t flags;
  float scale;
  int64_t q_stride, k_stride, v_stride;
  const void *q, *k, *v;
  const float *log_alpha, *beta;
  const int32_t *cu_seqlens;
  const int32_t *cu_seqlens_host;
  const float *S0;
  void *o;
  float *S_final;
} tr_scan_args;

size_t tr_gdn_scan_workspace_size(const tr_scan_args *args);
tr_status tr_gdn_scan(const tr_scan_args *args, void *ws, size_t ws_bytes, void *stream);

/* Transition product of each (sequence, head) of a packed batch
 * (Tail-Replay reading notes, section 2.3: the error identity E_m = (T_m ... T_{a+1}) S_a;
 * HYPIC, abstract: the segment transition operator):
 *   P = T_t ... T_1 over the sequence's tokens,  T_i = alpha_i (I - beta_i k_i k_i^T).
 * In the M = S^T layout a state M_0 before the sequence becomes P M_0 + M_hat after it,
 * M_hat being the zero-start state tr_gdn_scan returns.  So an earlier exact state M_a
 * repairs a tail replay exactly, M_m = P M_a + M_hat_m, and ||P||_2 <= prod alpha_i
 * bounds how much of M_a the zero start loses.
 *   args  as for tr_gdn_scan; only n_seqs, n_heads, d_k, total_tokens, dtype, flags
 *         (TR_NORMALIZE_QK), k, k_stride, log_alpha, beta, cu_seqlens and
 *         cu_seqlens_host are read (v, q, S0, o, S_final and d_v are ignored).
 *   P     [N, H, d_k, d_k] fp32 output (device).
 * Computed by the scan itself, with v = 0 from S0 = I (the chunked kernels when dtype is
 * bf16 and d_k = 128: bf16 operands, fp32 products, like the states).
 * Workspace: tr_transition_product_workspace_size(args) bytes, 256-byte aligned.
 */
size_t tr_transition_product_workspace_size(const tr_scan_args *args);
tr_status tr_transition_product(const tr_scan_args *args, float *P, void *ws, size_t ws_bytes,
                                void *stream);

/*
 * ---------------------------------------------------------- tr_replay_group
 * Replay of one group's LA layers over the packed k-token tails (RN section
 * 2.2 steps 2-3; GS "Key Mechanisms"; the group is the run of LA layers after
 * one FA layer, RN section 2.1 figure 1).  Each request's tail starts from the
 * cached FA output hiddens h_{m-k+1..m} (exact, RN section 2.4) with every LA
 * state zero; the hiddens pass through the LA layers in order, giving S_hat_m
 * for every LA layer.  Passing the whole prefix (k = m) gives the full-prefill
 * S_m (RN section 3.1, "Full").
 *
 * Per LA layer (the pages give no layer internals; this is the reading used):
 *   x_hat = bf16(RMSNorm(x) * gain)            eps = rms_eps (0 -> 1e-6)
 *   [q|k|v|a_alpha|a_beta] = x_hat W_in^T      fp32 accumulate
 *     (for the layers after the first the norm is computed inside the residual GEMM
 *     before the layer and the projection: x_hat = bf16(x * gain) and the projection's
 *     outputs are multiplied by the row's 1 / sqrt(mean x^2 + rms_eps); the same value,
 *     the bf16 rounding taken before the scale)
 *   q, k <- bf16(x / sqrt(sum x^2 + norm_eps)) per head (norm_eps 0 -> 1e-6)
 *   v <- bf16(v); log alpha = -softplus(a_alpha), beta = sigmoid(a_beta) (fp32)
 *   o, S_hat[layer] = tr_gdn_scan(q, k, v, log alpha, beta), zero start
 *   x <- x + bf16(o) W_o^T                     fp32 residual
 * Optional Gated DeltaNet details (the pages omit them; these are the public Gated
 * DeltaNet layer's, off unless asked for):
 *   conv_width > 0: the bf16 q|k|v projections (stored without the L2 norm) go through
 *     a causal depthwise convolution of that width and silu, with zero history at each
 *     tail start, before the L2 norm of q and k:
 *       y_t[c] = silu(sum_j conv_w[c][j] * x_{t-W+1+j}[c]) (fp32), q, k, v <- bf16(...)
 *     conv_state (optional) receives each layer's convolution state: the last W-1
 *     projected rows of every sequence, oldest first, zero-padded.
 *   A_log, dt_bias [H] (per layer, optional):
 *       log alpha = -exp(A_log) * softplus(a_alpha + dt_bias)
 *   TR_OUTPUT_GATE: z = x_hat W_z^T from the extra W_in rows (bf16), and per head
 *       o <- bf16(o / sqrt(mean_{d_v} o^2 + rms_eps) * o_norm_gain * silu(z))
 * and, where the layer has FFN weights (W_gate not NULL), the FFN sublayer that
 * RN section 2.5 says still runs between a group's LA layers (the pages do not
 * give its form; the reading is a dense SwiGLU with its own pre-norm):
 *   x_hat = bf16(RMSNorm(x) * ffn_gain)        eps = rms_eps
 *   h = bf16(silu(x_hat W_gate^T) * (x_hat W_up^T))   fp32 products, silu in fp32
 *   x <- x + h W_down^T                        fp32 residual
 * x starts as h_tail.  The cast points above are part of this contract.
 *
 * Arguments (T = total_tokens, D = d_model, H = n_heads):
 *   h_tail   [T, D] bf16, the N requests' tails packed by cu_seqlens.
 *   layers   HOST array of n_layers tr_la_layer:
 *              rms_gain [D] fp32 or NULL (ones)
 *              W_in     [2 H d_k + H d_v + 2 H, D] bf16 (output x input features;
 *                       rows: q heads, k heads, v heads, a_alpha, a_beta); with
 *                       TR_OUTPUT_GATE [2 H d_k + 2 H d_v + 2 H, D], rows q, k, v,
 *                       z heads, a_alpha, a_beta
 *              W_o      [D, H d_v] bf16
 *              ffn_gain [D] fp32 or NULL (ones)
 *              W_gate   [d_ff, D] bf16, or NULL: the layer has no FFN sublayer
 *              W_up     [d_ff, D] bf16 (with W_gate)
 *              W_down   [D, d_ff] bf16 (with W_gate)
 *              conv_w   [2 H d_k + H d_v, conv_width] fp32, given exactly when
 *                       conv_width > 0 (tap conv_width-1 weighs the current token)
 *              A_log, dt_bias  [H] fp32 or NULL (0)
 *              o_norm_gain     [d_v] fp32 or NULL (ones); only with TR_OUTPUT_GATE
 *   d_ff     FFN width, a multiple of 128; 0 when no layer has an FFN.
 *   conv_width   0 (no convolution) or 2..4; needs d_k = d_v.
 *   conv_state   [n_layers, N, conv_width - 1, 2 H d_k + H d_v] bf16 output, or NULL.
 *                With it, the last layer's q projection is computed even under
 *                TR_SKIP_LAST_OUTPUT (the state holds the q channels too).
 *   S_hat    [n_layers, N, H, d_k, d_v] fp32 output.
 *   x_out    [T, D] fp32 output of the last layer, or NULL (then the last
 *            layer's output projection and FFN are not run).  Must be NULL with
 *            TR_SKIP_LAST_OUTPUT, which skips the last FFN as well.
 * Supported: d_k = d_v = 128 or 64; D a multiple of 64; 1 <= n_layers <= 64.
 * Workspace: tr_replay_group_workspace_size(args) bytes.
 */
typedef struct tr_la_layer {
  const float *rms_gain;
  const void *W_in;
  const void *W_o;
  const float *ffn_gain;
  const void *W_gate;
  const void *W_up;
  const void *W_down;
  const float *conv_w;
  const float *A_log;
  const float *dt_bias;
  const float *o_norm_gain;
} tr_la_layer;

typedef struct tr_group_args {
  int32_t n_seqs, n_heads, d_k, d_v, d_model, n_layers;
  int64_t total_tokens;
  uint32_t flags;
  float rms_eps, norm_eps;
  int32_t d_ff;
  const void *h_tail;
  const int32_t *cu_seqlens;
  const int32_t *cu_seqlens_host;
  const tr_la_layer *layers;
  float *S_hat;
  float *x_out;
  int32_t conv_width;
  void *conv_state;
} tr_group_args;

size_t tr_replay_group_workspace_size(const tr_group_args *args);
tr_status tr_replay_group(const tr_group_args *args, void *ws, size_t ws_bytes, void *stream);

/*
 * The same replay with timing marks: `events` is a HOST array of n_events
 * created cudaEvent_t handles (passed as void*).  events[0] is recorded on
 * `stream` before the first kernel and events[i] after the i-th kernel launch,
 * in launch order (the first layer's RMSNorm, then per layer the input projection,
 * the scan, and the output projection when it runs).  n_events must be at least
 * 1 + tr_replay_group_kernel_count(args); the rest are left alone.
 */
int32_t tr_replay_group_kernel_count(const tr_group_args *args);
/* The names of those kernels, comma-separated, in launch order (a thread-local string,
 * valid until the next call from the same thread; "" for invalid args).  Host-only.
 * They describe an uncaptured call: a call made while its stream captures a graph runs
 * the scan as separate prep and chain kernels (the single-launch form synchronises its
 * parts through per-call tags, which a replayed graph would repeat). */
const char *tr_replay_group_kernel_names(const tr_group_args *args);
tr_status tr_replay_group_profiled(const tr_group_args *args, void *ws, size_t ws_bytes,
                                   void *stream, void *const *events, int32_t n_events);

/*
 * All groups of all hits in one call (groups are independent: RN section 2.4,
 * GS "Key Mechanisms").  groups is a HOST array of n_groups tr_group_args; each
 * group carries its own LA weights and its own tails (the hits of one group
 * share its weights and are packed by that group's cu_seqlens).  The workspace
 * is shared: tr_replay_groups_workspace_size() is the largest single group's, and
 * with that much the groups run one after another on `stream`.
 *
 * Lanes: a workspace of tr_replay_groups_lanes_workspace_size(groups, n, L) bytes
 * (L slices of the single-group size, L = 2..4) lets the call run the groups on L
 * lanes at once: group g on lane g % L with its own slice, lane 0 on `stream`, the
 * others on streams the library keeps per device (created on first use), forked
 * from `stream` by an event and joined back into it before the call returns, so
 * work enqueued on `stream` after the call sees every group's results.  The lanes
 * overlap one group's partly idle phases (a chunk chain on few SMs, a GEMM's last
 * wave) with another group's kernels; the results are bitwise those of the
 * sequential call.  The lanes are used as far as the workspace allows, never
 * while `stream` is being captured into a graph (the groups then run in turn).
 */
size_t tr_replay_groups_workspace_size(const tr_group_args *groups, int32_t n_groups);
size_t tr_replay_groups_lanes_workspace_size(const tr_group_args *groups, int32_t n_groups,
                                             int32_t lanes);
tr_status tr_replay_groups(const tr_group_args *groups, int32_t n_groups, void *ws,
                           size_t ws_bytes, void *stream);

/*
 * tr_replay_groups with the full-attention KV transfer overlapped (Tail-Replay reading
 * notes, section 2.5: the KV of the matched prefix moves to the device on a separate
 * stream while the linear-attention states are replayed, T ~ max(T_KV, T_replay)).
 * `kv_bytes` are copied from `kv_host` (pinned host memory) to `kv_dev` on `copy_stream`,
 * issued before the replay's kernels on `stream`.  The copy waits for everything enqueued
 * on `stream` before the call (an event recorded at entry), so earlier work that still
 * reads kv_dev finishes first; `stream` then waits for the copy, so work enqueued on it
 * afterwards sees both the KV and the states.  One cudaMemcpyAsync;
 * kv_bytes = 0 replays only.  The two streams must differ.  Same workspace as
 * tr_replay_groups.  Every argument (the KV pointers and streams, each group, the
 * workspace) is checked before the copy is issued: a rejected call moves no bytes.
 */
tr_status tr_replay_groups_overlapped(const tr_group_args *groups, int32_t n_groups, void *ws,
                                      size_t ws_bytes, const void *kv_host, void *kv_dev,
                                      size_t kv_bytes, void *stream, void *copy_stream);

/*
 * ---------------------------------------------------------- tr_state_error
 * Relative Frobenius error of a rebuilt state against the full-prefill state
 * (E_m = S_m - S_hat_m, RN section 2.3):
 *   err_per_mat[i] = ||S_i - S_hat_i||_F / ||S_i||_F  over each d_k x d_v matrix
 *   err_total      = ||S - S_hat||_F / ||S||_F        over all n_mats matrices
 * with fp64 accumulation of the fp32 data.  When a denominator is 0 the error
 * is 0 if the numerator is 0, else +inf.
 *   S, S_hat     [n_mats, d_k, d_v] fp32 (device).
 *   err_per_mat  [n_mats] fp64 (device) or NULL.
 *   err_total    [1] fp64 (device) or NULL.
 * Workspace: tr_state_error_workspace_size(n_mats) bytes.
 */
size_t tr_state_error_workspace_size(int64_t n_mats);
tr_status tr_state_error(const float *S, const float *S_hat, int64_t n_mats, int32_t d_k,
                         int32_t d_v, double *err_per_mat, double *err_total, void *ws,
                         size_t ws_bytes, void *stream);

/*
 * tr_state_error_noalloc: the same result as tr_state_error, for callers that
 * cannot allocate device memory when they make the call (an engine whose
 * allocator owns all device memory, or code where cudaMalloc would synchronize
 * the device).  The paper has no counterpart: this is a deployment variant.
 *   - Scratch space is a fixed array inside the library (2 x 65536 doubles, 1 MiB
 *     per GPU that loads the library, held until the process exits); n_mats above
 *     65536 is rejected with TR_ERR_UNSUPPORTED.  Nothing is allocated.
 *   - Every call made outside stream capture looks up the array's device address in
 *     the current context (cudaGetSymbolAddress), so a context created again after
 *     cudaDeviceReset is served correctly.  A call made while its stream captures
 *     reuses the address of the last uncaptured call on that device: make one
 *     uncaptured call on a device (in the current context) before capturing one;
 *     without it the captured call returns TR_ERR_INVALID_ARG.
 *   - All calls share the array: calls whose kernels may overlap on the GPU race.
 *     Each call writes every scratch entry it reads, so nothing needs clearing.
 */
tr_status tr_state_error_noalloc(const float *S, const float *S_hat, int64_t n_mats, int32_t d_k,
                                 int32_t d_v, double *err_per_mat, double *err_total,
                                 void *stream);

/*
 * ---------------------------------------------- steps of one LA layer, alone
 * The three dense steps of tr_replay_group, exposed so that each can be checked
 * on its own.  Same arithmetic and cast points as inside tr_replay_group (the
 * group's first layer: its later layers fold the RMSNorm into the GEMMs, see above).
 *
 * tr_rmsnorm: x_hat[t] = bf16(x[t] / sqrt(mean_j x[t,j]^2 + eps) * gain)
 *   x [n_rows, D] of x_dtype (bf16 or fp32); gain [D] fp32 or NULL;
 *   x_hat [n_rows, D] bf16.  eps 0 -> 1e-6.  D a multiple of 8.
 */
tr_status tr_rmsnorm(const void *x, int32_t x_dtype, const float *gain, int64_t n_rows,
                     int32_t d_model, float eps, void *x_hat, void *stream);

/*
 * tr_in_projection: y = x_hat W_in^T (tcgen05 tensor cores, fp32 accumulate) with
 * the gate and key-norm epilogue:
 *   qkv [T, 2 H d_k + H d_v] bf16 = [L2norm(q) | L2norm(k) | v] per head,
 *   log_alpha [T, H] = -softplus(a_alpha), beta [T, H] = sigmoid(a_beta), fp32.
 * With TR_SKIP_LAST_OUTPUT in flags the q columns are neither computed nor
 * written.  x_hat [T, D] bf16, W_in as in tr_la_layer.  norm_eps 0 -> 1e-6.
 */
tr_status tr_in_projection(const void *x_hat, const void *W_in, int64_t n_tokens,
                           int32_t d_model, int32_t n_heads, int32_t d_k, int32_t d_v,
                           uint32_t flags, float norm_eps, void *qkv, float *log_alpha,
                           float *beta, void *stream);

/*
 * tr_out_projection: x_out = x_res + o W_o^T (tcgen05, fp32 accumulate, fp32 out).
 *   o [T, H d_v] bf16 (row stride o_stride elements, 0 = H d_v); W_o [D, H d_v] bf16;
 *   x_res [T, D] of x_res_dtype (bf16 or fp32); x_out [T, D] fp32 (may equal x_res
 *   when x_res is fp32).
 */
tr_status tr_out_projection(const void *o, int64_t o_stride, const void *W_o, const void *x_res,
                            int32_t x_res_dtype, int64_t n_tokens, int32_t d_model,
                            int32_t hv, float *x_out, void *stream);

/*
 * tr_set_wait_limit_ns: the wall-clock limit of every bounded wait in the chunked scan's
 * kernels (their mbarrier waits on copies, products and the other roles of a CTA), for
 * calls made after it; 0 restores the default of 4 s, above 60 s is rejected.  A wait that
 * runs out makes its CTA stop: it lets the copies and products it already issued finish
 * (a drain bounded separately, at 0.2 s), writes no further output, and sets the device
 * error word that tr_check reports as TR_ERR_TIMEOUT; the outputs of that call are then
 * undefined, and later calls work normally.  Process-wide (not per thread or device).
 * Every legitimate wait ends within microseconds; a short limit serves to test this path.
 */
tr_status tr_set_wait_limit_ns(uint64_t ns);

/*
 * tr_check: waits for `stream`, then reads and clears the library's device error
 * word.  Returns TR_ERR_TIMEOUT if a kernel gave up a bounded wait since the
 * last check, TR_ERR_CUDA if the stream reports an error, else TR_OK.
 */
tr_status tr_check(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TAIL_REPLAY_TR_H */
