// tr_api.cu -- the extern "C" boundary of libtr.so (declared in include/tr.h):
// argument validation, workspace layout, launch sequencing and error reporting.
// Every argument error is found before the first launch of a call, so a failed
// call enqueues nothing.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/tr.h"
#include "tr_internal.h"

namespace {

thread_local std::string g_last_error;

tr_status fail(tr_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

tr_status ok() {
  g_last_error.clear();
  return TR_OK;
}

tr_status cuda_fail(cudaError_t e, const char *what) {
  return fail(TR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The library's device error word; kernels OR their ERRBIT_* into it.
__device__ unsigned g_err_word;

constexpr int kMaxDevices = 64;
unsigned *g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];
std::mutex g_dev_mu;

// The device's SM count and the address of the library's error word in the current
// context.  The address is looked up again on every call made outside stream capture (a
// context created anew after cudaDeviceReset has its own copy of the word); a call made
// while `s` captures reuses what the last uncaptured call on this device found.
bool device_state(cudaStream_t s, int *dev_out, unsigned **err_out, std::string *err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    if (err) *err = std::string("cudaGetDevice: ") + cudaGetErrorString(e);
    return false;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) {
    if (err) *err = std::string("cudaStreamIsCapturing: ") + cudaGetErrorString(e);
    return false;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (cap == cudaStreamCaptureStatusNone || !g_err_ptr[dev]) {
    if (cap != cudaStreamCaptureStatusNone) {
      if (err) *err = "the first call on a device must come before any stream capture";
      return false;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_err_word);
    if (e != cudaSuccess) {
      if (err) *err = std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e);
      return false;
    }
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = sms > 0 ? sms : 1;
    g_err_ptr[dev] = static_cast<unsigned *>(p);
  }
  *dev_out = dev;
  *err_out = g_err_ptr[dev];
  return true;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

namespace tr {

int record_error(int status, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = status == TR_OK ? std::string() : std::string(buf);
  return status;
}

std::atomic<unsigned long long> g_wait_ns{4000000000ull};

unsigned long long scan_wait_limit_ns() { return g_wait_ns.load(); }

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  return g_sms[dev] > 0 ? g_sms[dev] : 148;
}

bool make_tmap_bf16_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                       std::string *err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    if (err) *err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) {
      char b[160];
      snprintf(b, sizeof(b), "cuTensorMapEncodeTiled failed (%d): dims %llu x %llu stride %llu",
               (int)r, (unsigned long long)inner, (unsigned long long)outer,
               (unsigned long long)row_stride_bytes);
      *err = b;
    }
    return false;
  }
  return true;
}

bool make_tmap_f32_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                      std::string *err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    if (err) *err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) {
      char b[160];
      snprintf(b, sizeof(b), "cuTensorMapEncodeTiled (fp32) failed (%d): dims %llu x %llu",
               (int)r, (unsigned long long)inner, (unsigned long long)outer);
      *err = b;
    }
    return false;
  }
  return true;
}

}  // namespace tr

// ---------------------------------------------------------------- validation
namespace {

tr_status check_cu_host(const int32_t *cu, int32_t n, int64_t T) {
  if (!cu) return fail(TR_ERR_INVALID_ARG, "cu_seqlens_host is NULL");
  if (cu[0] != 0) return fail(TR_ERR_SHAPE, "cu_seqlens_host[0] = %d, expected 0", cu[0]);
  for (int32_t i = 0; i < n; ++i)
    if (cu[i + 1] < cu[i]) return fail(TR_ERR_SHAPE, "cu_seqlens_host decreases at %d", i);
  if (cu[n] != T)
    return fail(TR_ERR_SHAPE, "cu_seqlens_host[N] = %d but total_tokens = %lld", cu[n],
                (long long)T);
  return TR_OK;
}

tr_status validate_scan(const tr_scan_args *a, tr::ScanLaunch *out) {
  if (!a) return fail(TR_ERR_INVALID_ARG, "args is NULL");
  if (a->n_seqs < 0 || a->n_heads <= 0 || a->total_tokens < 0)
    return fail(TR_ERR_INVALID_ARG, "negative or zero size (n_seqs %d, n_heads %d, T %lld)",
                a->n_seqs, a->n_heads, (long long)a->total_tokens);
  if (a->total_tokens > 0x7fffffffLL) return fail(TR_ERR_UNSUPPORTED, "total_tokens > 2^31-1");
  if (a->dtype != TR_DTYPE_F32 && a->dtype != TR_DTYPE_BF16)
    return fail(TR_ERR_DTYPE, "dtype %d", a->dtype);
  if ((a->d_k != 64 && a->d_k != 128) || (a->d_v != 64 && a->d_v != 128))
    return fail(TR_ERR_UNSUPPORTED, "d_k = %d, d_v = %d: supported values are 64 and 128", a->d_k,
                a->d_v);
  if (a->flags & ~(unsigned)(TR_NORMALIZE_QK | TR_SCAN_RECURRENT | TR_SCAN_STALL_TEST))
    return fail(TR_ERR_INVALID_ARG, "unknown scan flags 0x%x", a->flags);
  if (!a->S_final || !a->cu_seqlens)
    return fail(TR_ERR_INVALID_ARG, "a required pointer is NULL");
  if (a->total_tokens > 0 && (!a->k || !a->v || !a->log_alpha || !a->beta))
    return fail(TR_ERR_INVALID_ARG, "a required pointer is NULL");
  if (a->total_tokens > 0 && a->o && !a->q)
    return fail(TR_ERR_INVALID_ARG, "q is NULL but o is requested");
  if (a->S0 && a->S0 == a->S_final) return fail(TR_ERR_INVALID_ARG, "S_final aliases S0");
  tr_status st = check_cu_host(a->cu_seqlens_host, a->n_seqs, a->total_tokens);
  if (st != TR_OK) return st;
  const int64_t H = a->n_heads;
  const int64_t qs = a->q_stride ? a->q_stride : H * a->d_k;
  const int64_t ks = a->k_stride ? a->k_stride : H * a->d_k;
  const int64_t vs = a->v_stride ? a->v_stride : H * a->d_v;
  if (qs < H * a->d_k || ks < H * a->d_k || vs < H * a->d_v)
    return fail(TR_ERR_SHAPE, "a token stride is smaller than H * d");
  const int esz = a->dtype == TR_DTYPE_BF16 ? 2 : 4;
  if ((a->q && !aligned16(a->q)) || !aligned16(a->k) || !aligned16(a->v) ||
      (a->o && !aligned16(a->o)) || (qs * esz) % 16 || (ks * esz) % 16 || (vs * esz) % 16)
    return fail(TR_ERR_ALIGNMENT, "q/k/v/o and their token strides must be 16-byte aligned");
  if (!aligned16(a->S_final) || (a->S0 && !aligned16(a->S0)))
    return fail(TR_ERR_ALIGNMENT, "S0/S_final must be 16-byte aligned");
  tr::ScanLaunch &p = *out;
  p = tr::ScanLaunch{};   // every field not set below is off
  p.n_seqs = a->n_seqs;
  p.H = a->n_heads;
  p.dk = a->d_k;
  p.dv = a->d_v;
  p.T = a->total_tokens;
  p.dtype = a->dtype;
  p.flags = a->flags;
  p.scale = a->scale;
  p.q_stride = qs;
  p.k_stride = ks;
  p.v_stride = vs;
  p.o_stride = H * a->d_v;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.log_alpha = a->log_alpha;
  p.beta = a->beta;
  p.cu_seqlens = a->cu_seqlens;
  p.cu_seqlens_host = a->cu_seqlens_host;
  p.S0 = a->S0;
  p.o = a->o;
  p.S_final = a->S_final;
  p.err_word = nullptr;
  p.ws = nullptr;
  p.ws_bytes = 0;
  p.pdl = true;
  p.wait_ns = tr::scan_wait_limit_ns();
  p.precise_state = false;
  return TR_OK;
}

bool use_chunked(const tr::ScanLaunch &p) {
  return p.dtype == TR_DTYPE_BF16 && !(p.flags & TR_SCAN_RECURRENT) && tr::scan_chunked_supported(p);
}

size_t scan_ws_bytes(const tr::ScanLaunch &p) {
  if (!p.cu_seqlens_host) return 0;
  return use_chunked(p) ? tr::scan_chunked_workspace(p) : 0;
}

// Names of the kernels one scan call launches, in launch order.
std::vector<const char *> scan_kernel_names(const tr::ScanLaunch &p, bool with_readout) {
  if (use_chunked(p)) return tr::scan_chunked_kernel_names(p, with_readout);
  return {"scan_recurrent"};
}

tr_status run_scan(const tr::ScanLaunch &p, cudaStream_t s,
                   const std::function<cudaError_t()> &between = nullptr) {
  cudaError_t e;
  if (use_chunked(p)) {
    std::string err;
    e = tr::launch_scan_chunked(p, s, &err, between);
    if (e != cudaSuccess)
      return err.empty() ? cuda_fail(e, "scan (chunked)") : fail(TR_ERR_CUDA, "%s", err.c_str());
  } else {
    e = tr::launch_scan_recurrent(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "scan (recurrent)");
  }
  return TR_OK;
}

// ------------------------------------------------------------- replay group
struct GroupLayout {
  size_t x, xhat, qkv, post, zbuf, la, beta, o, hmid, ssq, scan, total;
  int64_t ldq;
};

bool has_ffn(const tr_la_layer &w) { return w.W_gate != nullptr; }
bool output_gate(const tr_group_args *a) { return (a->flags & TR_OUTPUT_GATE) != 0; }

// W_in rows: [q | k | v | z (with the output gate) | a_alpha | a_beta]
int in_rows(const tr_group_args *a) {
  return 2 * a->n_heads * a->d_k + a->n_heads * a->d_v * (output_gate(a) ? 2 : 1) +
         2 * a->n_heads;
}

// The scan launch of one LA layer of a group (pointers filled in by the caller).
tr::ScanLaunch group_scan_launch(const tr_group_args *a) {
  tr::ScanLaunch sp{};
  sp.n_seqs = a->n_seqs;
  sp.H = a->n_heads;
  sp.dk = a->d_k;
  sp.dv = a->d_v;
  sp.T = a->total_tokens;
  sp.dtype = TR_DTYPE_BF16;
  sp.flags = 0;
  sp.scale = 1.f;
  sp.cu_seqlens_host = a->cu_seqlens_host;
  sp.wait_ns = tr::scan_wait_limit_ns();
  sp.precise_state = false;
  return sp;
}

GroupLayout group_layout(const tr_group_args *a) {
  GroupLayout L;
  const size_t T = (size_t)a->total_tokens, D = (size_t)a->d_model, H = (size_t)a->n_heads;
  L.ldq = 2 * (int64_t)H * a->d_k + (int64_t)H * a->d_v;
  size_t off = 0;
  L.x = off;    off = align256(off + T * D * 4);
  L.xhat = off; off = align256(off + T * D * 2);
  L.qkv = off;  off = align256(off + T * (size_t)L.ldq * 2);
  L.post = off; off = align256(off + (a->conv_width > 0 ? T * (size_t)L.ldq * 2 : 0));
  L.zbuf = off; off = align256(off + (output_gate(a) ? T * H * (size_t)a->d_v * 2 : 0));
  L.la = off;   off = align256(off + T * H * 4);
  L.beta = off; off = align256(off + T * H * 4);
  L.o = off;    off = align256(off + T * H * (size_t)a->d_v * 2);
  L.hmid = off; off = align256(off + T * (size_t)(a->d_ff > 0 ? a->d_ff : 0) * 2);
  // the folded RMSNorm's per-row partial sums of squares (layers after the first)
  L.ssq = off;  off = align256(off + (a->n_layers > 1 ? T * (size_t)tr::resid_ssq_partials((int)D) * 4 : 0));
  L.scan = off; off = align256(off + scan_ws_bytes(group_scan_launch(a)));
  L.total = off;
  return L;
}

tr_status validate_group(const tr_group_args *a) {
  if (!a) return fail(TR_ERR_INVALID_ARG, "args is NULL");
  if (a->n_seqs < 0 || a->n_heads <= 0 || a->d_model <= 0 || a->total_tokens < 0)
    return fail(TR_ERR_INVALID_ARG, "bad sizes (n_seqs %d, n_heads %d, d_model %d, T %lld)",
                a->n_seqs, a->n_heads, a->d_model, (long long)a->total_tokens);
  if (a->n_layers < 1 || a->n_layers > 64)
    return fail(TR_ERR_UNSUPPORTED, "n_layers = %d (1..64 supported)", a->n_layers);
  if (a->total_tokens > 0x7fffffffLL) return fail(TR_ERR_UNSUPPORTED, "total_tokens > 2^31-1");
  if ((a->d_k != 64 && a->d_k != 128) || (a->d_v != 64 && a->d_v != 128))
    return fail(TR_ERR_UNSUPPORTED, "d_k = %d, d_v = %d: supported values are 64 and 128", a->d_k,
                a->d_v);
  if (a->d_model % 64) return fail(TR_ERR_UNSUPPORTED, "d_model = %d is not a multiple of 64",
                                   a->d_model);
  if (a->flags & ~(unsigned)(TR_SKIP_LAST_OUTPUT | TR_SKIP_LAST_FFN | TR_OUTPUT_GATE))
    return fail(TR_ERR_INVALID_ARG, "unknown replay flags 0x%x", a->flags);
  if (a->conv_width != 0 && (a->conv_width < 2 || a->conv_width > 4))
    return fail(TR_ERR_UNSUPPORTED, "conv_width = %d (0 or 2..4 supported)", a->conv_width);
  if (a->conv_width > 0 && a->d_k != a->d_v)
    return fail(TR_ERR_UNSUPPORTED, "the short convolution needs d_k = d_v");
  if (a->conv_state && a->conv_width == 0)
    return fail(TR_ERR_INVALID_ARG, "conv_state given without a convolution");
  if (a->conv_state && !aligned16(a->conv_state))
    return fail(TR_ERR_ALIGNMENT, "conv_state must be 16-byte aligned");
  if (a->d_ff < 0 || a->d_ff % 128)
    return fail(TR_ERR_UNSUPPORTED, "d_ff = %d is not a non-negative multiple of 128", a->d_ff);
  if ((a->flags & TR_SKIP_LAST_OUTPUT) && a->x_out)
    return fail(TR_ERR_INVALID_ARG, "x_out must be NULL with TR_SKIP_LAST_OUTPUT");
  if (!a->cu_seqlens || !a->layers || !a->S_hat || (a->total_tokens > 0 && !a->h_tail))
    return fail(TR_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(a->h_tail) || !aligned16(a->S_hat) || (a->x_out && !aligned16(a->x_out)))
    return fail(TR_ERR_ALIGNMENT, "h_tail/S_hat/x_out must be 16-byte aligned");
  for (int l = 0; l < a->n_layers; ++l) {
    const tr_la_layer &w = a->layers[l];
    if (!w.W_in || !w.W_o) return fail(TR_ERR_INVALID_ARG, "layer %d: W_in or W_o is NULL", l);
    if (!aligned16(w.W_in) || !aligned16(w.W_o) || (w.rms_gain && !aligned16(w.rms_gain)))
      return fail(TR_ERR_ALIGNMENT, "layer %d: weights must be 16-byte aligned", l);
    if (has_ffn(w)) {
      if (a->d_ff == 0)
        return fail(TR_ERR_INVALID_ARG, "layer %d has FFN weights but d_ff = 0", l);
      if (!w.W_up || !w.W_down)
        return fail(TR_ERR_INVALID_ARG, "layer %d: W_gate without W_up or W_down", l);
      if (!aligned16(w.W_gate) || !aligned16(w.W_up) || !aligned16(w.W_down) ||
          (w.ffn_gain && !aligned16(w.ffn_gain)))
        return fail(TR_ERR_ALIGNMENT, "layer %d: FFN weights must be 16-byte aligned", l);
    } else if (w.W_up || w.W_down || w.ffn_gain) {
      return fail(TR_ERR_INVALID_ARG, "layer %d: FFN weights without W_gate", l);
    }
    if ((a->conv_width > 0) != (w.conv_w != nullptr))
      return fail(TR_ERR_INVALID_ARG, "layer %d: conv_w must be given exactly when conv_width > 0",
                  l);
    if (w.o_norm_gain && !output_gate(a))
      return fail(TR_ERR_INVALID_ARG, "layer %d: o_norm_gain without TR_OUTPUT_GATE", l);
    if (!aligned4(w.conv_w) || !aligned4(w.A_log) || !aligned4(w.dt_bias) ||
        !aligned4(w.o_norm_gain))
      return fail(TR_ERR_ALIGNMENT, "layer %d: GDN parameters must be 4-byte aligned", l);
  }
  return check_cu_host(a->cu_seqlens_host, a->n_seqs, a->total_tokens);
}

// Events recorded between kernel launches (profiling variant); inactive when ev == nullptr.
struct Marks {
  void *const *ev = nullptr;
  int n = 0, next = 0;
  cudaError_t mark(cudaStream_t s) {
    if (!ev || next >= n) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev[next++]), s);
  }
};

// Whether layer l runs its FFN sublayer: it has FFN weights, its LA output is computed,
// and it is not the last layer under the tail-FFN skip.
bool runs_ffn(const tr_group_args *a, int l) {
  const bool last = l == a->n_layers - 1;
  if (!has_ffn(a->layers[l])) return false;
  if (last && ((a->flags & (TR_SKIP_LAST_OUTPUT | TR_SKIP_LAST_FFN)) || !a->x_out)) return false;
  return true;
}

// Names of the kernels tr_replay_group launches for `a`, in launch order (the order in
// which replay_group_enqueue records its events).
std::vector<const char *> group_kernel_names(const tr_group_args *a) {
  std::vector<const char *> n;
  for (int l = 0; l < a->n_layers; ++l) {
    const bool last = l == a->n_layers - 1;
    const bool skip = last && (a->flags & TR_SKIP_LAST_OUTPUT);
    // later layers' RMSNorm is folded into the previous layer's last residual GEMM
    if (l == 0) n.push_back("rmsnorm");
    n.push_back("in_proj");
    if (a->conv_width > 0) n.push_back("short_conv");
    for (const char *k : scan_kernel_names(group_scan_launch(a), !skip)) n.push_back(k);
    if (!skip && (!last || a->x_out)) {
      if (output_gate(a)) n.push_back("gated_norm");
      n.push_back("out_proj");
    }
    if (runs_ffn(a, l)) {
      n.push_back("ffn_rmsnorm");
      n.push_back("ffn_gate_up");
      n.push_back("ffn_down");
    }
  }
  return n;
}

int group_kernel_count(const tr_group_args *a) { return (int)group_kernel_names(a).size(); }

thread_local std::string g_names;

tr_status replay_group_enqueue(const tr_group_args *a, void *ws, unsigned *err_word,
                               cudaStream_t s, Marks *mk = nullptr) {
  Marks none;
  if (!mk) mk = &none;
  // programmatic dependent launch between the kernels, except when events are recorded
  // between them (the per-kernel timing path)
  const bool pdl = mk->ev == nullptr;
  if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
  const GroupLayout L = group_layout(a);
  uint8_t *base = static_cast<uint8_t *>(ws);
  float *x = reinterpret_cast<float *>(base + L.x);
  void *xhat = base + L.xhat;
  auto *qkv = reinterpret_cast<__nv_bfloat16 *>(base + L.qkv);
  float *la = reinterpret_cast<float *>(base + L.la);
  float *be = reinterpret_cast<float *>(base + L.beta);
  auto *obuf = reinterpret_cast<__nv_bfloat16 *>(base + L.o);
  auto *hmid = reinterpret_cast<__nv_bfloat16 *>(base + L.hmid);
  auto *post = reinterpret_cast<__nv_bfloat16 *>(base + L.post);
  auto *zbuf = reinterpret_cast<__nv_bfloat16 *>(base + L.zbuf);
  float *ssq = reinterpret_cast<float *>(base + L.ssq);
  const int T = (int)a->total_tokens, D = a->d_model, H = a->n_heads, dk = a->d_k, dv = a->d_v;
  const int n_in = in_rows(a);
  const bool conv = a->conv_width > 0;
  // q and k after the convolution (or straight from the projection)
  const __nv_bfloat16 *qkv_s = conv ? post : qkv;
  const float rms_eps = a->rms_eps > 0.f ? a->rms_eps : 1e-6f;
  const float norm_eps = a->norm_eps > 0.f ? a->norm_eps : 1e-6f;
  const size_t state_elems = (size_t)a->n_seqs * H * dk * dv;
  std::string err;
  cudaError_t e;
  for (int l = 0; l < a->n_layers; ++l) {
    const tr_la_layer &w = a->layers[l];
    const bool last = l == a->n_layers - 1;
    const bool skip = last && (a->flags & TR_SKIP_LAST_OUTPUT);
    // the q columns are still projected when the convolution state (which holds them) is kept
    const bool skip_q = skip && !a->conv_state;
    const void *x_in = l == 0 ? a->h_tail : static_cast<const void *>(x);
    const int in_bf16 = l == 0 ? 1 : 0;
    // the RMSNorm of layers after the first was folded into the residual GEMM that wrote x
    // (xhat = bf16(x * gain) and the rows' partial sums of squares); the projection's
    // epilogue applies 1/rms
    const bool folded = l > 0;
    if (!folded) {
      e = tr::launch_rmsnorm(x_in, in_bf16, w.rms_gain, T, D, rms_eps, xhat, s, pdl);
      if (e != cudaSuccess) return cuda_fail(e, "rmsnorm");
      if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
    }
    // the residual GEMM that writes the next layer's input folds that layer's RMSNorm in
    auto fold_next = [&](tr::ResidEpi &rp) {
      if (l + 1 >= a->n_layers) return;
      rp.xhat_out = static_cast<__nv_bfloat16 *>(xhat);
      rp.gain = a->layers[l + 1].rms_gain;
      rp.ssq_part = ssq;
      rp.part_ld = T;
    };
    tr::InProjEpi ep{};
    if (folded) {
      ep.ssq_part = ssq;
      ep.n_part = tr::resid_ssq_partials(D);
      ep.part_ld = T;
      ep.inv_d = 1.f / (float)D;
      ep.rms_eps = rms_eps;
    }
    ep.qkv = qkv;
    ep.ldq = L.ldq;
    ep.log_alpha = la;
    ep.beta = be;
    ep.H = H;
    ep.dk = dk;
    ep.dv = dv;
    ep.col_offset = skip_q ? H * dk : 0;
    ep.norm_eps = norm_eps;
    ep.raw_qk = conv ? 1 : 0;
    ep.z = output_gate(a) ? zbuf : nullptr;
    ep.A_log = w.A_log;
    ep.dt_bias = w.dt_bias;
    const void *Wb = static_cast<const __nv_bfloat16 *>(w.W_in) + (size_t)ep.col_offset * D;
    e = tr::launch_gemm_inproj(xhat, Wb, T, n_in - ep.col_offset, D, ep, err_word, s, pdl, &err);
    if (e != cudaSuccess)
      return err.empty() ? cuda_fail(e, "input projection") : fail(TR_ERR_CUDA, "%s", err.c_str());
    if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
    if (conv) {
      tr::ShortConvLaunch cp{};
      cp.pre = qkv;
      cp.post = post;
      cp.ld = L.ldq;
      cp.w = w.conv_w;
      cp.width = a->conv_width;
      cp.cu_seqlens = a->cu_seqlens;
      cp.n_seqs = a->n_seqs;
      cp.T = T;
      cp.H = H;
      cp.dk = dk;
      cp.dv = dv;
      cp.skip_q = skip_q ? 1 : 0;
      cp.norm_eps = norm_eps;
      cp.state = a->conv_state
                     ? static_cast<__nv_bfloat16 *>(a->conv_state) +
                           (size_t)l * a->n_seqs * (a->conv_width - 1) * L.ldq
                     : nullptr;
      e = tr::launch_short_conv(cp, s, pdl);
      if (e != cudaSuccess) return cuda_fail(e, "short convolution");
      if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
    }
    tr::ScanLaunch sp = group_scan_launch(a);
    sp.ws = base + L.scan;
    sp.ws_bytes = L.total - L.scan;
    sp.q_stride = sp.k_stride = sp.v_stride = L.ldq;
    sp.o_stride = (int64_t)H * dv;
    sp.q = skip ? nullptr : qkv_s;
    sp.k = qkv_s + (size_t)H * dk;
    sp.v = qkv_s + (size_t)2 * H * dk;
    sp.log_alpha = la;
    sp.beta = be;
    sp.cu_seqlens = a->cu_seqlens;
    sp.cu_seqlens_host = a->cu_seqlens_host;
    sp.S0 = nullptr;
    sp.o = skip ? nullptr : obuf;
    sp.S_final = a->S_hat + (size_t)l * state_elems;
    sp.err_word = err_word;
    sp.pdl = pdl;
    tr_status st = run_scan(sp, s, [&]() { return mk->mark(s); });
    if (st != TR_OK) return st;
    if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
    if (!skip) {
      float *out = last ? a->x_out : x;
      if (out && output_gate(a)) {
        e = tr::launch_gated_norm(obuf, zbuf, w.o_norm_gain, T, H, dv, rms_eps, s, pdl);
        if (e != cudaSuccess) return cuda_fail(e, "output gate");
        if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
      }
      if (out) {
        tr::ResidEpi rp{};
        rp.x_res = x_in;
        rp.res_is_bf16 = in_bf16;
        rp.x_out = out;
        rp.ld = D;
        if (!runs_ffn(a, l)) fold_next(rp);
        e = tr::launch_gemm_resid(obuf, (int64_t)H * dv, w.W_o, T, D, H * dv, rp, err_word, s,
                                  pdl, &err);
        if (e != cudaSuccess)
          return err.empty() ? cuda_fail(e, "output projection")
                             : fail(TR_ERR_CUDA, "%s", err.c_str());
        if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
      }
    }
    if (runs_ffn(a, l)) {
      // FFN sublayer on the residual the LA sublayer just wrote, in place
      float *xr = last ? a->x_out : x;
      e = tr::launch_rmsnorm(xr, 0, w.ffn_gain, T, D, rms_eps, xhat, s, pdl);
      if (e != cudaSuccess) return cuda_fail(e, "FFN rmsnorm");
      if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
      tr::SwigluEpi sw{};
      sw.h = hmid;
      sw.ld = a->d_ff;
      e = tr::launch_gemm_swiglu(xhat, w.W_gate, w.W_up, T, a->d_ff, D, sw, err_word, s, pdl,
                                 &err);
      if (e != cudaSuccess)
        return err.empty() ? cuda_fail(e, "FFN gate/up projection")
                           : fail(TR_ERR_CUDA, "%s", err.c_str());
      if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
      tr::ResidEpi rp{};
      rp.x_res = xr;
      rp.res_is_bf16 = 0;
      rp.x_out = xr;
      rp.ld = D;
      fold_next(rp);
      e = tr::launch_gemm_resid(hmid, a->d_ff, w.W_down, T, D, a->d_ff, rp, err_word, s, pdl,
                                &err);
      if (e != cudaSuccess)
        return err.empty() ? cuda_fail(e, "FFN down projection")
                           : fail(TR_ERR_CUDA, "%s", err.c_str());
      if (mk->mark(s) != cudaSuccess) return fail(TR_ERR_CUDA, "cudaEventRecord");
    }
  }
  return TR_OK;
}

// ------------------------------------------------------- transition product
// The scan on v = 0 from S0 = I: its final state is the transition product P.
__global__ void set_identity(float *M, int64_t n_mats, int d) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_mats * d) M[(i / d) * d * d + (i % d) * (d + 1)] = 1.f;
}

struct TpLayout {
  size_t v0 = 0, ident = 0, scan = 0, total = 0;
  size_t v0_bytes = 0, ident_bytes = 0;
};

// Scan arguments of the product: d_v = d_k, v from the zero buffer, S0 the identities,
// S_final = P, no readout.
tr_scan_args tp_scan_args(const tr_scan_args *a, float *P, void *v0, float *ident) {
  tr_scan_args b = *a;
  b.d_v = a->d_k;
  b.v = v0;
  b.v_stride = 0;
  b.q = nullptr;
  b.q_stride = 0;
  b.o = nullptr;
  b.S0 = ident;
  b.S_final = P;
  return b;
}

tr_status tp_layout(const tr_scan_args *a, TpLayout *L, tr::ScanLaunch *p) {
  if (!a) return fail(TR_ERR_INVALID_ARG, "args is NULL");
  const size_t esz = a->dtype == TR_DTYPE_BF16 ? 2 : 4;
  const size_t T = a->total_tokens > 0 ? (size_t)a->total_tokens : 0;
  L->v0_bytes = T * (size_t)a->n_heads * (size_t)a->d_k * esz;
  L->ident_bytes = (size_t)(a->n_seqs > 0 ? a->n_seqs : 0) * (size_t)a->n_heads * (size_t)a->d_k *
                   (size_t)a->d_k * sizeof(float);
  size_t off = 0;
  L->v0 = off;    off = align256(off + L->v0_bytes);
  L->ident = off; off = align256(off + L->ident_bytes);
  L->scan = off;
  // placeholders (aligned, non-NULL) to validate the derived scan arguments and size them
  uint8_t *fake = reinterpret_cast<uint8_t *>(static_cast<uintptr_t>(1) << 12);
  tr_scan_args b = tp_scan_args(a, reinterpret_cast<float *>(fake), fake,
                                reinterpret_cast<float *>(fake + 256));
  tr_status st = validate_scan(&b, p);
  if (st != TR_OK) return st;
  L->total = off + scan_ws_bytes(*p);
  return TR_OK;
}

// Extra streams and fork/join events of tr_replay_groups' lanes, per device (created on
// first use, kept for the process; a mutex serialises the calls that use them).
constexpr int kMaxLanes = 4;
struct LaneSet {
  cudaStream_t s[kMaxLanes] = {};
  cudaEvent_t fork = nullptr, join[kMaxLanes] = {};
  bool ready = false;
};
std::mutex g_lane_mu;
LaneSet g_lanes[64];

size_t single_group_bytes(const tr_group_args *groups, int32_t n_groups) {
  size_t need = 0;
  for (int32_t g = 0; g < n_groups; ++g) need = std::max(need, group_layout(&groups[g]).total);
  return need;
}

// The group array, every group and the shared workspace of tr_replay_groups.
tr_status validate_groups(const tr_group_args *groups, int32_t n_groups, const void *ws,
                          size_t ws_bytes) {
  if (n_groups < 0 || (n_groups > 0 && !groups))
    return fail(TR_ERR_INVALID_ARG, "bad group array");
  size_t need = 0;
  for (int32_t g = 0; g < n_groups; ++g) {
    tr_status st = validate_group(&groups[g]);
    if (st != TR_OK) {
      std::string m = g_last_error;
      return fail(st, "group %d: %s", g, m.c_str());
    }
    need = std::max(need, group_layout(&groups[g]).total);
  }
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(TR_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws_bytes, need);
  if (need > 0 && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(TR_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  return TR_OK;
}

}  // namespace

// ============================================================== extern "C"
extern "C" {

const char *tr_last_error(void) { return g_last_error.c_str(); }

tr_status tr_set_wait_limit_ns(uint64_t ns) {
  if (ns > 60000000000ull) return fail(TR_ERR_INVALID_ARG, "wait limit above 60 s");
  tr::g_wait_ns.store(ns ? ns : 4000000000ull);
  return ok();
}

const char *tr_version(void) {
  return "libtr (Tail-Replay GDN tail replay), sm_100a";
}

int64_t tr_tail_len(int64_t m, int64_t r_num, int64_t r_den) {
  if (r_den <= 0 || m < 0) return -1;
  if (m == 0 || r_num <= 0) return 0;
  // ceil(r_num * m / r_den) without overflow for m, r_num < 2^31
  const __int128 num = (__int128)r_num * m;
  int64_t k = (int64_t)((num + r_den - 1) / r_den);
  if (k > m) k = m;
  return k;
}

size_t tr_gdn_scan_workspace_size(const tr_scan_args *args) {
  tr::ScanLaunch p;
  if (validate_scan(args, &p) != TR_OK) return 0;
  return scan_ws_bytes(p);
}

tr_status tr_gdn_scan(const tr_scan_args *args, void *ws, size_t ws_bytes, void *stream) {
  tr::ScanLaunch p;
  tr_status st = validate_scan(args, &p);
  if (st != TR_OK) return st;
  const size_t need = scan_ws_bytes(p);
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(TR_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws_bytes, need);
  if (need > 0 && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(TR_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  p.ws = ws;
  p.ws_bytes = ws_bytes;
  int dev;
  unsigned *errw;
  std::string err;
  if (!device_state(static_cast<cudaStream_t>(stream), &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  p.err_word = errw;
  st = run_scan(p, static_cast<cudaStream_t>(stream));
  return st == TR_OK ? ok() : st;
}

size_t tr_transition_product_workspace_size(const tr_scan_args *args) {
  TpLayout L;
  tr::ScanLaunch p;
  if (tp_layout(args, &L, &p) != TR_OK) return 0;
  return L.total;
}

tr_status tr_transition_product(const tr_scan_args *args, float *P, void *ws, size_t ws_bytes,
                                void *stream) {
  if (!P) return fail(TR_ERR_INVALID_ARG, "P is NULL");
  if (!aligned16(P)) return fail(TR_ERR_ALIGNMENT, "P must be 16-byte aligned");
  TpLayout L;
  tr::ScanLaunch p;
  tr_status st = tp_layout(args, &L, &p);
  if (st != TR_OK) return st;
  if (!ws || ws_bytes < L.total)
    return fail(TR_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws_bytes, L.total);
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(TR_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  uint8_t *base = static_cast<uint8_t *>(ws);
  tr_scan_args b = tp_scan_args(args, P, base + L.v0, reinterpret_cast<float *>(base + L.ident));
  st = validate_scan(&b, &p);
  if (st != TR_OK) return st;
  int dev;
  unsigned *errw;
  std::string err;
  if (!device_state(static_cast<cudaStream_t>(stream), &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (L.v0_bytes) e = cudaMemsetAsync(base + L.v0, 0, L.v0_bytes, s);
  if (e == cudaSuccess && L.ident_bytes) e = cudaMemsetAsync(base + L.ident, 0, L.ident_bytes, s);
  if (e != cudaSuccess) return cuda_fail(e, "transition product setup");
  const int64_t n_mats = (int64_t)args->n_seqs * args->n_heads;
  if (n_mats > 0) {
    const int64_t n = n_mats * args->d_k;
    set_identity<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(reinterpret_cast<float *>(base + L.ident),
                                                              n_mats, args->d_k);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "transition product setup");
  }
  p.ws = base + L.scan;
  p.ws_bytes = ws_bytes - L.scan;
  p.err_word = errw;
  // P is the whole result and, under slow decay, keeps every chunk's rounding: the chunked
  // chain takes the state into its products as a bf16 hi + lo pair
  p.precise_state = true;
  st = run_scan(p, s);
  return st == TR_OK ? ok() : st;
}

size_t tr_replay_group_workspace_size(const tr_group_args *args) {
  if (validate_group(args) != TR_OK) return 0;
  return group_layout(args).total;
}

tr_status tr_replay_group(const tr_group_args *args, void *ws, size_t ws_bytes, void *stream) {
  tr_status st = validate_group(args);
  if (st != TR_OK) return st;
  const size_t need = group_layout(args).total;
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(TR_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws_bytes, need);
  if (need > 0 && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(TR_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  int dev;
  unsigned *errw;
  std::string err;
  if (!device_state(static_cast<cudaStream_t>(stream), &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  st = replay_group_enqueue(args, ws, errw, static_cast<cudaStream_t>(stream));
  return st == TR_OK ? ok() : st;
}

int32_t tr_replay_group_kernel_count(const tr_group_args *args) {
  if (!args || args->n_layers < 1 || args->n_layers > 64) return 0;
  return group_kernel_count(args);
}

const char *tr_replay_group_kernel_names(const tr_group_args *args) {
  g_names.clear();
  if (!args || args->n_layers < 1 || args->n_layers > 64 || !args->layers) return g_names.c_str();
  for (const char *k : group_kernel_names(args)) {
    if (!g_names.empty()) g_names += ',';
    g_names += k;
  }
  return g_names.c_str();
}

tr_status tr_replay_group_profiled(const tr_group_args *args, void *ws, size_t ws_bytes,
                                   void *stream, void *const *events, int32_t n_events) {
  tr_status st = validate_group(args);
  if (st != TR_OK) return st;
  if (!events || n_events < 1 + group_kernel_count(args))
    return fail(TR_ERR_INVALID_ARG, "need %d events, got %d", 1 + group_kernel_count(args),
                n_events);
  for (int32_t i = 0; i < n_events; ++i)
    if (!events[i]) return fail(TR_ERR_INVALID_ARG, "event %d is NULL", i);
  const size_t need = group_layout(args).total;
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(TR_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws_bytes, need);
  if (need > 0 && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(TR_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  int dev;
  unsigned *errw;
  std::string err;
  if (!device_state(static_cast<cudaStream_t>(stream), &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  Marks mk;
  mk.ev = events;
  mk.n = n_events;
  st = replay_group_enqueue(args, ws, errw, static_cast<cudaStream_t>(stream), &mk);
  return st == TR_OK ? ok() : st;
}

size_t tr_replay_groups_workspace_size(const tr_group_args *groups, int32_t n_groups) {
  size_t m = 0;
  for (int32_t g = 0; groups && g < n_groups; ++g)
    m = std::max(m, tr_replay_group_workspace_size(&groups[g]));
  return m;
}

size_t tr_replay_groups_lanes_workspace_size(const tr_group_args *groups, int32_t n_groups,
                                             int32_t lanes) {
  if (lanes < 1 || lanes > kMaxLanes) return 0;
  return (size_t)lanes * align256(tr_replay_groups_workspace_size(groups, n_groups));
}

tr_status tr_replay_groups(const tr_group_args *groups, int32_t n_groups, void *ws,
                           size_t ws_bytes, void *stream) {
  tr_status vst = validate_groups(groups, n_groups, ws, ws_bytes);
  if (vst != TR_OK) return vst;
  int dev;
  unsigned *errw;
  std::string err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!device_state(s, &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  // lanes: as many workspace slices as fit (at most kMaxLanes, at most one per group), none
  // under capture
  const size_t slice = align256(single_group_bytes(groups, n_groups));
  int lanes = slice > 0 ? (int)std::min<size_t>(ws_bytes / slice, kMaxLanes) : 1;
  lanes = std::max(1, std::min(lanes, (int)n_groups));
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (lanes > 1 && (cudaStreamIsCapturing(s, &cs) != cudaSuccess ||
                    cs != cudaStreamCaptureStatusNone || dev < 0 || dev >= 64))
    lanes = 1;
  if (lanes == 1) {
    for (int32_t g = 0; g < n_groups; ++g) {
      tr_status st = replay_group_enqueue(&groups[g], ws, errw, s);
      if (st != TR_OK) return st;
    }
    return ok();
  }
  std::lock_guard<std::mutex> lock(g_lane_mu);
  LaneSet &L = g_lanes[dev];
  if (!L.ready) {
    cudaError_t e = cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming);
    for (int i = 1; e == cudaSuccess && i < kMaxLanes; ++i) {
      e = cudaStreamCreateWithFlags(&L.s[i], cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L.join[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return cuda_fail(e, "lane streams");
    L.ready = true;
  }
  // fork: every extra lane starts after the work already on `stream`
  cudaError_t e = cudaEventRecord(L.fork, s);
  for (int i = 1; e == cudaSuccess && i < lanes; ++i) e = cudaStreamWaitEvent(L.s[i], L.fork, 0);
  if (e != cudaSuccess) return cuda_fail(e, "lane fork");
  tr_status st = TR_OK;
  for (int32_t g = 0; g < n_groups && st == TR_OK; ++g) {
    const int lane = g % lanes;
    st = replay_group_enqueue(&groups[g], static_cast<uint8_t *>(ws) + (size_t)lane * slice, errw,
                              lane == 0 ? s : L.s[lane]);
  }
  // join (also after a failed enqueue, so `stream` never runs ahead of a lane)
  for (int i = 1; i < lanes; ++i) {
    cudaError_t je = cudaEventRecord(L.join[i], L.s[i]);
    if (je == cudaSuccess) je = cudaStreamWaitEvent(s, L.join[i], 0);
    if (je != cudaSuccess && st == TR_OK) st = cuda_fail(je, "lane join");
  }
  return st == TR_OK ? ok() : st;
}

tr_status tr_replay_groups_overlapped(const tr_group_args *groups, int32_t n_groups, void *ws,
                                      size_t ws_bytes, const void *kv_host, void *kv_dev,
                                      size_t kv_bytes, void *stream, void *copy_stream) {
  if (kv_bytes > 0 && (!kv_host || !kv_dev)) return fail(TR_ERR_INVALID_ARG, "KV pointer is NULL");
  if (kv_bytes > 0 && stream == copy_stream)
    return fail(TR_ERR_INVALID_ARG, "the copy needs a stream of its own");
  // every argument is checked before the copy starts, so a rejected call moves no bytes
  tr_status vst = validate_groups(groups, n_groups, ws, ws_bytes);
  if (vst != TR_OK) return vst;
  cudaStream_t s = static_cast<cudaStream_t>(stream), cs = static_cast<cudaStream_t>(copy_stream);
  cudaEvent_t done = nullptr, entry = nullptr;
  if (kv_bytes > 0) {
    // the copy starts after everything already enqueued on `stream` (earlier readers of
    // kv_dev, such as the previous step's attention, finish before it overwrites them)
    cudaError_t e = cudaEventCreateWithFlags(&entry, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(entry, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, entry, 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(kv_dev, kv_host, kv_bytes, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&done, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(done, cs);
    if (entry) cudaEventDestroy(entry);
    if (e != cudaSuccess) {
      if (done) cudaEventDestroy(done);
      return cuda_fail(e, "KV transfer");
    }
  }
  tr_status st = tr_replay_groups(groups, n_groups, ws, ws_bytes, stream);
  if (done) {
    // the join is enqueued even when the replay failed, so the stream never runs ahead of
    // the copy; the event is released once it has completed
    cudaError_t e = cudaStreamWaitEvent(s, done, 0);
    cudaEventDestroy(done);
    if (st == TR_OK && e != cudaSuccess) return cuda_fail(e, "KV transfer join");
  }
  return st == TR_OK ? ok() : st;
}

size_t tr_state_error_workspace_size(int64_t n_mats) {
  // 2 doubles per matrix piece, up to 16 pieces per matrix
  return n_mats > 0 ? align256((size_t)n_mats * 16 * 2 * sizeof(double)) : 0;
}

tr_status tr_state_error(const float *S, const float *S_hat, int64_t n_mats, int32_t d_k,
                         int32_t d_v, double *err_per_mat, double *err_total, void *ws,
                         size_t ws_bytes, void *stream) {
  if (n_mats < 0 || d_k <= 0 || d_v <= 0) return fail(TR_ERR_INVALID_ARG, "bad sizes");
  if (n_mats > 0 && (!S || !S_hat)) return fail(TR_ERR_INVALID_ARG, "S or S_hat is NULL");
  if (!aligned16(S) || !aligned16(S_hat)) return fail(TR_ERR_ALIGNMENT, "S/S_hat alignment");
  const size_t need = tr_state_error_workspace_size(n_mats);
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(TR_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws_bytes, need);
  if (!err_per_mat && !err_total) return ok();
  int dev;
  unsigned *errw;
  std::string err;
  if (!device_state(static_cast<cudaStream_t>(stream), &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  const int64_t elems = (int64_t)d_k * d_v;
  const int splits = tr::state_error_splits(n_mats, elems, (int64_t)(ws_bytes / (2 * sizeof(double))));
  cudaError_t e = tr::launch_state_error(S, S_hat, n_mats, elems, splits,
                                         static_cast<double *>(ws), err_per_mat, err_total,
                                         static_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "state error");
  return ok();
}

tr_status tr_rmsnorm(const void *x, int32_t x_dtype, const float *gain, int64_t n_rows,
                     int32_t d_model, float eps, void *x_hat, void *stream) {
  if (n_rows < 0 || d_model <= 0 || d_model % 8) return fail(TR_ERR_INVALID_ARG, "bad sizes");
  if (x_dtype != TR_DTYPE_F32 && x_dtype != TR_DTYPE_BF16) return fail(TR_ERR_DTYPE, "x_dtype");
  if (n_rows > 0 && (!x || !x_hat)) return fail(TR_ERR_INVALID_ARG, "x or x_hat is NULL");
  if (!aligned16(x) || !aligned16(x_hat) || (gain && !aligned16(gain)))
    return fail(TR_ERR_ALIGNMENT, "x/x_hat/gain must be 16-byte aligned");
  cudaError_t e = tr::launch_rmsnorm(x, x_dtype == TR_DTYPE_BF16, gain, n_rows, d_model,
                                     eps > 0.f ? eps : 1e-6f, x_hat,
                                     static_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm");
  return ok();
}

tr_status tr_in_projection(const void *x_hat, const void *W_in, int64_t n_tokens, int32_t d_model,
                           int32_t n_heads, int32_t d_k, int32_t d_v, uint32_t flags,
                           float norm_eps, void *qkv, float *log_alpha, float *beta,
                           void *stream) {
  if (n_tokens < 0 || n_tokens > 0x7fffffffLL || d_model <= 0 || n_heads <= 0)
    return fail(TR_ERR_INVALID_ARG, "bad sizes");
  if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128))
    return fail(TR_ERR_UNSUPPORTED, "d_k/d_v must be 64 or 128");
  if (d_model % 64) return fail(TR_ERR_UNSUPPORTED, "d_model must be a multiple of 64");
  if (flags & ~(unsigned)TR_SKIP_LAST_OUTPUT) return fail(TR_ERR_INVALID_ARG, "flags");
  if (!x_hat || !W_in || !qkv || !log_alpha || !beta)
    return fail(TR_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(x_hat) || !aligned16(W_in) || !aligned16(qkv))
    return fail(TR_ERR_ALIGNMENT, "x_hat/W_in/qkv must be 16-byte aligned");
  int dev;
  unsigned *errw;
  std::string err;
  if (!device_state(static_cast<cudaStream_t>(stream), &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  const int n_in = 2 * n_heads * d_k + n_heads * d_v + 2 * n_heads;
  tr::InProjEpi ep{};
  ep.qkv = static_cast<__nv_bfloat16 *>(qkv);
  ep.ldq = 2 * (int64_t)n_heads * d_k + (int64_t)n_heads * d_v;
  ep.log_alpha = log_alpha;
  ep.beta = beta;
  ep.H = n_heads;
  ep.dk = d_k;
  ep.dv = d_v;
  ep.col_offset = (flags & TR_SKIP_LAST_OUTPUT) ? n_heads * d_k : 0;
  ep.norm_eps = norm_eps > 0.f ? norm_eps : 1e-6f;
  const void *Wb = static_cast<const __nv_bfloat16 *>(W_in) + (size_t)ep.col_offset * d_model;
  cudaError_t e = tr::launch_gemm_inproj(x_hat, Wb, (int)n_tokens, n_in - ep.col_offset, d_model,
                                         ep, errw, static_cast<cudaStream_t>(stream), true, &err);
  if (e != cudaSuccess)
    return err.empty() ? cuda_fail(e, "input projection") : fail(TR_ERR_CUDA, "%s", err.c_str());
  return ok();
}

tr_status tr_out_projection(const void *o, int64_t o_stride, const void *W_o, const void *x_res,
                            int32_t x_res_dtype, int64_t n_tokens, int32_t d_model, int32_t hv,
                            float *x_out, void *stream) {
  if (n_tokens < 0 || n_tokens > 0x7fffffffLL || d_model <= 0 || hv <= 0)
    return fail(TR_ERR_INVALID_ARG, "bad sizes");
  if (d_model % 64 || hv % 64) return fail(TR_ERR_UNSUPPORTED, "d_model and H*d_v must be multiples of 64");
  if (x_res_dtype != TR_DTYPE_F32 && x_res_dtype != TR_DTYPE_BF16)
    return fail(TR_ERR_DTYPE, "x_res_dtype");
  if (!o || !W_o || !x_res || !x_out) return fail(TR_ERR_INVALID_ARG, "a required pointer is NULL");
  const int64_t ld = o_stride ? o_stride : hv;
  if (ld < hv || (ld * 2) % 16) return fail(TR_ERR_ALIGNMENT, "o_stride");
  if (!aligned16(o) || !aligned16(W_o) || !aligned16(x_res) || !aligned16(x_out))
    return fail(TR_ERR_ALIGNMENT, "o/W_o/x_res/x_out must be 16-byte aligned");
  int dev;
  unsigned *errw;
  std::string err;
  if (!device_state(static_cast<cudaStream_t>(stream), &dev, &errw, &err)) return fail(TR_ERR_CUDA, "%s", err.c_str());
  tr::ResidEpi rp{};
  rp.x_res = x_res;
  rp.res_is_bf16 = x_res_dtype == TR_DTYPE_BF16;
  rp.x_out = x_out;
  rp.ld = d_model;
  cudaError_t e = tr::launch_gemm_resid(o, ld, W_o, (int)n_tokens, d_model, hv, rp, errw,
                                        static_cast<cudaStream_t>(stream), true, &err);
  if (e != cudaSuccess)
    return err.empty() ? cuda_fail(e, "output projection") : fail(TR_ERR_CUDA, "%s", err.c_str());
  return ok();
}

tr_status tr_check(void *stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream");
  unsigned word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, g_err_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (word) {
    cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero));
    if (word & (tr::ERRBIT_GEMM_TIMEOUT | tr::ERRBIT_SCAN_TIMEOUT))
      return fail(TR_ERR_TIMEOUT, "a kernel gave up a bounded wait (error word 0x%x)", word);
    return fail(TR_ERR_CUDA, "device error word 0x%x", word);
  }
  return ok();
}

}  // extern "C"
