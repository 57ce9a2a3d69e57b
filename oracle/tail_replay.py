"""fp64 restatement of the Tail-Replay hot path (test infrastructure only).

Citations name the page and the section/equation on it:
  RN = "Tail-Replay reading notes" (cc.laoqi.cc page), GS = "Tail-Replay
  technical summary" (gist.science page).

Readings where the pages are silent (the GDN layer internals are never given;
RN section 2.3 says no model dimensions are to be made up from Eq. (1)):
  * state layout M = S^T, [d_k][d_v]; readout o_t = scale * M_t^T q_t after the
    update of token t;
  * per LA layer: RMSNorm (eps 1e-6, gain ones unless given) -> one projection
    x_hat W_in^T = [q | k | v | a_alpha | a_beta] (no bias, no short
    convolution, no activation on v) -> q and k L2-normalised per head
    (x / sqrt(sum x^2 + 1e-6)) -> alpha = exp(-softplus(a_alpha)),
    beta = sigmoid(a_beta) -> Eq. (1) scan -> x <- x + o W_o^T;
  * the Gated DeltaNet details the pages leave out, each optional: a short causal
    depthwise convolution + silu over the bf16 q, k, v projections (zero
    history at the tail start), per-head gate parameters A_log and dt_bias,
    and a gated RMSNorm of the readout (z rows appended to W_in after v);
  * the FFN sublayer: where a layer carries FFN weights, a dense SwiGLU with its
    own RMSNorm, x <- x + (silu(x_hat W_gate^T) * x_hat W_up^T) W_down^T, runs
    after the LA sublayer, except after a group's last LA layer (RN section 2.5,
    the tail-FFN skip); a layer without FFN weights passes the residual after its
    LA sublayer straight to the next LA layer;
  * bf16 cast points of the boundary (``emulate_casts``): the projection
    operands x_hat and o (and the FFN's pre-norm output and hidden activation)
    and the stored q, k, v are rounded to bf16
    (round-to-nearest-even); everything else stays fp64 here.  For the LA layers
    after a group's first, the RMSNorm's 1/rms factor sits after the projection
    (``fold_norm``): the operand rounded to bf16 is x * gain, and the projection's
    outputs are multiplied by the row's 1/rms, the same value in exact arithmetic
    with the bf16 rounding taken before the scale (the implementation computes the
    norm inside the residual and projection GEMMs there).
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import numpy as np

from . import _build

_lib = None


def _scan_lib():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        f = lib.oracle_gdn_scan_f64
        P = ctypes.c_void_p
        f.argtypes = [ctypes.c_int64] * 4 + [P] * 7 + [ctypes.c_double, P, P, ctypes.c_int]
        f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact fp64 values of an array-like (bf16/fp32 torch tensors included)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------- a0
def tail_len(m: int, r_num: int, r_den: int) -> int:
    """k = ceil(r * m) with r = r_num / r_den, in integers, clamped to [0, m].

    RN section 2.1, symbol table: k = ceil(r m) replayed tokens, r in {0.05, 0.10}
    in the experiments.  Integer arithmetic avoids 0.07 * 100 -> 7.000000000000001
    rounding up to 8.
    """
    m, r_num, r_den = int(m), int(r_num), int(r_den)
    if r_den <= 0:
        raise ValueError("r_den must be positive")
    if m <= 0 or r_num <= 0:
        return 0
    k = -((-r_num * m) // r_den)
    return max(0, min(m, k))


def tail_rows(m: int, k: int) -> Tuple[int, int]:
    """0-based half-open row range of the tail h_{m-k+1..m} (RN section 2.2, step 2)."""
    if not 0 <= k <= m:
        raise ValueError("need 0 <= k <= m")
    return m - k, m


# ------------------------------------------------------------------- cast points
def bf16_round(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64.

    Goes through fp32 first (round-to-nearest) and then keeps the top 16 bits of
    the fp32 pattern with round-to-nearest-even, as a device fp32 -> bf16
    conversion does.
    """
    f = np.ascontiguousarray(_f64(x), dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(f)
    out = r.astype(np.uint32).view(np.float32).astype(np.float64)
    if nan.any():
        out[nan] = np.nan
    return out


# ------------------------------------------------------------------------- a2
def rmsnorm(x, gain=None, eps: float = 1e-6) -> np.ndarray:
    """x_hat = x / sqrt(mean_j x_j^2 + eps) * gain, per row.

    Not on the pages (layer internals are never given); the RMSNorm in front of
    each LA layer is the reading stated in the module docstring.
    """
    x = _f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if gain is not None:
        y = y * _f64(gain)
    return y


# ------------------------------------------------------------------------- a3
def in_projection(x_hat, W_in, n_heads: int, d_k: int, d_v: int, output_gate: bool = False):
    """[q | k | v | a_alpha | a_beta] = x_hat W_in^T, split per head.

    W_in is [2 H d_k + H d_v + 2 H, D] (output features x input features).
    Reading (pages silent): one bias-free projection.  With ``output_gate`` W_in
    has H d_v more rows, [q | k | v | z | a_alpha | a_beta], and z [T, H, d_v]
    (the output gate's input) is returned after v.
    """
    x_hat = _f64(x_hat)
    W = _f64(W_in)
    y = x_hat @ W.T
    T = y.shape[0]
    H = n_heads
    o = 0
    q = y[:, o:o + H * d_k].reshape(T, H, d_k); o += H * d_k
    k = y[:, o:o + H * d_k].reshape(T, H, d_k); o += H * d_k
    v = y[:, o:o + H * d_v].reshape(T, H, d_v); o += H * d_v
    z = None
    if output_gate:
        z = y[:, o:o + H * d_v].reshape(T, H, d_v); o += H * d_v
    a_alpha = y[:, o:o + H]; o += H
    a_beta = y[:, o:o + H]; o += H
    assert o == W.shape[0]
    if output_gate:
        return q, k, v, z, a_alpha, a_beta
    return q, k, v, a_alpha, a_beta


# ----------------------------------------------------------- a3b short convolution
def short_conv(x, w, cu_seqlens) -> np.ndarray:
    """y_t[c] = silu(sum_j w[c, j] x_{t-W+1+j}[c]) per packed sequence, zero history.

    Reading (the pages give no layer internals; this is the Gated DeltaNet layer's
    short causal depthwise convolution): ``w`` [C, W], tap W-1 weighs the current
    token; rows before a sequence's first token are zero (the replay starts every
    state at zero, RN section 2.2 step 2, the convolution's included).
    """
    x = _f64(x)
    w = _f64(w)
    cu = [int(c) for c in cu_seqlens]
    W = w.shape[1]
    y = np.zeros_like(x)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        xp = np.concatenate([np.zeros((W - 1, x.shape[1])), x[a:b]], 0)
        acc = np.zeros((b - a, x.shape[1]))
        for j in range(W):
            acc += w[:, j][None, :] * xp[j:j + b - a]
        y[a:b] = acc
    return silu(y)


def conv_state(x, width: int, cu_seqlens) -> np.ndarray:
    """[N, W-1, C]: each sequence's last W-1 convolution inputs, oldest first, zero where
    the sequence is shorter (the state the convolution carries to the next token)."""
    x = _f64(x)
    cu = [int(c) for c in cu_seqlens]
    out = np.zeros((len(cu) - 1, width - 1, x.shape[1]))
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        for i in range(width - 1):
            t = b - (width - 1) + i
            if t >= a:
                out[s, i] = x[t]
    return out


def gated_rmsnorm(o, z, gain=None, eps: float = 1e-6) -> np.ndarray:
    """o / sqrt(mean_{d_v} o^2 + eps) * gain * silu(z), per token and head.

    Reading (pages silent; the Gated DeltaNet layer's output gate and norm): the
    readout of each head is RMS-normalised over d_v, scaled by a gain shared by the
    heads ([d_v], ones when None) and gated by silu of a projection z of x_hat.
    """
    o = _f64(o)
    z = _f64(z)
    r = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    if gain is not None:
        r = r * _f64(gain)
    return r * silu(z)


# ------------------------------------------------------------------------- a4
def l2_normalize(x, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(sum x^2 + eps) along the last axis.

    RN section 2.3 (after Eq. (1)): unit-norm keys with beta in [0, 2] make
    I - beta k k^T non-expansive; q is normalised the same way (reading).
    """
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def gates(a_alpha, a_beta, A_log=None, dt_bias=None):
    """log alpha = -exp(A_log) softplus(a_alpha + dt_bias), beta = sigmoid(a_beta).

    RN section 2.3 only fixes alpha in (0, 1]; the exp(-softplus) form gives
    alpha in (0, 1) and beta in (0, 1), inside the [0, 2] range of the
    non-expansive condition.  softplus(a) = max(a, 0) + log1p(exp(-|a|)) is the
    overflow-free form of log(1 + e^a).  The per-head A_log and dt_bias [H] of the
    Gated DeltaNet layer are optional (None: A_log = 0, dt_bias = 0).
    """
    a = _f64(a_alpha)
    b = _f64(a_beta)
    if dt_bias is not None:
        a = a + _f64(dt_bias)[None, :]
    softplus = np.maximum(a, 0.0) + np.log1p(np.exp(-np.abs(a)))
    log_alpha = -softplus
    if A_log is not None:
        log_alpha = log_alpha * np.exp(_f64(A_log))[None, :]
    beta = np.where(b >= 0, 1.0 / (1.0 + np.exp(-np.abs(b))),
                    np.exp(-np.abs(b)) / (1.0 + np.exp(-np.abs(b))))
    return log_alpha, beta


# ------------------------------------------------------------------------- a5
def gdn_scan(q, k, v, log_alpha, beta, cu_seqlens, S0=None, scale: float = 1.0,
             want_o: bool = True, normalize_qk: bool = False, norm_eps: float = 1e-6,
             n_threads: Optional[int] = None):
    """Eq. (1) of RN section 2.3, token by token from S0 (zero when None).

    Returns (o [T, H, d_v] or None, S_final [N, H, d_k, d_v]) in the M = S^T
    layout.  With ``normalize_qk`` q and k are first L2-normalised per head
    (step a4).  The recurrence itself runs in the plain C file eq1_scan.c.
    """
    q = _f64(q) if q is not None else None
    k = _f64(k)
    if normalize_qk:
        k = l2_normalize(k, norm_eps)
        if q is not None:
            q = l2_normalize(q, norm_eps)
    v = _f64(v)
    la = _f64(log_alpha)
    b = _f64(beta)
    cu = np.ascontiguousarray(_f64(cu_seqlens).astype(np.int64))
    T, H, dk = k.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("bad cu_seqlens")
    S = np.zeros((N, H, dk, dv), dtype=np.float64)
    o = np.zeros((T, H, dv), dtype=np.float64) if want_o else None
    if want_o and q is None:
        raise ValueError("q is needed for the readout")
    qc = np.ascontiguousarray(q) if q is not None else None
    kc, vc = np.ascontiguousarray(k), np.ascontiguousarray(v)
    lac, bc = np.ascontiguousarray(la), np.ascontiguousarray(b)
    S0c = np.ascontiguousarray(_f64(S0)) if S0 is not None else None
    if S0c is not None and S0c.shape != S.shape:
        raise ValueError("S0 shape")
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    P = lambda a: a.ctypes.data_as(ctypes.c_void_p) if a is not None else None
    rc = _scan_lib().oracle_gdn_scan_f64(N, H, dk, dv, P(cu), P(qc), P(kc), P(vc), P(lac), P(bc),
                                         P(S0c), float(scale), P(o), P(S), int(n_threads))
    if rc != 0:
        raise RuntimeError("oracle scan rejected its arguments")
    return o, S


def transition_product(k, log_alpha, beta, cu_seqlens):
    """P = T_t ... T_1 over each sequence's tokens, per head, T_i = alpha_i (I - beta_i k_i k_i^T).

    RN section 2.3 writes the tail's error as E_m = (T_m ... T_{a+1}) S_a; HYPIC (abstract)
    caches this product as the segment transition operator.  In the M = S^T layout a
    state M_0 before the sequence becomes P M_0 + M_hat after it (M_hat: the zero-start
    state of the scan).  Returns [N, H, d_k, d_k] fp64.  Each step applies T_i to the
    running product as the rank-one update alpha_i (P - beta_i k_i (k_i^T P)), which is
    T_i P without forming T_i.
    """
    k = _f64(k)
    la = _f64(log_alpha)
    b = _f64(beta)
    cu = _f64(cu_seqlens).astype(np.int64)
    T, H, dk = k.shape
    N = cu.shape[0] - 1
    out = np.zeros((N, H, dk, dk), dtype=np.float64)
    for n in range(N):
        P = np.broadcast_to(np.eye(dk), (H, dk, dk)).copy()
        for t in range(int(cu[n]), int(cu[n + 1])):
            kt = k[t]                                   # [H, dk]
            kP = np.einsum('hd,hde->he', kt, P)         # k^T P, [H, dk]
            P = np.exp(la[t])[:, None, None] * (P - b[t][:, None, None] * kt[:, :, None] * kP[:, None, :])
        out[n] = P
    return out


# ------------------------------------------------------------------------- a6
def out_projection_residual(x, o, W_o) -> np.ndarray:
    """x + o W_o^T with o flattened to [T, H d_v] and W_o [D, H d_v].

    Reading (pages silent on the layer internals): the LA layer's attention
    sublayer adds its output projection to the residual stream.
    """
    x = _f64(x)
    o = _f64(o)
    T = o.shape[0]
    return x + o.reshape(T, -1) @ _f64(W_o).T


# ------------------------------------------------------------------------ a6b
def silu(z) -> np.ndarray:
    """z * sigmoid(z) = z / (1 + exp(-z)), elementwise (-0 where exp(-z) overflows)."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def ffn_residual(x, W_gate, W_up, W_down, ffn_gain=None, rms_eps: float = 1e-6,
                 emulate_casts: bool = True) -> np.ndarray:
    """x + (silu(x_hat W_gate^T) * (x_hat W_up^T)) W_down^T, x_hat = RMSNorm(x) * ffn_gain.

    RN section 2.5: inside a group, the FFN after each LA layer but the last still
    runs, because it makes the next LA layer's input.  Reading (the pages never give
    the FFN's form): a dense SwiGLU sublayer with its own pre-norm and a residual
    add, W_gate and W_up [d_ff, D], W_down [D, d_ff], no biases.  Cast points: the
    pre-norm output and the hidden activation are rounded to bf16 (the GEMM
    operands); the two products and the residual stay fp64 here.
    """
    x = _f64(x)
    cast = bf16_round if emulate_casts else (lambda a: a)
    x_hat = cast(rmsnorm(x, ffn_gain, rms_eps))
    g = x_hat @ _f64(W_gate).T
    u = x_hat @ _f64(W_up).T
    hmid = cast(silu(g) * u)
    return x + hmid @ _f64(W_down).T


# ---------------------------------------------------------------------- a2..a6
def replay_layer(x, W_in, W_o, rms_gain, cu_seqlens, n_heads: int, d_k: int, d_v: int,
                 want_output: bool = True, emulate_casts: bool = True,
                 rms_eps: float = 1e-6, norm_eps: float = 1e-6, n_threads=None, ffn=None,
                 conv_w=None, A_log=None, dt_bias=None, output_gate: bool = False,
                 o_norm_gain=None, conv_states: Optional[list] = None,
                 fold_norm: bool = False):
    """One LA layer of the replay from a zero state: returns (S_hat, x_next or None).

    ``fold_norm``: the RMSNorm's cast point of the layers after a group's first (module
    docstring): x_hat = bf16(x * gain), and the projection's outputs times 1/rms.

    ``ffn`` = (W_gate, W_up, W_down, ffn_gain) runs the FFN sublayer on x_next
    (``ffn_residual``); None leaves it out.  The Gated DeltaNet details the pages
    leave out are options: ``conv_w`` [2 H d_k + H d_v, W] the short convolution
    over the bf16 q, k, v projections (``short_conv``, zero history; its state
    is appended to ``conv_states`` when a list is given), ``A_log``/``dt_bias``
    the gate parameters (``gates``), ``output_gate`` the gated RMSNorm of the
    bf16 readout (``gated_rmsnorm`` with gain ``o_norm_gain``, eps = rms_eps,
    rounded to bf16 again).
    """
    x = _f64(x)
    cast = bf16_round if emulate_casts else (lambda a: a)
    if fold_norm:
        # RMSNorm(x) W_in^T = (1 / rms) ((x * gain) W_in^T), the rounding taken on x * gain
        inv_rms = 1.0 / np.sqrt(np.mean(x * x, axis=-1) + rms_eps)
        x_g = x * _f64(rms_gain) if rms_gain is not None else x
        proj = in_projection(cast(x_g), W_in, n_heads, d_k, d_v, output_gate)
        proj = tuple(a * (inv_rms[:, None, None] if a.ndim == 3 else inv_rms[:, None])
                     for a in proj)
    else:
        x_hat = cast(rmsnorm(x, rms_gain, rms_eps))
        proj = in_projection(x_hat, W_in, n_heads, d_k, d_v, output_gate)
    if output_gate:
        q, k, v, z, a_alpha, a_beta = proj
    else:
        q, k, v, a_alpha, a_beta = proj
    if conv_w is not None:
        T = q.shape[0]
        nq, nk = n_heads * d_k, 2 * n_heads * d_k
        pre = cast(np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], 1))
        if conv_states is not None:
            conv_states.append(conv_state(pre, _f64(conv_w).shape[1], cu_seqlens))
        y = short_conv(pre, conv_w, cu_seqlens)
        q = y[:, :nq].reshape(q.shape)
        k = y[:, nq:nk].reshape(k.shape)
        v = y[:, nk:].reshape(v.shape)
    q = cast(l2_normalize(q, norm_eps))
    k = cast(l2_normalize(k, norm_eps))
    v = cast(v)
    log_alpha, beta = gates(a_alpha, a_beta, A_log, dt_bias)
    o, S_hat = gdn_scan(q, k, v, log_alpha, beta, cu_seqlens, None, 1.0, want_o=want_output,
                        n_threads=n_threads)
    x_next = None
    if want_output:
        o = cast(o)
        if output_gate:
            o = cast(gated_rmsnorm(o, cast(z), o_norm_gain, rms_eps))
        x_next = out_projection_residual(x, o, W_o)
        if ffn is not None:
            W_gate, W_up, W_down, ffn_gain = ffn
            x_next = ffn_residual(x_next, W_gate, W_up, W_down, ffn_gain, rms_eps, emulate_casts)
    return S_hat, x_next


def replay_group(h_tail, cu_seqlens, layers: Sequence, n_heads: int, d_k: int, d_v: int,
                 emulate_casts: bool = True, skip_last_output: bool = False,
                 rms_eps: float = 1e-6, norm_eps: float = 1e-6, n_threads=None,
                 skip_last_ffn: bool = True, output_gate: bool = False,
                 conv_states: Optional[list] = None):
    """Replay one group's LA layers over the packed tails (RN section 2.2 steps 2-3).

    Every LA state of the group starts at zero at the tail start (step 2, GS
    "Key Mechanisms": initialise the replay state to zero); the tail hiddens
    h_{m-k+1..m} go through the group's LA layers in order (step 3), each layer
    feeding the next.  ``layers`` is a sequence of objects with W_in, W_o and
    rms_gain, and W_gate, W_up, W_down, ffn_gain where the layer has an FFN
    sublayer (W_gate None or absent: no FFN).  Returns (S_hat [L, N, H, d_k, d_v],
    x_out [T, D] or None).
    With ``skip_last_ffn`` the last layer's FFN is not run (RN section 2.5, the
    tail-FFN skip: the next group starts from its own cached FA output, so that
    FFN output rebuilds no state); x_out is then the residual after the last LA
    sublayer.  With ``skip_last_output`` the last layer's readout and output
    projection are not computed either (the same argument one sublayer earlier),
    and x_out is None.
    The optional Gated DeltaNet details (``replay_layer``) come from the layer
    objects' conv_w, A_log, dt_bias and o_norm_gain (absent or None: not used) and
    ``output_gate`` (every layer's W_in then carries the z rows); a list passed as
    ``conv_states`` receives each layer's convolution state [N, W-1, C].
    """
    x = _f64(h_tail)
    S_all = []
    L = len(layers)
    for i, lw in enumerate(layers):
        want = not (skip_last_output and i == L - 1)
        ffn = None
        if getattr(lw, "W_gate", None) is not None and not (skip_last_ffn and i == L - 1):
            ffn = (lw.W_gate, lw.W_up, lw.W_down, getattr(lw, "ffn_gain", None))
        S_hat, x_next = replay_layer(x, lw.W_in, lw.W_o, lw.rms_gain, cu_seqlens, n_heads, d_k, d_v,
                                     want_output=want, emulate_casts=emulate_casts,
                                     rms_eps=rms_eps, norm_eps=norm_eps, n_threads=n_threads,
                                     ffn=ffn, conv_w=getattr(lw, "conv_w", None),
                                     A_log=getattr(lw, "A_log", None),
                                     dt_bias=getattr(lw, "dt_bias", None),
                                     output_gate=output_gate,
                                     o_norm_gain=getattr(lw, "o_norm_gain", None),
                                     conv_states=conv_states, fold_norm=i > 0)
        S_all.append(S_hat)
        x = x_next
    return np.stack(S_all, 0), x


# ------------------------------------------------------------------------- a8
def state_error(S, S_hat):
    """||S - S_hat||_F / ||S||_F per d_k x d_v matrix and over the whole tensor.

    RN section 2.3 defines E_m = S_m - S_hat_m; the relative Frobenius norm is
    the measure the workloads ask for.  Reading for ||S|| = 0: the error is 0
    when S_hat is 0 too, else +inf.
    """
    S = _f64(S)
    Sh = _f64(S_hat)
    dk, dv = S.shape[-2:]
    d = (S - Sh).reshape(-1, dk * dv)
    s = S.reshape(-1, dk * dv)
    num = np.sum(d * d, axis=1)
    den = np.sum(s * s, axis=1)

    def ratio(n, dd):
        with np.errstate(divide="ignore", invalid="ignore"):
            r = np.sqrt(n / dd)
        r = np.where(dd > 0, r, np.where(n > 0, np.inf, 0.0))
        return r

    per = ratio(num, den)
    tot = float(ratio(np.array([num.sum()]), np.array([den.sum()]))[0])
    return per, tot
