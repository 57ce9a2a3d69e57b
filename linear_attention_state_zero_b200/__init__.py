"""Tail-Replay on B200: zero-initialised tail replay of Gated DeltaNet layers.

Python binding of ``libtr.so`` (declared in ``include/tr.h``).  This module only
marshals arguments: it checks devices, dtypes and strides of torch tensors,
allocates outputs and workspaces with PyTorch, and calls the C ABI.  Every step
of the computation runs in the library's CUDA kernels; there is no CPU path.
Importing fails if the library has not been built
(``python linear_attention_state_zero_b200/_build.py``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtr.so")

TR_OK = 0
TR_DTYPE_F32, TR_DTYPE_BF16 = 0, 1
TR_NORMALIZE_QK, TR_SKIP_LAST_OUTPUT, TR_SCAN_RECURRENT, TR_SKIP_LAST_FFN = 1, 2, 4, 8
TR_OUTPUT_GATE = 16
TR_SCAN_STALL_TEST = 256

STATUS_NAMES = {0: "TR_OK", 1: "TR_ERR_INVALID_ARG", 2: "TR_ERR_SHAPE", 3: "TR_ERR_DTYPE",
                4: "TR_ERR_ALIGNMENT", 5: "TR_ERR_UNSUPPORTED", 6: "TR_ERR_WORKSPACE",
                7: "TR_ERR_CUDA", 8: "TR_ERR_TIMEOUT"}

c_i32, c_i64, c_u32, c_f32, c_vp, c_sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                          ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t)


class ScanArgs(ctypes.Structure):
    _fields_ = [("n_seqs", c_i32), ("n_heads", c_i32), ("d_k", c_i32), ("d_v", c_i32),
                ("total_tokens", c_i64), ("dtype", c_i32), ("flags", c_u32), ("scale", c_f32),
                ("q_stride", c_i64), ("k_stride", c_i64), ("v_stride", c_i64),
                ("q", c_vp), ("k", c_vp), ("v", c_vp), ("log_alpha", c_vp), ("beta", c_vp),
                ("cu_seqlens", c_vp), ("cu_seqlens_host", c_vp), ("S0", c_vp), ("o", c_vp),
                ("S_final", c_vp)]


class LALayer(ctypes.Structure):
    _fields_ = [("rms_gain", c_vp), ("W_in", c_vp), ("W_o", c_vp), ("ffn_gain", c_vp),
                ("W_gate", c_vp), ("W_up", c_vp), ("W_down", c_vp), ("conv_w", c_vp),
                ("A_log", c_vp), ("dt_bias", c_vp), ("o_norm_gain", c_vp)]


class GroupArgs(ctypes.Structure):
    _fields_ = [("n_seqs", c_i32), ("n_heads", c_i32), ("d_k", c_i32), ("d_v", c_i32),
                ("d_model", c_i32), ("n_layers", c_i32), ("total_tokens", c_i64),
                ("flags", c_u32), ("rms_eps", c_f32), ("norm_eps", c_f32), ("d_ff", c_i32),
                ("h_tail", c_vp), ("cu_seqlens", c_vp), ("cu_seqlens_host", c_vp),
                ("layers", ctypes.POINTER(LALayer)), ("S_hat", c_vp), ("x_out", c_vp),
                ("conv_width", c_i32), ("conv_state", c_vp)]


# exported symbol -> (restype, argtypes)
_SIGNATURES = {
    "tr_last_error": (ctypes.c_char_p, []),
    "tr_version": (ctypes.c_char_p, []),
    "tr_tail_len": (c_i64, [c_i64, c_i64, c_i64]),
    "tr_gdn_scan_workspace_size": (c_sz, [ctypes.POINTER(ScanArgs)]),
    "tr_gdn_scan": (ctypes.c_int, [ctypes.POINTER(ScanArgs), c_vp, c_sz, c_vp]),
    "tr_transition_product_workspace_size": (c_sz, [ctypes.POINTER(ScanArgs)]),
    "tr_transition_product": (ctypes.c_int, [ctypes.POINTER(ScanArgs), c_vp, c_vp, c_sz, c_vp]),
    "tr_replay_group_workspace_size": (c_sz, [ctypes.POINTER(GroupArgs)]),
    "tr_replay_group": (ctypes.c_int, [ctypes.POINTER(GroupArgs), c_vp, c_sz, c_vp]),
    "tr_replay_groups_overlapped": (ctypes.c_int, [ctypes.POINTER(GroupArgs), c_i32, c_vp, c_sz,
                                                   c_vp, c_vp, c_sz, c_vp, c_vp]),
    "tr_replay_group_kernel_count": (c_i32, [ctypes.POINTER(GroupArgs)]),
    "tr_replay_group_kernel_names": (ctypes.c_char_p, [ctypes.POINTER(GroupArgs)]),
    "tr_replay_group_profiled": (ctypes.c_int, [ctypes.POINTER(GroupArgs), c_vp, c_sz, c_vp,
                                                ctypes.POINTER(c_vp), c_i32]),
    "tr_replay_groups_workspace_size": (c_sz, [ctypes.POINTER(GroupArgs), c_i32]),
    "tr_replay_groups_lanes_workspace_size": (c_sz, [ctypes.POINTER(GroupArgs), c_i32, c_i32]),
    "tr_replay_groups": (ctypes.c_int, [ctypes.POINTER(GroupArgs), c_i32, c_vp, c_sz, c_vp]),
    "tr_state_error_workspace_size": (c_sz, [c_i64]),
    "tr_state_error": (ctypes.c_int, [c_vp, c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_sz,
                                      c_vp]),
    "tr_state_error_noalloc": (ctypes.c_int, [c_vp, c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp]),
    "tr_rmsnorm": (ctypes.c_int, [c_vp, c_i32, c_vp, c_i64, c_i32, c_f32, c_vp, c_vp]),
    "tr_in_projection": (ctypes.c_int, [c_vp, c_vp, c_i64, c_i32, c_i32, c_i32, c_i32, c_u32,
                                        c_f32, c_vp, c_vp, c_vp, c_vp]),
    "tr_out_projection": (ctypes.c_int, [c_vp, c_i64, c_vp, c_vp, c_i32, c_i64, c_i32, c_i32,
                                         c_vp, c_vp]),
    "tr_check": (ctypes.c_int, [c_vp]),
    "tr_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libtr.so is not built (%s); run "
                          "`python linear_attention_state_zero_b200/_build.py`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


class TrError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.tr_last_error().decode(errors="replace")
        super().__init__("%s: %s (%s)" % (where, STATUS_NAMES.get(status, status), msg))
        self.status = status


def _ok(st: int, where: str) -> None:
    if st != TR_OK:
        raise TrError(st, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream, device=None) -> Optional[int]:
    """The raw handle of `stream`, or of the current stream of `device` when None."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TR_DTYPE_BF16
    if t.dtype == torch.float32:
        return TR_DTYPE_F32
    raise TypeError("unsupported dtype %s" % t.dtype)


def _need_cuda(*ts):
    """Every given tensor lives on one CUDA device; returns that device (None if no tensor).

    The library launches on the current device, so each call below runs with this device
    made current (``torch.cuda.device``) and on its current stream unless one is given."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("tensors must live on one device (%s and %s)" % (dev, t.device))
    return dev


def _need_layout(name, t, dtype, shape=None):
    """A weight or parameter tensor must be contiguous, of the dtype the kernels read, and
    (where given) of the expected shape; None passes."""
    if t is None:
        return
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError("%s must be a contiguous %s tensor, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def seqlens(cu_seqlens, device):
    """cu_seqlens prepared once as (host int32 tensor, device int32 tensor); the calls below
    accept this pair in place of cu_seqlens and then copy nothing."""
    return _seqlens(cu_seqlens, device)


def _seqlens(cu_seqlens, device):
    """(host int32 tensor, device int32 tensor) for a cu_seqlens given either way."""
    if isinstance(cu_seqlens, tuple) and len(cu_seqlens) == 2:
        host, dev = cu_seqlens
        if host.device.type != "cpu" or dev.device != torch.device(device) or \
                host.dtype != torch.int32 or dev.dtype != torch.int32:
            raise ValueError("a (host, device) cu_seqlens pair must hold int32 tensors")
        return host, dev
    cu = torch.as_tensor(cu_seqlens, dtype=torch.int32)
    host = cu.cpu().contiguous()
    dev = cu.to(device).contiguous() if not (cu.is_cuda and cu.is_contiguous()) else cu
    return host, dev


def version() -> str:
    return lib.tr_version().decode()


def tail_len(m: int, r_num: int, r_den: int) -> int:
    """k = ceil(r m) for r = r_num / r_den, exact, clamped to [0, m] (C ABI, host-only)."""
    k = lib.tr_tail_len(int(m), int(r_num), int(r_den))
    if k < 0:
        raise ValueError("bad tail length arguments")
    return int(k)


def gdn_scan(q, k, v, log_alpha, beta, cu_seqlens, *, S0=None, want_o=True, scale=1.0,
             normalize_qk=False, recurrent=False, o=None, S_final=None, stream=None,
             stall_test=False):
    """Eq. (1) scan over a packed batch: returns (o or None, S_final [N, H, d_k, d_v] fp32)."""
    dev_ = _need_cuda(q, k, v, log_alpha, beta, S0, o, S_final)
    T, H, dk = k.shape
    dv = v.shape[2]
    for t in (q, k, v):
        if t is not None and (t.stride(2) != 1 or t.stride(1) != t.shape[2]):
            raise ValueError("q/k/v must be [T, H, d] with contiguous heads")
    la = log_alpha.contiguous()
    be = beta.contiguous()
    host, dev = _seqlens(cu_seqlens, k.device)
    N = host.numel() - 1
    if want_o and o is None:
        o = torch.empty((T, H, dv), dtype=k.dtype, device=k.device)
    if not want_o:
        o = None
    if S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=k.device)
    flags = (TR_NORMALIZE_QK if normalize_qk else 0) | (TR_SCAN_RECURRENT if recurrent else 0) | \
        (TR_SCAN_STALL_TEST if stall_test else 0)
    a = ScanArgs(N, H, dk, dv, T, _dtype_code(k), flags, float(scale),
                 q.stride(0) if q is not None else 0, k.stride(0), v.stride(0),
                 _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be),
                 _ptr(dev), host.data_ptr(), _ptr(S0), _ptr(o), _ptr(S_final))
    ws_bytes = lib.tr_gdn_scan_workspace_size(ctypes.byref(a))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=k.device) if ws_bytes else None
    with torch.cuda.device(dev_):
        _ok(lib.tr_gdn_scan(ctypes.byref(a), _ptr(ws), ws_bytes, _stream(stream, dev_)),
            "tr_gdn_scan")
    return o, S_final


def transition_product(k, log_alpha, beta, cu_seqlens, *, normalize_qk=False, recurrent=False,
                       P=None, stream=None):
    """P = T_t ... T_1 per (sequence, head): [N, H, d_k, d_k] fp32 (M = S^T convention:
    a state M_0 before the sequence becomes P M_0 + the zero-start state after it)."""
    dev_ = _need_cuda(k, log_alpha, beta, P)
    T, H, dk = k.shape
    if k.stride(2) != 1 or k.stride(1) != dk:
        raise ValueError("k must be [T, H, d] with contiguous heads")
    la = log_alpha.contiguous()
    be = beta.contiguous()
    host, dev = _seqlens(cu_seqlens, k.device)
    N = host.numel() - 1
    if P is None:
        P = torch.empty((N, H, dk, dk), dtype=torch.float32, device=k.device)
    flags = (TR_NORMALIZE_QK if normalize_qk else 0) | (TR_SCAN_RECURRENT if recurrent else 0)
    a = ScanArgs(N, H, dk, dk, T, _dtype_code(k), flags, 1.0, 0, k.stride(0), 0,
                 None, _ptr(k), None, _ptr(la), _ptr(be), _ptr(dev), host.data_ptr(), None, None,
                 None)
    ws_bytes = lib.tr_transition_product_workspace_size(ctypes.byref(a))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=k.device) if ws_bytes else None
    with torch.cuda.device(dev_):
        _ok(lib.tr_transition_product(ctypes.byref(a), _ptr(P), _ptr(ws), ws_bytes,
                                      _stream(stream, dev_)), "tr_transition_product")
    return P


@dataclass
class Layer:
    """One LA layer's weights, device tensors (W_in [2Hd_k + Hd_v + 2H, D], W_o [D, H d_v]),
    and, if the layer has an FFN sublayer, W_gate and W_up [d_ff, D], W_down [D, d_ff]
    (bf16) and ffn_gain [D] fp32 (None: ones).  Optional Gated DeltaNet details (fp32):
    conv_w [2Hd_k + Hd_v, width] (the short convolution), A_log and dt_bias [H] (gate
    parameters), o_norm_gain [d_v] (the output gate's norm; W_in then has the z rows)."""
    W_in: torch.Tensor
    W_o: torch.Tensor
    rms_gain: Optional[torch.Tensor] = None
    W_gate: Optional[torch.Tensor] = None
    W_up: Optional[torch.Tensor] = None
    W_down: Optional[torch.Tensor] = None
    ffn_gain: Optional[torch.Tensor] = None
    conv_w: Optional[torch.Tensor] = None
    A_log: Optional[torch.Tensor] = None
    dt_bias: Optional[torch.Tensor] = None
    o_norm_gain: Optional[torch.Tensor] = None


class GroupReplay:
    """A prepared tr_replay_group call: fixed buffers, so repeated calls cost one C call.

    ``h_tail`` [T, D] bf16 and ``cu_seqlens`` describe the packed tails of the
    group's requests; ``layers`` the group's LA layers (objects with the fields of
    ``Layer``; FFN fields absent or None: no FFN sublayer).  Outputs: ``S_hat``
    [L, N, H, d_k, d_v] fp32 and, unless ``skip_last_output``, ``x_out`` [T, D].
    ``skip_last_ffn`` (default on, the tail-FFN skip) leaves out the last layer's FFN.
    ``output_gate`` turns on the gated output norm (W_in with the z rows); the layers'
    conv_w turn on the short convolution, and ``want_conv_state`` returns its state
    ``conv_state`` [L, N, width - 1, 2Hd_k + Hd_v] bf16.
    """

    def __init__(self, h_tail, cu_seqlens, layers: Sequence, n_heads: int, d_k: int, d_v: int,
                 *, skip_last_output=False, want_x_out=True, rms_eps=0.0, norm_eps=0.0,
                 skip_last_ffn=True, output_gate=False, want_conv_state=False,
                 S_hat=None, x_out=None, workspace=None):
        _need_cuda(h_tail)
        if h_tail.dtype != torch.bfloat16 or not h_tail.is_contiguous():
            raise ValueError("h_tail must be contiguous bf16 [T, D]")
        dev = h_tail.device
        T, D = h_tail.shape
        self.host, self.dev_cu = _seqlens(cu_seqlens, dev)
        N = self.host.numel() - 1
        L = len(layers)
        self.layers = list(layers)
        self._layer_arr = (LALayer * L)()
        d_ff = 0
        conv_width = 0
        n_in = 2 * n_heads * d_k + n_heads * d_v * (2 if output_gate else 1) + 2 * n_heads
        for i, lw in enumerate(self.layers):
            _need_cuda(h_tail, lw.W_in, lw.W_o, lw.rms_gain)
            _need_layout("W_in", lw.W_in, torch.bfloat16, (n_in, D))
            _need_layout("W_o", lw.W_o, torch.bfloat16, (D, n_heads * d_v))
            _need_layout("rms_gain", lw.rms_gain, torch.float32, (D,))
            Wg = getattr(lw, "W_gate", None)
            Wu, Wd, fg = (getattr(lw, n, None) for n in ("W_up", "W_down", "ffn_gain"))
            if Wg is not None:
                _need_cuda(h_tail, Wg, Wu, Wd, fg)
                if d_ff and Wg.shape[0] != d_ff:
                    raise ValueError("all FFN sublayers of a group must have one width")
                d_ff = Wg.shape[0]
                _need_layout("W_gate", Wg, torch.bfloat16, (d_ff, D))
                _need_layout("W_up", Wu, torch.bfloat16, (d_ff, D))
                _need_layout("W_down", Wd, torch.bfloat16, (D, d_ff))
                _need_layout("ffn_gain", fg, torch.float32, (D,))
            cw, al, db, og = (getattr(lw, n, None) for n in ("conv_w", "A_log", "dt_bias",
                                                                 "o_norm_gain"))
            _need_cuda(h_tail, cw, al, db, og)
            _need_layout("conv_w", cw, torch.float32)
            if cw is not None and cw.shape[0] != 2 * n_heads * d_k + n_heads * d_v:
                raise ValueError("conv_w must be [2 H d_k + H d_v, width]")
            _need_layout("A_log", al, torch.float32, (n_heads,))
            _need_layout("dt_bias", db, torch.float32, (n_heads,))
            _need_layout("o_norm_gain", og, torch.float32, (d_v,))
            widths = {cw.shape[1]} if cw is not None else {0}
            if i == 0:
                conv_width = widths.pop()
            elif widths.pop() != conv_width:
                raise ValueError("every layer of a group has the same convolution width")
            self._layer_arr[i] = LALayer(_ptr(lw.rms_gain), _ptr(lw.W_in), _ptr(lw.W_o),
                                         _ptr(fg), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(cw),
                                         _ptr(al), _ptr(db), _ptr(og))
        _need_cuda(h_tail, S_hat, x_out, workspace)
        self.S_hat = S_hat if S_hat is not None else torch.empty(
            (L, N, n_heads, d_k, d_v), dtype=torch.float32, device=dev)
        if skip_last_output:
            want_x_out = False
        self.x_out = None
        if want_x_out:
            self.x_out = x_out if x_out is not None else torch.empty((T, D), dtype=torch.float32,
                                                                     device=dev)
        flags = (TR_SKIP_LAST_OUTPUT if skip_last_output else 0) | \
            (TR_SKIP_LAST_FFN if skip_last_ffn else 0) | (TR_OUTPUT_GATE if output_gate else 0)
        self.conv_state = None
        if want_conv_state and conv_width > 0:
            self.conv_state = torch.empty(
                (L, N, conv_width - 1, (2 * d_k + d_v) * n_heads), dtype=torch.bfloat16,
                device=dev)
        self.h_tail = h_tail
        self.args = GroupArgs(N, n_heads, d_k, d_v, D, L, T, flags, float(rms_eps),
                              float(norm_eps), d_ff, _ptr(h_tail), _ptr(self.dev_cu),
                              self.host.data_ptr(), self._layer_arr, _ptr(self.S_hat),
                              _ptr(self.x_out), conv_width, _ptr(self.conv_state))
        self.ws_bytes = lib.tr_replay_group_workspace_size(ctypes.byref(self.args))
        # allocated at the first run(): a description used only inside GroupsReplay (which
        # has a workspace of its own) never holds one
        self.workspace = workspace

    def _ws(self):
        if self.workspace is None and self.ws_bytes:
            self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8,
                                         device=self.h_tail.device)
        return self.workspace

    def run(self, stream=None):
        self._ws()
        dev = self.h_tail.device
        with torch.cuda.device(dev):
            _ok(lib.tr_replay_group(ctypes.byref(self.args), _ptr(self.workspace), self.ws_bytes,
                                    _stream(stream, dev)), "tr_replay_group")
        return self.S_hat, self.x_out

    def kernel_count(self) -> int:
        return int(lib.tr_replay_group_kernel_count(ctypes.byref(self.args)))

    def kernel_names(self) -> list:
        """The kernels one run() launches, in order (the events of run_profiled bracket them)."""
        names = lib.tr_replay_group_kernel_names(ctypes.byref(self.args)).decode()
        return names.split(",") if names else []

    def run_profiled(self, event_handles, stream=None):
        """Same as run(), recording the given raw cudaEvent_t handles between kernel launches."""
        arr = (c_vp * len(event_handles))(*event_handles)
        self._ws()
        dev = self.h_tail.device
        with torch.cuda.device(dev):
            _ok(lib.tr_replay_group_profiled(ctypes.byref(self.args), _ptr(self.workspace),
                                             self.ws_bytes, _stream(stream, dev), arr,
                                             len(event_handles)), "tr_replay_group_profiled")
        return self.S_hat, self.x_out


def replay_group(h_tail, cu_seqlens, layers, n_heads, d_k, d_v, **kw):
    """One group's replay: returns (S_hat [L, N, H, d_k, d_v], x_out or None)."""
    stream = kw.pop("stream", None)
    return GroupReplay(h_tail, cu_seqlens, layers, n_heads, d_k, d_v, **kw).run(stream)


class GroupsReplay:
    """A prepared tr_replay_groups call over several GroupReplay descriptions (shared workspace).
    With lanes = 2..4 the workspace holds that many group slices and the groups run on that
    many streams at once (bitwise the same results)."""

    def __init__(self, groups: Sequence[GroupReplay], lanes: int = 1):
        self.groups = list(groups)
        n = len(self.groups)
        if not 1 <= lanes <= 4:
            raise ValueError("lanes must be 1..4")
        self._arr = (GroupArgs * n)()
        for i, g in enumerate(self.groups):
            self._arr[i] = g.args
        self.lanes = lanes
        self.ws_bytes = (lib.tr_replay_groups_workspace_size(self._arr, n) if lanes == 1 else
                         lib.tr_replay_groups_lanes_workspace_size(self._arr, n, lanes))
        dev = self.groups[0].h_tail.device
        for g in self.groups:
            if g.h_tail.device != dev:
                raise ValueError("every group must live on one device")
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev) \
            if self.ws_bytes else None

    def run(self, stream=None):
        dev = self.groups[0].h_tail.device
        with torch.cuda.device(dev):
            _ok(lib.tr_replay_groups(self._arr, len(self.groups), _ptr(self.workspace),
                                     self.ws_bytes, _stream(stream, dev)), "tr_replay_groups")
        return [(g.S_hat, g.x_out) for g in self.groups]

    def run_overlapped(self, kv_host, kv_dev, stream=None, copy_stream=None):
        """run() with kv_host (pinned) copied to kv_dev on copy_stream during the replay;
        `stream` waits for the copy before anything enqueued after this call."""
        if copy_stream is None:
            raise ValueError("the KV copy needs a stream of its own (copy_stream)")
        if kv_host.numel() * kv_host.element_size() != kv_dev.numel() * kv_dev.element_size():
            raise ValueError("kv_host and kv_dev differ in size")
        if not kv_host.is_pinned():
            raise ValueError("kv_host must be pinned host memory")
        nbytes = kv_host.numel() * kv_host.element_size()
        dev = self.groups[0].h_tail.device
        if _need_cuda(kv_dev) != dev:
            raise ValueError("kv_dev must live on the groups' device")
        with torch.cuda.device(dev):
            _ok(lib.tr_replay_groups_overlapped(self._arr, len(self.groups),
                                                _ptr(self.workspace), self.ws_bytes,
                                                kv_host.data_ptr(), _ptr(kv_dev), nbytes,
                                                _stream(stream, dev), _stream(copy_stream, dev)),
                "tr_replay_groups_overlapped")
        return [(g.S_hat, g.x_out) for g in self.groups]


def kv_transfer(kv_host, kv_dev, stream=None, copy_stream=None):
    """The FA KV copy of tr_replay_groups_overlapped alone (no groups): kv_host (pinned) to
    kv_dev on copy_stream, after the work already on `stream`, which then waits for it."""
    dev = _need_cuda(kv_dev)
    if copy_stream is None:
        raise ValueError("the KV copy needs a stream of its own (copy_stream)")
    if kv_host.numel() * kv_host.element_size() != kv_dev.numel() * kv_dev.element_size():
        raise ValueError("kv_host and kv_dev differ in size")
    if not kv_host.is_pinned():
        raise ValueError("kv_host must be pinned host memory")
    nbytes = kv_host.numel() * kv_host.element_size()
    with torch.cuda.device(dev):
        _ok(lib.tr_replay_groups_overlapped(None, 0, None, 0, kv_host.data_ptr(), _ptr(kv_dev),
                                            nbytes, _stream(stream, dev),
                                            _stream(copy_stream, dev)),
            "tr_replay_groups_overlapped")


def state_error(S, S_hat, *, per_mat=True, stream=None):
    """(err_per_mat [n_mats] fp64 or None, err_total [1] fp64), device tensors."""
    dev = _need_cuda(S, S_hat)
    if S.shape != S_hat.shape or S.dtype != torch.float32 or S_hat.dtype != torch.float32:
        raise ValueError("S and S_hat must be fp32 tensors of one shape")
    dk, dv = S.shape[-2:]
    S, S_hat = S.contiguous(), S_hat.contiguous()
    n = S.numel() // (dk * dv)
    per = torch.empty(n, dtype=torch.float64, device=dev) if per_mat else None
    tot = torch.empty(1, dtype=torch.float64, device=dev)
    ws_bytes = lib.tr_state_error_workspace_size(n)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    with torch.cuda.device(dev):
        _ok(lib.tr_state_error(_ptr(S), _ptr(S_hat), n, dk, dv, _ptr(per), _ptr(tot), _ptr(ws),
                               ws_bytes, _stream(stream, dev)), "tr_state_error")
    return per, tot


def state_error_noalloc(S, S_hat, *, per_mat=True, stream=None):
    """Same as state_error, through the entry point that allocates no scratch
    (for callers that cannot allocate device memory at the call; see include/tr.h)."""
    dev = _need_cuda(S, S_hat)
    if S.shape != S_hat.shape or S.dtype != torch.float32 or S_hat.dtype != torch.float32:
        raise ValueError("S and S_hat must be fp32 tensors of one shape")
    dk, dv = S.shape[-2:]
    S, S_hat = S.contiguous(), S_hat.contiguous()
    n = S.numel() // (dk * dv)
    per = torch.empty(n, dtype=torch.float64, device=dev) if per_mat else None
    tot = torch.empty(1, dtype=torch.float64, device=dev)
    # the library's fixed scratch and the kernel belong to the current device: make the
    # tensors' device current for the call
    with torch.cuda.device(dev):
        _ok(lib.tr_state_error_noalloc(_ptr(S), _ptr(S_hat), n, dk, dv, _ptr(per), _ptr(tot),
                                       _stream(stream, dev)), "tr_state_error_noalloc")
    return per, tot


def rmsnorm(x, gain=None, eps=0.0, stream=None):
    dev = _need_cuda(x, gain)
    x = x.contiguous()
    T, D = x.shape
    out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _ok(lib.tr_rmsnorm(_ptr(x), _dtype_code(x), _ptr(gain), T, D, float(eps), _ptr(out),
                           _stream(stream, dev)), "tr_rmsnorm")
    return out


def in_projection(x_hat, W_in, n_heads, d_k, d_v, *, skip_q=False, norm_eps=0.0, stream=None):
    """(qkv [T, 2Hd_k + Hd_v] bf16, log_alpha [T, H], beta [T, H])."""
    dev = _need_cuda(x_hat, W_in)
    T, D = x_hat.shape
    x_hat = x_hat.contiguous()
    W_in = W_in.contiguous()
    qkv = torch.zeros((T, 2 * n_heads * d_k + n_heads * d_v), dtype=torch.bfloat16, device=dev)
    la = torch.empty((T, n_heads), dtype=torch.float32, device=dev)
    be = torch.empty((T, n_heads), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _ok(lib.tr_in_projection(_ptr(x_hat), _ptr(W_in), T, D, n_heads,
                                 d_k, d_v, TR_SKIP_LAST_OUTPUT if skip_q else 0, float(norm_eps),
                                 _ptr(qkv), _ptr(la), _ptr(be), _stream(stream, dev)),
            "tr_in_projection")
    return qkv, la, be


def out_projection(o, W_o, x_res, stream=None):
    """x_res + o W_o^T in fp32; o [T, H d_v] bf16 (rows may be strided)."""
    dev = _need_cuda(o, W_o, x_res)
    T, hv = o.shape
    D = W_o.shape[0]
    W_o = W_o.contiguous()
    x_res = x_res.contiguous()
    out = torch.empty((T, D), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _ok(lib.tr_out_projection(_ptr(o), o.stride(0), _ptr(W_o),
                                  _ptr(x_res), _dtype_code(x_res), T, D, hv, _ptr(out),
                                  _stream(stream, dev)), "tr_out_projection")
    return out


def set_wait_limit_ns(ns: int) -> None:
    """Wall-clock limit of the scan kernels' bounded waits for later calls (0: the default 4 s)."""
    _ok(lib.tr_set_wait_limit_ns(int(ns)), "tr_set_wait_limit_ns")


def check(stream=None) -> None:
    """Wait for the stream and raise if a kernel reported a device-side failure."""
    _ok(lib.tr_check(_stream(stream)), "tr_check")
