"""Seeded synthetic inputs for the Tail-Replay tail-replay path.

This module only draws random numbers with fixed seeds and shapes them like the
workloads described for the method (cached full-attention output hiddens ``h``,
projection weights, and the per-token scan inputs q, k, v, alpha, beta).  It holds
none of the method's arithmetic: no recurrence, no normalisation layer, no gate
parameterisation.  Both the CUDA path's tests/benchmark and the fp64 oracle read
their inputs from here, so the two sides see the same bits.

Distributions (all from ``torch.Generator`` on the CPU, or on the device for
inputs too large to draw on the host; the same seed gives the same stream):

* ``h``: N(0, 1), rounded to bf16 (hidden vectors leaving a full-attention layer).
* projection weights (the LA layer's and, where a layer has an FFN sublayer, its gate,
  up and down weights): N(0, 0.02^2), rounded to bf16.
* optional Gated DeltaNet layer parameters: short-convolution taps U[-0.5, 0.5] (fp32,
  [channels, width]); per-head A_log U[0, log 16] and dt_bias U[-7, -2] (fp32); the
  output-gate norm gain 1 + N(0, 0.1^2).
* scan q, k: directions drawn uniformly on the unit sphere (a normalised Gaussian
  vector), then cast to the requested dtype.
* scan v: N(0, 1).
* scan alpha: U[lo, hi]; the scan takes ``log_alpha = log(alpha)`` in fp32.
* scan beta: logistic of N(0, 1), in (0, 1).

Seeds: ``SEED_BASE + workload index``; each tensor gets its own sub-stream
(``seed * 1000 + tensor id``), so adding a tensor never shifts another one.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

SEED_BASE = 0x7A110001

# tensor ids for sub-streams
_T_H, _T_WIN, _T_WO, _T_GAIN = 1, 2, 3, 4
_T_WGATE, _T_WUP, _T_WDOWN, _T_FGAIN = 5, 6, 7, 8
_T_CONV, _T_ALOG, _T_DTB, _T_OGAIN = 9, 10, 18, 19
_T_Q, _T_K, _T_V, _T_ALPHA, _T_BETA, _T_S0, _T_LENS = 11, 12, 13, 14, 15, 16, 17


def _gen(seed: int, tensor_id: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000 + tensor_id) & 0x7FFFFFFFFFFFFFFF)
    return g


def normal(shape, seed: int, tensor_id: int, std: float = 1.0, device: str = "cpu") -> torch.Tensor:
    x = torch.randn(*shape, generator=_gen(seed, tensor_id, device), dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x


def uniform(shape, seed: int, tensor_id: int, lo: float, hi: float, device: str = "cpu") -> torch.Tensor:
    x = torch.rand(*shape, generator=_gen(seed, tensor_id, device), dtype=torch.float64, device=device)
    return lo + (hi - lo) * x


def unit_sphere(shape, seed: int, tensor_id: int) -> torch.Tensor:
    """Directions uniform on the unit sphere along the last axis (fp32)."""
    x = normal(shape, seed, tensor_id).double()
    x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    return x.float()


def cu_seqlens_of(lengths: Sequence[int]) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


@dataclass
class ScanCase:
    """Inputs of one Gated DeltaNet scan call (packed varlen layout)."""
    q: torch.Tensor           # [T, H, d_k]
    k: torch.Tensor           # [T, H, d_k]
    v: torch.Tensor           # [T, H, d_v]
    log_alpha: torch.Tensor   # [T, H] fp32
    beta: torch.Tensor        # [T, H] fp32
    cu_seqlens: torch.Tensor  # [N + 1] int32
    S0: Optional[torch.Tensor] = None  # [N, H, d_k, d_v] fp32

    @property
    def n_seqs(self) -> int:
        return self.cu_seqlens.numel() - 1


def scan_case(lengths: Sequence[int], n_heads: int, d_k: int, d_v: int, dtype: torch.dtype,
              alpha_lo: float, alpha_hi: float, seed: int, with_S0: bool = False) -> ScanCase:
    T = int(sum(lengths))
    q = unit_sphere((T, n_heads, d_k), seed, _T_Q).to(dtype)
    k = unit_sphere((T, n_heads, d_k), seed, _T_K).to(dtype)
    v = normal((T, n_heads, d_v), seed, _T_V).to(dtype)
    alpha = uniform((T, n_heads), seed, _T_ALPHA, alpha_lo, alpha_hi)
    log_alpha = torch.log(alpha).float()
    beta = torch.sigmoid(normal((T, n_heads), seed, _T_BETA).double()).float()
    S0 = None
    if with_S0:
        S0 = normal((len(lengths), n_heads, d_k, d_v), seed, _T_S0, std=0.1)
    return ScanCase(q, k, v, log_alpha, beta, cu_seqlens_of(lengths), S0)


def scan_case_from_prefix(m: int, tail: int, n_heads: int, d_k: int, d_v: int, dtype: torch.dtype,
                          alpha_lo: float, alpha_hi: float, seed: int) -> tuple[ScanCase, ScanCase]:
    """A full prefix of m tokens and its last ``tail`` tokens as a second case.

    The tail tensors are exact row slices of the prefix tensors, so a replay of
    the tail sees bit-identical inputs to the last ``tail`` steps of the prefix.
    """
    full = scan_case([m], n_heads, d_k, d_v, dtype, alpha_lo, alpha_hi, seed)
    a = m - tail
    t = ScanCase(full.q[a:].clone(), full.k[a:].clone(), full.v[a:].clone(),
                 full.log_alpha[a:].clone(), full.beta[a:].clone(), cu_seqlens_of([tail]))
    return full, t


@dataclass
class LALayerWeights:
    W_in: torch.Tensor            # bf16 [2H*d_k + H*d_v + 2H, D]  (out x in)
    W_o: torch.Tensor             # bf16 [D, H*d_v]
    rms_gain: Optional[torch.Tensor] = None  # fp32 [D] or None (= ones)
    # FFN sublayer after the LA sublayer (all None: the layer has none)
    W_gate: Optional[torch.Tensor] = None    # bf16 [d_ff, D]
    W_up: Optional[torch.Tensor] = None      # bf16 [d_ff, D]
    W_down: Optional[torch.Tensor] = None    # bf16 [D, d_ff]
    ffn_gain: Optional[torch.Tensor] = None  # fp32 [D] or None (= ones)
    # optional Gated DeltaNet layer parameters (None: not used)
    conv_w: Optional[torch.Tensor] = None       # fp32 [2H*d_k + H*d_v, width]
    A_log: Optional[torch.Tensor] = None        # fp32 [H]
    dt_bias: Optional[torch.Tensor] = None      # fp32 [H]
    o_norm_gain: Optional[torch.Tensor] = None  # fp32 [d_v]


def in_features(n_heads: int, d_k: int, d_v: int, output_gate: bool = False) -> int:
    return 2 * n_heads * d_k + n_heads * d_v * (2 if output_gate else 1) + 2 * n_heads


def la_layers(n_layers: int, d_model: int, n_heads: int, d_k: int, d_v: int, seed: int,
              std: float = 0.02, device: str = "cpu", with_gain: bool = False,
              d_ff: int = 0, conv_width: int = 0, gate_params: bool = False,
              output_gate: bool = False) -> List[LALayerWeights]:
    """Weights of ``n_layers`` LA layers; with ``d_ff > 0`` each also gets an FFN sublayer,
    with ``conv_width > 0`` short-convolution taps, with ``gate_params`` A_log and dt_bias,
    with ``output_gate`` the z rows of W_in (after v) and the output norm's gain."""
    out = []
    n_in = in_features(n_heads, d_k, d_v, output_gate)
    for l in range(n_layers):
        s = seed * 64 + l
        W_in = normal((n_in, d_model), s, _T_WIN, std, device).to(torch.bfloat16)
        W_o = normal((d_model, n_heads * d_v), s, _T_WO, std, device).to(torch.bfloat16)
        gain = None
        if with_gain:
            gain = 1.0 + normal((d_model,), s, _T_GAIN, 0.1, device)
        lw = LALayerWeights(W_in, W_o, gain)
        if d_ff > 0:
            lw.W_gate = normal((d_ff, d_model), s, _T_WGATE, std, device).to(torch.bfloat16)
            lw.W_up = normal((d_ff, d_model), s, _T_WUP, std, device).to(torch.bfloat16)
            lw.W_down = normal((d_model, d_ff), s, _T_WDOWN, std, device).to(torch.bfloat16)
            if with_gain:
                lw.ffn_gain = 1.0 + normal((d_model,), s, _T_FGAIN, 0.1, device)
        if conv_width > 0:
            lw.conv_w = uniform((2 * n_heads * d_k + n_heads * d_v, conv_width), s, _T_CONV,
                                -0.5, 0.5, device).float()
        if gate_params:
            lw.A_log = uniform((n_heads,), s, _T_ALOG, 0.0, math.log(16.0), device).float()
            lw.dt_bias = uniform((n_heads,), s, _T_DTB, -7.0, -2.0, device).float()
        if output_gate:
            lw.o_norm_gain = 1.0 + normal((d_v,), s, _T_OGAIN, 0.1, device)
        out.append(lw)
    return out


def hidden_prefix(m: int, d_model: int, seed: int, device: str = "cpu") -> torch.Tensor:
    """Cached FA output hiddens for positions 1..m of one request, bf16 [m, D]."""
    return normal((m, d_model), seed, _T_H, 1.0, device).to(torch.bfloat16)


def varlen_prefix_lengths(n: int, lo: int, hi: int, seed: int) -> List[int]:
    """Integer matched-prefix lengths m_i ~ U[lo, hi] (inclusive), seeded."""
    g = _gen(seed, _T_LENS)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]

