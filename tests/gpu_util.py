"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rel_fro(got, want) -> float:
    """||got - want||_F / ||want||_F (0 when both are 0)."""
    g, w = f64(got), f64(want)
    num = np.linalg.norm((g - w).ravel())
    den = np.linalg.norm(w.ravel())
    if den == 0:
        return 0.0 if num == 0 else float("inf")
    return float(num / den)


def per_matrix_rel_fro(got, want) -> np.ndarray:
    g, w = f64(got), f64(want)
    dk, dv = w.shape[-2:]
    g = g.reshape(-1, dk * dv)
    w = w.reshape(-1, dk * dv)
    num = np.linalg.norm(g - w, axis=1)
    den = np.linalg.norm(w, axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), np.where(num > 0, np.inf, 0.0))


def to_dev(layers, device):
    import linear_attention_state_zero_b200 as tr
    import dataclasses

    def mv(t):
        return None if t is None else t.to(device)
    names = [f.name for f in dataclasses.fields(tr.Layer)]
    return [tr.Layer(**{n: mv(getattr(l, n, None)) for n in names}) for l in layers]
