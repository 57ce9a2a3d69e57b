"""GPU parity of tr_state_error (fp64 accumulation) against the oracle's definition."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import linear_attention_state_zero_b200 as tr
from gpu_util import f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,dk,dv", [(37, 128, 128), (1, 64, 64), (3, 8, 6)])
def test_matches_oracle(cuda_device, n, dk, dv):
    S = synth.normal((n, dk, dv), 401, 1)
    Sh = S + synth.normal((n, dk, dv), 401, 2, 1e-3) * torch.arange(1, n + 1).reshape(n, 1, 1)
    per, tot = tr.state_error(S.to(cuda_device), Sh.to(cuda_device))
    wper, wtot = oracle.state_error(S, Sh)
    np.testing.assert_allclose(f64(per), wper, rtol=1e-12)
    assert math.isclose(float(tot.item()), wtot, rel_tol=1e-12)


def test_special_cases(cuda_device):
    Z = torch.zeros(3, 16, 16, device=cuda_device)
    Y = Z.clone()
    Y[2, 0, 0] = 1e-3
    per, tot = tr.state_error(Z, Z)
    assert float(tot.item()) == 0.0 and not per.any()
    per, tot = tr.state_error(Z, Y)
    assert f64(per).tolist()[:2] == [0.0, 0.0] and math.isinf(f64(per)[2])
    assert math.isinf(float(tot.item()))
    S = synth.normal((4, 16, 16), 402, 1).to(cuda_device)
    per, tot = tr.state_error(S, torch.zeros_like(S))
    np.testing.assert_allclose(f64(per), 1.0, rtol=1e-14)
    per, tot = tr.state_error(S, S)
    assert float(tot.item()) == 0.0


def test_reproducible(cuda_device):
    S = synth.normal((64, 128, 128), 403, 1).to(cuda_device)
    Sh = S * 0.999
    a = tr.state_error(S, Sh)[1].item()
    b = tr.state_error(S, Sh)[1].item()
    assert a == b
