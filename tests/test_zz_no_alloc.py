"""The allocation-free state-error entry point (tr_state_error_noalloc).

Some callers cannot allocate device memory when they call the library (an engine whose
allocator owns all device memory, or code where cudaMalloc would synchronize the device).
This entry point keeps its scratch in a fixed array inside the library.  It must give the
same result as tr_state_error, call after call, although every call reuses the same scratch.
This file is collected last so that a run that stops at the first failure has run the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import linear_attention_state_zero_b200 as tr
from gpu_util import f64

pytestmark = pytest.mark.gpu


def _pair(seed, n, dk, dv):
    S = synth.normal((n, dk, dv), seed, 1)
    Sh = S + synth.normal((n, dk, dv), seed, 2, 1e-3)
    return S, Sh


def test_matches_workspace_entry_point_on_consecutive_calls(cuda_device):
    # two calls in a row, different sizes and data: nothing of the first may leak into the second
    for seed, (n, dk, dv) in ((501, (300, 128, 128)), (502, (7, 64, 64))):
        S, Sh = _pair(seed, n, dk, dv)
        S, Sh = S.to(cuda_device), Sh.to(cuda_device)
        per_a, tot_a = tr.state_error_noalloc(S, Sh)
        per_b, tot_b = tr.state_error(S, Sh)
        torch.cuda.synchronize()
        np.testing.assert_allclose(f64(per_a), f64(per_b), rtol=1e-12, atol=0)
        np.testing.assert_allclose(f64(tot_a), f64(tot_b), rtol=1e-12, atol=0)
        # and directly against the oracle's fp64 definition (both sides sum fp32 inputs in
        # fp64; only the summation order differs)
        wper, wtot = oracle.state_error(S.cpu(), Sh.cpu())
        np.testing.assert_allclose(f64(per_a), wper, rtol=1e-9, atol=0)
        np.testing.assert_allclose(f64(tot_a)[0], wtot, rtol=1e-9, atol=0)


def test_rejects_more_matrices_than_the_fixed_scratch(cuda_device):
    S = torch.zeros(65537, 2, 2, device=cuda_device)
    with pytest.raises(tr.TrError) as e:
        tr.state_error_noalloc(S, S)
    assert e.value.status == 5  # TR_ERR_UNSUPPORTED
    assert "65536" in tr.lib.tr_last_error().decode()
