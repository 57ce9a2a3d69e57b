"""GPU parity of the dense steps of one LA layer (RMSNorm, input projection with gates and key
norm, output projection with residual) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
import linear_attention_state_zero_b200 as tr
from gpu_util import f64, rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,D", [(300, 512), (1, 64), (1639, 2048), (37, 1024), (130, 4096), (5, 2056)])
def test_rmsnorm(cuda_device, in_dtype, T, D):
    x = synth.normal((T, D), 101, 1).to(in_dtype)
    g = 1.0 + synth.normal((D,), 101, 2, 0.1)
    got = tr.rmsnorm(x.to(cuda_device), g.to(cuda_device))
    want = oracle.bf16_round(oracle.rmsnorm(x, g))
    d = np.abs(f64(got) - want)
    # both sides round to bf16: agree except for near-ties, by at most one bf16 ulp
    assert np.all(d <= np.abs(want) * 2.0 ** -7 + 1e-30)
    assert np.mean(d > 0) < 0.01
    assert rel_fro(got, want) < 1e-3


# T <= 128: one CTA per 128-row tile; T > 128: 256-row tiles on CTA pairs, whose second CTA
# may hold no valid row (T = 129, 300) and whose partial last round runs as half-width units
# (T = 1639: 175 pair tiles)
@pytest.mark.parametrize("T,D,H,d", [(100, 256, 2, 128), (300, 256, 2, 128), (129, 512, 4, 64),
                                     (1639, 2048, 16, 128)])
@pytest.mark.parametrize("skip_q", [False, True])
def test_in_projection(cuda_device, T, D, H, d, skip_q):
    x_hat = synth.normal((T, D), 102, 1).to(torch.bfloat16)
    W_in = synth.la_layers(1, D, H, d, d, seed=102)[0].W_in
    qkv, la, be = tr.in_projection(x_hat.to(cuda_device), W_in.to(cuda_device), H, d, d,
                                   skip_q=skip_q)
    q, k, v, aa, ab = oracle.in_projection(x_hat, W_in, H, d, d)
    qkv = f64(qkv)
    gq = qkv[:, :H * d].reshape(T, H, d)
    gk = qkv[:, H * d:2 * H * d].reshape(T, H, d)
    gv = qkv[:, 2 * H * d:].reshape(T, H, d)
    want_la, want_b = oracle.gates(aa, ab)
    assert rel_fro(gk, oracle.bf16_round(oracle.l2_normalize(k))) < 2e-3
    assert rel_fro(gv, oracle.bf16_round(v)) < 2e-3
    if skip_q:
        assert not gq.any()  # the q columns are neither computed nor written
    else:
        assert rel_fro(gq, oracle.bf16_round(oracle.l2_normalize(q))) < 2e-3
        np.testing.assert_allclose(np.linalg.norm(gq, axis=-1), 1.0, atol=1e-2)
    assert rel_fro(la, want_la) < 1e-5
    assert rel_fro(be, want_b) < 1e-5


@pytest.mark.parametrize("res_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,D,hv", [(300, 512, 256), (1639, 2048, 2048), (7, 128, 64)])
def test_out_projection(cuda_device, res_dtype, T, D, hv):
    o = synth.normal((T, hv), 103, 1).to(torch.bfloat16)
    W_o = synth.normal((D, hv), 103, 2, 0.02).to(torch.bfloat16)
    x = synth.normal((T, D), 103, 3).to(res_dtype)
    got = tr.out_projection(o.to(cuda_device), W_o.to(cuda_device), x.to(cuda_device))
    want = oracle.out_projection_residual(x, o.reshape(T, -1, 1), W_o)
    assert rel_fro(got, want) < 1e-5
    # the product alone (x = 0) to the same relative accuracy
    got0 = tr.out_projection(o.to(cuda_device), W_o.to(cuda_device),
                             torch.zeros(T, D, dtype=res_dtype, device=cuda_device))
    assert rel_fro(got0, oracle.out_projection_residual(np.zeros((T, D)), o.reshape(T, -1, 1),
                                                        W_o)) < 1e-5


def test_out_projection_strided_o(cuda_device):
    T, D, hv = 200, 256, 128
    big = synth.normal((T, 3 * hv), 104, 1).to(torch.bfloat16)
    W_o = synth.normal((D, hv), 104, 2, 0.02).to(torch.bfloat16)
    x = synth.normal((T, D), 104, 3)
    o = big[:, hv:2 * hv]
    got = tr.out_projection(big.to(cuda_device)[:, hv:2 * hv], W_o.to(cuda_device),
                            x.to(cuda_device))
    want = oracle.out_projection_residual(x, o.reshape(T, -1, 1), W_o)
    assert rel_fro(got, want) < 1e-5
