"""GPU parity of the transition product (tr_transition_product) against the fp64 oracle.

P = T_t ... T_1 per (sequence, head) is the operator of the error identity in the reading
notes (section 2.3) and HYPIC's segment transition operator.  Tolerances as for the scan:
relative Frobenius 1e-5 on the fp32 path, 5e-3 with bf16 inputs (fp32 products)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import linear_attention_state_zero_b200 as tr
from gpu_util import f64, per_matrix_rel_fro, rel_fro

pytestmark = pytest.mark.gpu


def gpu_P(case, dev, **kw):
    return tr.transition_product(case.k.to(dev), case.log_alpha.to(dev), case.beta.to(dev),
                                 case.cu_seqlens, **kw)


def test_fp32_single_head(cuda_device):
    """One head, d = 64, fp32 (the 1e-5 path): the tail of m = 4096 at r = 5% (k = 205)."""
    full, tail = synth.scan_case_from_prefix(4096, 205, 1, 64, 64, torch.float32, 0.90, 1.00,
                                             seed=synth.SEED_BASE + 0)
    P = gpu_P(tail, cuda_device)
    want = oracle.transition_product(tail.k, tail.log_alpha, tail.beta, tail.cu_seqlens)
    assert rel_fro(P, want) < 1e-5


@pytest.mark.parametrize("recurrent", [False, True])
def test_bf16_varlen_ragged(cuda_device, recurrent):
    lengths = [1, 63, 64, 65, 300, 0, 129]
    case = synth.scan_case(lengths, 4, 128, 128, torch.bfloat16, 0.90, 1.00, seed=401)
    P = gpu_P(case, cuda_device, recurrent=recurrent)
    want = oracle.transition_product(case.k, case.log_alpha, case.beta, case.cu_seqlens)
    assert rel_fro(P, want) < 5e-3
    nz = [0, 1, 2, 3, 4, 6]
    assert np.all(per_matrix_rel_fro(P[nz], want[nz]) < 1e-2)
    np.testing.assert_array_equal(f64(P[5]), np.broadcast_to(np.eye(128), (4, 128, 128)))


def test_repair_and_bound_at_the_scan_cell_size(cuda_device):
    """32 heads, m = 8192, r = 10%, slow decay (alpha ~ U[0.999, 1], so the zero start misses a
    large part of S_m): with the exact S_a, P S_a + S_hat_m gives S_m back (all on the GPU);
    the oracle checks P itself; ||P||_2 <= prod alpha per head."""
    dev = cuda_device
    m, r = 8192, 10
    k = tr.tail_len(m, r, 100)
    a = m - k
    full = synth.scan_case([m], 32, 128, 128, torch.bfloat16, 0.999, 1.0, seed=402)
    d = [x.to(dev) for x in (full.q, full.k, full.v, full.log_alpha, full.beta)]
    _, S_m = tr.gdn_scan(*d, full.cu_seqlens, want_o=False)
    _, S_a = tr.gdn_scan(*[x[:a] for x in d], synth.cu_seqlens_of([a]), want_o=False)
    _, S_hat = tr.gdn_scan(*[x[a:] for x in d], synth.cu_seqlens_of([k]), want_o=False)
    P = tr.transition_product(d[1][a:], d[3][a:], d[4][a:], synth.cu_seqlens_of([k]))
    want = oracle.transition_product(full.k[a:], full.log_alpha[a:], full.beta[a:],
                                     synth.cu_seqlens_of([k]))
    assert rel_fro(P, want) < 5e-3
    repaired = torch.matmul(P, S_a) + S_hat
    assert rel_fro(repaired, f64(S_m)) < 5e-3
    # the zero start alone misses P S_a (tens of percent here); the repair removes that error
    assert rel_fro(S_hat, f64(S_m)) > 0.05
    decay = torch.exp(full.log_alpha[a:].double().sum(0)).numpy()
    norms = np.linalg.norm(f64(P)[0], 2, axis=(1, 2))
    assert np.all(norms <= decay * (1 + 5e-3) + 1e-6)
