"""The bounded-wait failure path of the chunked scan, made to run out on purpose.

Every mbarrier wait in the scan kernels gives up after a wall-clock limit; a CTA that gives
up stops, lets the copies and products it already issued finish, and sets the library's
device error word, which tr_check reports as TR_ERR_TIMEOUT.  The test hook
TR_SCAN_STALL_TEST makes the chain kernel withhold the signal that its first state is ready,
so the waits behind it run out (after 50 ms here); the next call, without the hook and with
the default limit, must work and be correct.  Nothing faults or hangs: each wait ends at its
limit and the CTAs exit.
"""
import pytest
import torch

import oracle
import synth
import linear_attention_state_zero_b200 as tr
from gpu_util import rel_fro

pytestmark = pytest.mark.gpu


def test_wait_limit_reports_timeout_and_recovers(cuda_device):
    case = synth.scan_case([300, 64, 130], 2, 128, 128, torch.bfloat16, 0.9, 1.0, seed=701)
    args = [x.to(cuda_device) for x in (case.q, case.k, case.v, case.log_alpha, case.beta)]
    tr.check()
    try:
        tr.set_wait_limit_ns(50_000_000)
        tr.gdn_scan(*args, case.cu_seqlens, stall_test=True)
        with pytest.raises(tr.TrError) as e:
            tr.check()
        assert e.value.status == 8   # TR_ERR_TIMEOUT
    finally:
        tr.set_wait_limit_ns(0)
    tr.check()                       # the failed check cleared the error word
    o, S = tr.gdn_scan(*args, case.cu_seqlens)
    tr.check()
    wo, wS = oracle.gdn_scan(case.q, case.k, case.v, case.log_alpha, case.beta, case.cu_seqlens)
    assert rel_fro(o, wo) < 5e-3 and rel_fro(S, wS) < 5e-3
