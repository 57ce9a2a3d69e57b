"""GPU parity at the workload configurations, through the C ABI, against the fp64 oracle.

Each workload runs at its full size in one call; the oracle checks every output it can
finish in seconds and a seeded sample of the rest, and properties that hold at any size
cover what it cannot (a unit replayed alone equals the same unit in the batch, bitwise;
the tail error obeys the contraction bound of the reading notes, section 2.3).

- 8 concurrent hits x 8 groups x 3 LA layers, d_model 2048, 16 heads of 128, m = 32768,
  r in {5%, 10%}: one tr_replay_groups call (each group call packs the 8 hits).
- a varlen batch of 64 requests with m ~ U[1024, 131072], r = 10%, d_model 4096, 32 heads,
  3 LA layers (one group of the 8: the groups are independent calls of the same kernels).
- the scan sweep: m in {4K .. 128K} x r in {1, 2, 5, 10, 20, 100}%, 32 heads, alpha from
  U[0.80, 1] and U[0.97, 1]; S_m, S_hat_m and the relative state error per cell.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import linear_attention_state_zero_b200 as tr
from gpu_util import f64, rel_fro, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

TOL = 5e-3


def test_eight_hits_eight_groups(cuda_device):
    D, H, d, L, G, N, m = 2048, 16, 128, 3, 8, 8, 32768
    ks = [tr.tail_len(m, 5 if i % 2 == 0 else 10, 100) for i in range(N)]
    assert ks[:2] == [1639, 3277]
    base = synth.SEED_BASE + 2
    groups, host = [], []
    for g in range(G):
        layers = synth.la_layers(L, D, H, d, d, seed=base * 16 + g)
        # the tail of hit i at group g's entry: the last k_i cached hiddens (drawn directly)
        tails = [synth.hidden_prefix(ks[i], D, base * 1024 + 8 * g + i) for i in range(N)]
        h = torch.cat(tails)
        cu = synth.cu_seqlens_of(ks)
        host.append((tails, layers))
        groups.append(tr.GroupReplay(h.to(cuda_device), cu, to_dev(layers, cuda_device), H, d, d,
                                     skip_last_output=True))
    outs = tr.GroupsReplay(groups).run()
    torch.cuda.synchronize()
    tr.check()
    # oracle on one hit per group (hit g at group g: both tail lengths, every group)
    for g in range(G):
        tails, layers = host[g]
        i = g % N
        wS, _ = oracle.replay_group(tails[i], [0, ks[i]], layers, H, d, d, skip_last_output=True)
        S = outs[g][0][:, i:i + 1]
        for l in range(L):
            assert rel_fro(S[l], wS[l]) < TOL, (g, i, l)
    # a unit replayed alone equals the same unit inside the packed batch, bitwise
    for g, i in ((3, 5), (6, 0)):
        tails, layers = host[g]
        S1, _ = tr.replay_group(tails[i].to(cuda_device), [0, ks[i]], to_dev(layers, cuda_device),
                                H, d, d, skip_last_output=True)
        assert torch.equal(S1[:, 0], outs[g][0][:, i]), (g, i)
    for g in range(G):
        assert torch.isfinite(outs[g][0]).all()


def test_varlen_64_requests_d4096(cuda_device):
    D, H, d, L, n = 4096, 32, 128, 3, 64
    seed = synth.SEED_BASE + 3
    ms = synth.varlen_prefix_lengths(n, 1024, 131072, seed)
    ks = [tr.tail_len(mi, 10, 100) for mi in ms]
    cu = synth.cu_seqlens_of(ks)
    T = int(cu[-1])
    # the packed tails, drawn on the device (about 3.5 GB of bf16)
    h = synth.hidden_prefix(T, D, seed, device=str(cuda_device))
    layers = synth.la_layers(L, D, H, d, d, seed=seed)
    dl = to_dev(layers, cuda_device)
    S, _ = tr.replay_group(h, cu, dl, H, d, d, skip_last_output=True)
    torch.cuda.synchronize()
    tr.check()
    assert S.shape == (L, n, H, d, d)
    # oracle on the shortest and the longest request and two seeded-random ones
    order = sorted(range(n), key=lambda i: ks[i])
    g = torch.Generator().manual_seed(seed)
    rnd = [order[int(j)] for j in torch.randint(1, n - 1, (2,), generator=g)]
    picks = [order[0], order[-1]] + rnd
    for i in picks:
        a, b = int(cu[i]), int(cu[i + 1])
        hi = h[a:b].cpu()
        wS, _ = oracle.replay_group(hi, [0, b - a], layers, H, d, d, skip_last_output=True)
        for l in range(L):
            assert rel_fro(S[l, i:i + 1], wS[l]) < TOL, (i, ks[i], l)
        if i in rnd:  # alone == in the batch, bitwise
            S1, _ = tr.replay_group(h[a:b].contiguous(), [0, b - a], dl, H, d, d,
                                    skip_last_output=True)
            assert torch.equal(S1[:, 0], S[:, i]), i
    assert torch.isfinite(S).all()


SWEEP_M = [4096, 8192, 16384, 32768, 65536, 131072]
SWEEP_R = [1, 2, 5, 10, 20, 100]  # percent


@pytest.mark.parametrize("alpha_lo", [0.80, 0.97])
def test_scan_sweep(cuda_device, alpha_lo):
    H, d = 32, 128
    for mi, m in enumerate(SWEEP_M):
        seed = synth.SEED_BASE + 4 + 16 * mi + (0 if alpha_lo == 0.80 else 8)
        full = synth.scan_case([m], H, d, d, torch.bfloat16, alpha_lo, 1.0, seed=seed)
        dev = [x.to(cuda_device) for x in (full.q, full.k, full.v, full.log_alpha, full.beta)]
        _, S_m = tr.gdn_scan(*dev, full.cu_seqlens, want_o=False)
        exact_sm = m <= 16384
        if exact_sm:
            _, wS_m = oracle.gdn_scan(full.q, full.k, full.v, full.log_alpha, full.beta,
                                      full.cu_seqlens, want_o=False)
            assert rel_fro(S_m, wS_m) < TOL, m
        for r in SWEEP_R:
            k = tr.tail_len(m, r, 100)
            a = m - k
            tail = [x[a:] for x in dev]
            o, S_hat = tr.gdn_scan(*tail, synth.cu_seqlens_of([k]), want_o=r != 100)
            per, tot = tr.state_error(S_m.reshape(-1, d, d), S_hat.reshape(-1, d, d))
            if r == 100:
                assert torch.equal(S_hat, S_m) and float(tot.item()) == 0.0
                continue
            if k <= 6554:  # the oracle replays every tail of up to 6554 tokens
                wo, wS_hat = oracle.gdn_scan(full.q[a:], full.k[a:], full.v[a:],
                                             full.log_alpha[a:], full.beta[a:],
                                             synth.cu_seqlens_of([k]))
                assert rel_fro(S_hat, wS_hat) < TOL, (m, r)
                assert rel_fro(o, wo) < TOL, (m, r)
                if exact_sm:
                    _, wtot = oracle.state_error(wS_m, wS_hat)
                    assert abs(float(tot.item()) - wtot) <= 1e-2, (m, r)
            # contraction bound (unit keys, beta in (0, 1)): per head
            #   ||S_m - S_hat_m||_F <= prod_{i > a} alpha_i * ||S_a||_F
            _, S_a = tr.gdn_scan(*[x[:a] for x in dev], synth.cu_seqlens_of([a]), want_o=False)
            decay = torch.exp(full.log_alpha[a:].double().sum(0))  # [H]
            na = torch.linalg.matrix_norm(S_a[0].double()).cpu()
            nm = torch.linalg.matrix_norm(S_m[0].double()).cpu()
            err = f64(per).reshape(H) * nm.numpy()
            bound = (decay * na).numpy()
            # the GPU states carry bf16-operand rounding (relative 5e-3 of ||S_m||)
            assert np.all(err <= bound + 5e-3 * nm.numpy()), (m, r)
