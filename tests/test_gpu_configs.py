"""GPU parity at the workload configurations, through the C ABI, against the fp64 oracle.

Each workload runs at its full size in one call; the oracle checks every output it can
finish in seconds to a minute on the host cores and a seeded sample of the rest, and
properties that hold at any size cover what it cannot (a unit replayed alone equals the
same unit in the batch, bitwise; the tail error obeys the contraction bound of the reading
notes, section 2.3).

- the full prefill (k = m) of the one-group workload: S_m per layer against the oracle
  (reading notes section 3.1, "Full"), d_model 2048, 16 heads, m = 32768 -- the reference
  states the benchmark's state error is measured against.
- 8 concurrent hits x 8 groups x 3 LA layers, d_model 2048, 16 heads of 128, m = 32768,
  r in {5%, 10%}: one tr_replay_groups call; the oracle replays all 64 (hit, group) tails,
  and the full prefill of two units (S_m); the call on 4 lanes gives the same states bitwise.
- a varlen batch of 64 requests with m ~ U[1024, 131072], r = 10%, d_model 4096, 32 heads,
  8 groups x 3 LA layers in one tr_replay_groups call; the oracle replays sampled requests of
  every group, the longest request of one group, and the full prefill (S_m) of the shortest.
- the scan sweep: m in {4K .. 128K} x r in {1, 2, 5, 10, 20, 100}%, 32 heads, alpha from
  U[0.80, 1] and U[0.97, 1]; S_m of every m, S_hat_m and o of every tail, and the relative
  state error per cell, all against the oracle.
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


def test_full_prefill_one_group(cuda_device):
    """Replay with k = m is the full prefill (reading notes section 3.1, "Full"): the GPU's
    S_m of the one-group workload (the benchmark's reference states) against the oracle's
    full-length replay, layer by layer."""
    D, H, d, L, m = 2048, 16, 128, 3, 32768
    seed = synth.SEED_BASE + 1          # the benchmark's request
    h = synth.hidden_prefix(m, D, seed)
    layers = synth.la_layers(L, D, H, d, d, seed=seed)
    cu = synth.cu_seqlens_of([m])
    S, _ = tr.replay_group(h.to(cuda_device), cu, to_dev(layers, cuda_device), H, d, d,
                           skip_last_output=True)
    torch.cuda.synchronize()
    tr.check()
    wS, _ = oracle.replay_group(h, cu, layers, H, d, d, skip_last_output=True)
    for l in range(L):
        assert rel_fro(S[l], wS[l]) < TOL, l


def test_eight_hits_eight_groups(cuda_device):
    D, H, d, L, G, N, m = 2048, 16, 128, 3, 8, 8, 32768
    ks = [tr.tail_len(m, 5 if i % 2 == 0 else 10, 100) for i in range(N)]
    assert ks[:2] == [1639, 3277]
    base = synth.SEED_BASE + 2
    full_units = {(3, 5), (6, 0)}       # units whose full prefill (S_m) is checked too
    groups, host, prefixes = [], [], {}
    for g in range(G):
        layers = synth.la_layers(L, D, H, d, d, seed=base * 16 + g)
        tails = []
        for i in range(N):
            if (g, i) in full_units:
                # this unit's tail is an exact slice of its full cached prefix
                hf = synth.hidden_prefix(m, D, base * 1024 + 8 * g + i)
                prefixes[(g, i)] = hf
                tails.append(hf[m - ks[i]:].contiguous())
            else:
                # the tail of hit i at group g's entry: the last k_i cached hiddens (drawn directly)
                tails.append(synth.hidden_prefix(ks[i], D, base * 1024 + 8 * g + i))
        h = torch.cat(tails)
        cu = synth.cu_seqlens_of(ks)
        host.append((tails, layers, h, cu))
        groups.append(tr.GroupReplay(h.to(cuda_device), cu, to_dev(layers, cuda_device), H, d, d,
                                     skip_last_output=True))
    outs = [(S.clone(), x) for S, x in tr.GroupsReplay(groups).run()]
    torch.cuda.synchronize()
    tr.check()
    for g in range(G):
        assert torch.isfinite(outs[g][0]).all()
    # the same call on 4 lanes (concurrent streams, a workspace slice each): bitwise the same
    lanes_out = tr.GroupsReplay(groups, lanes=4).run()
    torch.cuda.synchronize()
    tr.check()
    for g in range(G):
        assert torch.equal(lanes_out[g][0], outs[g][0]), g
    # the oracle on all 64 (hit, group) tails: one packed oracle call per group
    for g in range(G):
        tails, layers, h, cu = host[g]
        wS, _ = oracle.replay_group(h, cu, layers, H, d, d, skip_last_output=True)
        for i in range(N):
            for l in range(L):
                assert rel_fro(outs[g][0][l, i:i + 1], wS[l, i:i + 1]) < TOL, (g, i, l)
    # a unit replayed alone equals the same unit inside the packed batch, bitwise
    for g, i in sorted(full_units):
        tails, layers, _, _ = host[g]
        S1, _ = tr.replay_group(tails[i].to(cuda_device), [0, ks[i]], to_dev(layers, cuda_device),
                                H, d, d, skip_last_output=True)
        assert torch.equal(S1[:, 0], outs[g][0][:, i]), (g, i)
    # full prefill of two units: S_m against the oracle, and the state error of their tails
    for g, i in sorted(full_units):
        _, layers, _, _ = host[g]
        hf = prefixes[(g, i)]
        cu_m = synth.cu_seqlens_of([m])
        S_m, _ = tr.replay_group(hf.to(cuda_device), cu_m, to_dev(layers, cuda_device), H, d, d,
                                 skip_last_output=True)
        torch.cuda.synchronize()
        tr.check()
        wS_m, _ = oracle.replay_group(hf, cu_m, layers, H, d, d, skip_last_output=True)
        for l in range(L):
            assert rel_fro(S_m[l], wS_m[l]) < TOL, (g, i, l)
        tails, layers, h, cu = host[g]
        wS_t, _ = oracle.replay_group(tails[i], [0, ks[i]], layers, H, d, d,
                                      skip_last_output=True)
        _, tot = tr.state_error(S_m.reshape(-1, d, d), outs[g][0][:, i].reshape(-1, d, d))
        _, wtot = oracle.state_error(wS_m, wS_t)
        assert abs(float(tot.item()) - wtot) <= 1e-2, (g, i, float(tot.item()), wtot)


def test_varlen_64_requests_d4096_eight_groups(cuda_device):
    D, H, d, L, G, n = 4096, 32, 128, 3, 8, 64
    seed = synth.SEED_BASE + 3
    ms = synth.varlen_prefix_lengths(n, 1024, 131072, seed)
    ks = [tr.tail_len(mi, 10, 100) for mi in ms]
    cu = synth.cu_seqlens_of(ks)
    T = int(cu[-1])
    order = sorted(range(n), key=lambda i: ks[i])
    shortest, longest = order[0], order[-1]
    a0, b0 = int(cu[shortest]), int(cu[shortest + 1])
    groups, layers_all, hs = [], [], []
    full0 = None
    for g in range(G):
        # every group's packed tails (about 3.5 GB of bf16 each), drawn on the device
        h = synth.hidden_prefix(T, D, seed * 16 + g, device=str(cuda_device))
        if g == 0:
            # the shortest request of group 0 gets a full cached prefix whose last k rows are
            # its tail, so that its full prefill (S_m) can be checked as well
            full0 = synth.hidden_prefix(ms[shortest], D, seed * 16 + 100)
            h[a0:b0] = full0[ms[shortest] - ks[shortest]:].to(cuda_device)
        layers = synth.la_layers(L, D, H, d, d, seed=seed * 16 + g)
        layers_all.append(layers)
        hs.append(h)
        groups.append(tr.GroupReplay(h, cu, to_dev(layers, cuda_device), H, d, d,
                                     skip_last_output=True))
    outs = tr.GroupsReplay(groups).run()
    torch.cuda.synchronize()
    tr.check()
    gen = torch.Generator().manual_seed(seed)
    for g in range(G):
        S = outs[g][0]
        assert S.shape == (L, n, H, d, d)
        assert torch.isfinite(S).all()
        # the oracle on the shortest request and a seeded-random one of the shorter half,
        # in every group; the longest request too in group 0
        rnd = order[int(torch.randint(1, n // 2, (1,), generator=gen))]
        picks = [shortest, rnd] + ([longest] if g == 0 else [])
        for i in picks:
            a, b = int(cu[i]), int(cu[i + 1])
            hi = hs[g][a:b].cpu()
            wS, _ = oracle.replay_group(hi, [0, b - a], layers_all[g], H, d, d,
                                        skip_last_output=True)
            for l in range(L):
                assert rel_fro(S[l, i:i + 1], wS[l]) < TOL, (g, i, ks[i], l)
        # a request replayed alone equals the same request in the batch, bitwise
        a, b = int(cu[rnd]), int(cu[rnd + 1])
        S1, _ = tr.replay_group(hs[g][a:b].contiguous(), [0, b - a],
                                to_dev(layers_all[g], cuda_device), H, d, d,
                                skip_last_output=True)
        assert torch.equal(S1[:, 0], S[:, rnd]), (g, rnd)
    # full prefill of group 0's shortest request: S_m against the oracle
    cu_m = synth.cu_seqlens_of([ms[shortest]])
    S_m, _ = tr.replay_group(full0.to(cuda_device), cu_m, to_dev(layers_all[0], cuda_device),
                             H, d, d, skip_last_output=True)
    torch.cuda.synchronize()
    tr.check()
    wS_m, _ = oracle.replay_group(full0, cu_m, layers_all[0], H, d, d, skip_last_output=True)
    for l in range(L):
        assert rel_fro(S_m[l], wS_m[l]) < TOL, l


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
        # S_m of every prefix length against the oracle (the C recurrence, all host cores)
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
            # every tail (up to 26215 tokens): S_hat_m and o against the oracle
            wo, wS_hat = oracle.gdn_scan(full.q[a:], full.k[a:], full.v[a:],
                                         full.log_alpha[a:], full.beta[a:],
                                         synth.cu_seqlens_of([k]))
            assert rel_fro(S_hat, wS_hat) < TOL, (m, r)
            assert rel_fro(o, wo) < TOL, (m, r)
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
