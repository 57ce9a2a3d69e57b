"""Pins for the fp64 oracle: facts the pages and the mathematics fix, checked on the CPU.

Each test states the passage or the mathematical fact it checks.  None of them
re-types the oracle's own formula: they use explicit transition matrices in the
paper's own (d_v x d_k) layout, closed forms, invariants, special cases, and an
independent bf16 conversion.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(20260901)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_scan(T, H, dk, dv, alpha_lo=0.5, alpha_hi=1.0, seed=0):
    r = np.random.default_rng(seed)
    q = _unit(r.standard_normal((T, H, dk)))
    k = _unit(r.standard_normal((T, H, dk)))
    v = r.standard_normal((T, H, dv))
    la = np.log(r.uniform(alpha_lo, alpha_hi, (T, H)))
    b = 1.0 / (1.0 + np.exp(-r.standard_normal((T, H))))
    return q, k, v, la, b


def _explicit_T(alpha, beta, k):
    """T_i = alpha_i (I - beta_i k_i k_i^T) as an explicit d_k x d_k matrix (Eq. (1))."""
    return alpha * (np.eye(k.shape[0]) - beta * np.outer(k, k))


# --------------------------------------------------------------- a0: tail length
def test_worked_example_tail_positions():
    """Reading notes section 2.2 worked example: m = 10,000, r = 5% -> positions 9,501..10,000."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example_tail.json")))
    k = oracle.tail_len(g["m"], g["r_num"], g["r_den"])
    assert k == g["k"]
    a, b = oracle.tail_rows(g["m"], k)
    assert (a + 1, b) == (g["first_position_1based"], g["last_position_1based"])


@pytest.mark.parametrize("m,rn,rd,k", [
    (4096, 5, 100, 205),        # ceil(204.8)
    (32768, 5, 100, 1639),      # ceil(1638.4)
    (32768, 10, 100, 3277),     # ceil(3276.8)
    (131072, 20, 100, 26215),   # ceil(26214.4)
    (100, 7, 100, 7),           # exact: 0.07 * 100 in floating point is 7.000000000000001
    (4096, 1, 100, 41),         # ceil(40.96)
    (10, 0, 1, 0),              # r = 0: the Zero-only baseline
    (0, 5, 100, 0),
    (1000, 1, 1, 1000),         # r = 1: full prefill
    (1000, 3, 2, 1000),         # r > 1 is clamped to m
])
def test_tail_len_ceiling(m, rn, rd, k):
    """Symbol table of reading notes section 2.1: k = ceil(r m)."""
    assert oracle.tail_len(m, rn, rd) == k
    # the ceiling: k-1 < r m <= k (in rationals), unless clamped
    if 0 < k < m:
        assert (k - 1) * rd < rn * m <= k * rd


# ------------------------------------------------------------ a5: Eq. (1) scan
@pytest.mark.parametrize("dk,dv,T", [(2, 3, 7), (5, 2, 12), (8, 8, 10), (3, 1, 5)])
def test_eq1_brute_force_paper_layout(dk, dv, T):
    """Eq. (1) (reading notes section 2.3) with explicit d_k x d_k matrices T_i in the
    paper's own S in R^{d_v x d_k} layout, where the key-space operator acts from the
    right (the remark after Eq. (1)): S_i = S_{i-1} T_i + beta_i v_i k_i^T, o_i = S_i q_i.
    The oracle keeps M = S^T, so M must equal S^T and o must match."""
    H = 2
    q, k, v, la, b = _rand_scan(T, H, dk, dv, seed=dk * 100 + dv)
    S0 = rng.standard_normal((1, H, dk, dv)) * 0.3
    o, S = oracle.gdn_scan(q, k, v, la, b, [0, T], S0=S0)
    for h in range(H):
        Sp = S0[0, h].T.copy()                      # d_v x d_k
        for t in range(T):
            Ti = _explicit_T(math.exp(la[t, h]), b[t, h], k[t, h])
            Sp = Sp @ Ti + b[t, h] * np.outer(v[t, h], k[t, h])
            np.testing.assert_allclose(o[t, h], Sp @ q[t, h], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[0, h], Sp.T, rtol=1e-12, atol=1e-12)


def test_error_identity_first_layer():
    """Reading notes section 2.3: E_m = S_m - S_hat_m = (T_m ... T_{a+1}) S_a with a = m - k
    (the notes' own derivation; exact for a single recurrence).  Explicit products."""
    m, k, H, dk, dv = 40, 9, 2, 6, 4
    a = m - k
    q, kk, v, la, b = _rand_scan(m, H, dk, dv, alpha_lo=0.7, seed=3)
    _, S_m = oracle.gdn_scan(q, kk, v, la, b, [0, m], want_o=False)
    _, S_a = oracle.gdn_scan(q[:a], kk[:a], v[:a], la[:a], b[:a], [0, a], want_o=False)
    _, S_hat = oracle.gdn_scan(q[a:], kk[a:], v[a:], la[a:], b[a:], [0, k], want_o=False)
    for h in range(H):
        P = np.eye(dk)
        for i in range(a, m):                       # T_m ... T_{a+1}: later factors on the left
            P = _explicit_T(math.exp(la[i, h]), b[i, h], kk[i, h]) @ P
        E = S_m[0, h] - S_hat[0, h]
        np.testing.assert_allclose(E, P @ S_a[0, h], rtol=1e-10, atol=1e-13)


def test_contraction_bound():
    """Reading notes section 2.3: with unit keys and beta in [0, 2], ||I - beta k k^T||_2 <= 1,
    so ||E_m||_F <= (prod_{i>a} alpha_i) ||S_a||_F (the rho^k bound with per-step alphas)."""
    m, k, H, dk, dv = 300, 30, 4, 16, 8
    a = m - k
    q, kk, v, la, b = _rand_scan(m, H, dk, dv, alpha_lo=0.85, seed=4)
    b = b * 2.0 * 0.999                               # beta in (0, 2)
    _, S_m = oracle.gdn_scan(q, kk, v, la, b, [0, m], want_o=False)
    _, S_a = oracle.gdn_scan(q[:a], kk[:a], v[:a], la[:a], b[:a], [0, a], want_o=False)
    _, S_hat = oracle.gdn_scan(q[a:], kk[a:], v[a:], la[a:], b[a:], [0, k], want_o=False)
    for h in range(H):
        E = np.linalg.norm(S_m[0, h] - S_hat[0, h])
        bound = math.exp(la[a:, h].sum()) * np.linalg.norm(S_a[0, h])
        assert E <= bound * (1 + 1e-9) + 1e-300


def test_zero_tail_is_zero_state():
    """k = 0 is the Zero-only baseline (reading notes section 3.1): S_hat = 0."""
    q, k, v, la, b = _rand_scan(0, 3, 4, 5)
    o, S = oracle.gdn_scan(q, k, v, la, b, [0, 0])
    assert S.shape == (1, 3, 4, 5) and not S.any()


def test_full_replay_equals_prefill():
    """k = m replays every position: S_hat_m is the full-prefill S_m (reading notes 3.1, 'Full')."""
    m = 57
    assert oracle.tail_len(m, 1, 1) == m
    q, k, v, la, b = _rand_scan(m, 2, 8, 8, seed=5)
    a, e = oracle.tail_rows(m, m)
    o1, S1 = oracle.gdn_scan(q, k, v, la, b, [0, m])
    o2, S2 = oracle.gdn_scan(q[a:e], k[a:e], v[a:e], la[a:e], b[a:e], [0, e - a])
    assert np.array_equal(S1, S2) and np.array_equal(o1, o2)


def test_identity_transition():
    """alpha = 1, beta = 0: T_i = I and the write term vanishes, so S stays S0 and o_t = S0^T q_t."""
    T, H, dk, dv = 9, 2, 6, 5
    q, k, v, la, b = _rand_scan(T, H, dk, dv, seed=6)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = oracle.gdn_scan(q, k, v, np.zeros((T, H)), np.zeros((T, H)), [0, T], S0=S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o, np.einsum("hdj,thd->thj", S0[0], q), rtol=1e-13, atol=1e-13)


def test_delta_rule_recall():
    """beta_t = 1 with a unit key: M_t^T k_t = alpha (M - k k^T M)^T k + v = v exactly (for any
    alpha), the delta rule's write.  Read out with q_t = k_t."""
    T, H, dk, dv = 20, 2, 8, 6
    _, k, v, la, _ = _rand_scan(T, H, dk, dv, alpha_lo=0.3, seed=7)
    o, _ = oracle.gdn_scan(k, k, v, la, np.ones((T, H)), [0, T])
    np.testing.assert_allclose(o, v, rtol=1e-12, atol=1e-12)


def test_orthonormal_keys_accumulate():
    """alpha = beta = 1 with orthonormal keys: each write lands in a fresh direction, so
    M_n = sum_j k_j v_j^T (closed form)."""
    dk, dv, n, H = 8, 5, 6, 1
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :n].T.reshape(n, 1, dk)
    v = rng.standard_normal((n, H, dv))
    _, S = oracle.gdn_scan(k, k, v, np.zeros((n, H)), np.ones((n, H)), [0, n], want_o=False)
    np.testing.assert_allclose(S[0, 0], sum(np.outer(k[j, 0], v[j, 0]) for j in range(n)),
                               rtol=1e-12, atol=1e-12)


def test_scalar_recurrence_closed_form():
    """d_k = d_v = 1 reduces Eq. (1) to m_i = a_i m_{i-1} + b_i with a_i = alpha_i (1 - beta_i k_i^2),
    b_i = beta_i k_i v_i, whose solution is m_n = sum_j (prod_{i>j} a_i) b_j + (prod a_i) m_0."""
    T = 30
    r = np.random.default_rng(8)
    k = r.uniform(-1.2, 1.2, (T, 1, 1))
    v = r.standard_normal((T, 1, 1))
    la = np.log(r.uniform(0.6, 1.0, (T, 1)))
    b = r.uniform(0.0, 1.0, (T, 1))
    m0 = np.array([[[[0.7]]]])
    _, S = oracle.gdn_scan(k, k, v, la, b, [0, T], S0=m0, want_o=False)
    a = np.exp(la[:, 0]) * (1 - b[:, 0] * k[:, 0, 0] ** 2)
    bb = b[:, 0] * k[:, 0, 0] * v[:, 0, 0]
    expect = np.prod(a) * 0.7 + sum(np.prod(a[j + 1:]) * bb[j] for j in range(T))
    assert abs(S[0, 0, 0, 0] - expect) < 1e-12


def test_split_composition_and_varlen():
    """Scanning x[:t] and then x[t:] from the state reached equals scanning x; packing two
    sequences with cu_seqlens equals two separate calls (both exactly, in the oracle)."""
    T, H, dk, dv = 45, 3, 8, 4
    q, k, v, la, b = _rand_scan(T, H, dk, dv, seed=9)
    o, S = oracle.gdn_scan(q, k, v, la, b, [0, T])
    t = 17
    o1, S1 = oracle.gdn_scan(q[:t], k[:t], v[:t], la[:t], b[:t], [0, t])
    o2, S2 = oracle.gdn_scan(q[t:], k[t:], v[t:], la[t:], b[t:], [0, T - t], S0=S1)
    assert np.array_equal(S2, S) and np.array_equal(np.concatenate([o1, o2]), o)
    op, Sp = oracle.gdn_scan(q, k, v, la, b, [0, t, T])
    assert np.array_equal(Sp[0], S1[0]) and np.array_equal(op[:t], o1)
    _, Sb = oracle.gdn_scan(q[t:], k[t:], v[t:], la[t:], b[t:], [0, T - t])
    assert np.array_equal(Sp[1], Sb[0])


def test_scan_normalize_flag_matches_prenormalised():
    T, H, d = 12, 2, 8
    r = np.random.default_rng(10)
    q, k = r.standard_normal((T, H, d)) * 3, r.standard_normal((T, H, d)) * 0.2
    _, _, v, la, b = _rand_scan(T, H, d, d, seed=10)
    o1, S1 = oracle.gdn_scan(q, k, v, la, b, [0, T], normalize_qk=True, norm_eps=0.0)
    o2, S2 = oracle.gdn_scan(_unit(q), _unit(k), v, la, b, [0, T])
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)


# -------------------------------------------------------- a2-a4, a6 layer pieces
def test_bf16_round_matches_independent_conversion():
    """The oracle's bit-level bf16 rounding agrees with torch's own fp32 -> bf16 conversion,
    including ties to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 and rounds to 1."""
    x = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-20, 20, 10000),
                        [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0, 65504.0]])
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.bf16_round(x32), ref)
    assert oracle.bf16_round(np.array([1 + 2 ** -8]))[0] == 1.0
    assert oracle.bf16_round(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


def test_rmsnorm_special_cases():
    """x = +-c has mean square c^2, so x_hat = +-c / sqrt(c^2 + eps) * g; scale invariance."""
    D = 64
    c = 3.0
    x = np.where(np.arange(D) % 2 == 0, c, -c)[None]
    g = rng.uniform(0.5, 1.5, D)
    y = oracle.rmsnorm(x, g, eps=1e-6)
    np.testing.assert_allclose(y[0], np.sign(x[0]) * c / math.sqrt(c * c + 1e-6) * g, rtol=1e-14)
    z = rng.standard_normal((5, D))
    np.testing.assert_allclose(oracle.rmsnorm(z * 1e3, eps=0.0), oracle.rmsnorm(z, eps=0.0), rtol=1e-12)
    np.testing.assert_allclose(np.mean(oracle.rmsnorm(z, eps=0.0) ** 2, axis=1), 1.0, rtol=1e-12)


def test_l2_normalize():
    y = oracle.l2_normalize(np.array([[3.0, 4.0]]), eps=0.0)
    np.testing.assert_allclose(y, [[0.6, 0.8]], rtol=1e-15)
    z = rng.standard_normal((7, 3, 16))
    np.testing.assert_allclose(np.linalg.norm(oracle.l2_normalize(z, 0.0), axis=-1), 1.0, rtol=1e-13)


def test_gates_identities():
    """alpha = exp(-softplus(a)) = 1/(1 + e^a): alpha(0) = 1/2; log alpha(-a) - log alpha(a) = a;
    beta(a) + beta(-a) = 1; alpha in (0, 1), beta in (0, 1); no overflow at |a| = 800."""
    a = np.concatenate([rng.standard_normal(1000) * 5, [0.0, 30.0, -30.0, 800.0, -800.0]])
    la, b = oracle.gates(a, a)
    la_n, b_n = oracle.gates(-a, -a)
    assert np.all(np.isfinite(la)) and np.all(la <= 0)
    np.testing.assert_allclose(la_n - la, a, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b + b_n, 1.0, rtol=0, atol=1e-15)
    mid = np.abs(a) < 30
    np.testing.assert_allclose(np.exp(la[mid]), 1.0 / (1.0 + np.exp(a[mid])), rtol=1e-13)
    la0, b0 = oracle.gates(np.array([0.0]), np.array([0.0]))
    assert abs(la0[0] + math.log(2)) < 1e-16 and b0[0] == 0.5
    assert np.all((b >= 0) & (b <= 1))


def test_in_projection_split_order():
    """One-hot weight rows pick input columns: checks the [q | k | v | a_alpha | a_beta] split and
    the head-major order inside q, k, v."""
    H, dk, dv = 2, 3, 2
    n = synth.in_features(H, dk, dv)
    D = n
    W = np.eye(n)[np.arange(n)[::-1]]            # row r picks input column n-1-r
    x = rng.standard_normal((4, D))
    q, k, v, aa, ab = oracle.in_projection(x, W, H, dk, dv)
    col = lambda r: x[:, n - 1 - r]
    np.testing.assert_array_equal(q[:, 1, 2], col(1 * dk + 2))
    np.testing.assert_array_equal(k[:, 0, 1], col(H * dk + 1))
    np.testing.assert_array_equal(v[:, 1, 0], col(2 * H * dk + dv))
    np.testing.assert_array_equal(aa[:, 1], col(2 * H * dk + H * dv + 1))
    np.testing.assert_array_equal(ab[:, 0], col(2 * H * dk + H * dv + H))


def test_out_projection_residual():
    T, H, dv, D = 3, 2, 4, 5
    x = rng.standard_normal((T, D))
    o = rng.standard_normal((T, H, dv))
    np.testing.assert_array_equal(oracle.out_projection_residual(x, o, np.zeros((D, H * dv))), x)
    onehot = np.zeros((T, H, dv)); onehot[:, 1, 2] = 1.0
    W = rng.standard_normal((D, H * dv))
    np.testing.assert_allclose(oracle.out_projection_residual(x, onehot, W), x + W[:, dv + 2][None],
                               rtol=1e-15)


# ------------------------------------------------------------ a6b FFN sublayer
def test_silu_closed_forms():
    """silu(z) = z sigmoid(z): library routine, odd-part identity, known values, limits."""
    z = np.linspace(-30.0, 30.0, 241)
    np.testing.assert_allclose(oracle.silu(z), torch.nn.functional.silu(torch.from_numpy(z)).numpy(),
                               rtol=1e-14, atol=1e-300)
    # silu(z) - silu(-z) = z (sigmoid(z) + sigmoid(-z) = 1)
    np.testing.assert_allclose(oracle.silu(z) - oracle.silu(-z), z, rtol=1e-13, atol=1e-13)
    assert oracle.silu([0.0])[0] == 0.0
    assert abs(oracle.silu([1.0])[0] - math.e / (1.0 + math.e)) < 1e-15   # sigmoid(1)
    big = oracle.silu([800.0, -800.0])
    assert big[0] == 800.0 and big[1] == 0.0
    # slope 1/2 at the origin
    eps = 1e-6
    assert abs((oracle.silu([eps])[0] - oracle.silu([-eps])[0]) / (2 * eps) - 0.5) < 1e-9


def test_ffn_residual_worked_case():
    """D = 2, d_ff = 1: x = [1, -1] has RMS 1, so x_hat = x; g = 1, u = 1, and the FFN adds
    sigmoid(1) times the down column."""
    x = np.array([[1.0, -1.0]])
    Wg = np.array([[1.0, 0.0]])
    Wu = np.array([[0.0, -1.0]])
    Wd = np.array([[2.0], [3.0]])
    y = oracle.ffn_residual(x, Wg, Wu, Wd, rms_eps=0.0, emulate_casts=False)
    s1 = math.e / (1.0 + math.e)
    np.testing.assert_allclose(y, [[1.0 + 2 * s1, -1.0 + 3 * s1]], rtol=1e-15)
    # a gain scales x_hat: gain [2, 1] -> g = 2, u = 1
    y2 = oracle.ffn_residual(x, Wg, Wu, Wd, ffn_gain=np.array([2.0, 1.0]), rms_eps=0.0,
                             emulate_casts=False)
    s2 = 2.0 * math.exp(2.0) / (1.0 + math.exp(2.0))
    np.testing.assert_allclose(y2, [[1.0 + 2 * s2, -1.0 + 3 * s2]], rtol=1e-15)


def test_ffn_residual_invariants():
    """Zero down or up weights leave x; flipping the gate's sign changes the sublayer's output
    by exactly (g * u) W_down^T, since silu(z) - silu(-z) = z; the sublayer depends on x only
    through RMSNorm(x), so scaling x scales only the residual."""
    T, D, F = 5, 12, 20
    x = rng.standard_normal((T, D))
    Wg = rng.standard_normal((F, D)) * 0.3
    Wu = rng.standard_normal((F, D)) * 0.3
    Wd = rng.standard_normal((D, F)) * 0.3
    gain = 1.0 + 0.1 * rng.standard_normal(D)
    np.testing.assert_array_equal(oracle.ffn_residual(x, Wg, Wu, np.zeros((D, F))), x)
    np.testing.assert_array_equal(oracle.ffn_residual(x, Wg, np.zeros((F, D)), Wd), x)
    f_pos = oracle.ffn_residual(x, Wg, Wu, Wd, gain, rms_eps=0.0, emulate_casts=False) - x
    f_neg = oracle.ffn_residual(x, -Wg, Wu, Wd, gain, rms_eps=0.0, emulate_casts=False) - x
    # x_hat by hand: x / RMS(x) * gain
    xh = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True)) * gain
    np.testing.assert_allclose(f_pos - f_neg, ((xh @ Wg.T) * (xh @ Wu.T)) @ Wd.T,
                               rtol=1e-11, atol=1e-12)
    f_scaled = oracle.ffn_residual(3.5 * x, Wg, Wu, Wd, gain, rms_eps=0.0,
                                   emulate_casts=False) - 3.5 * x
    np.testing.assert_allclose(f_scaled, f_pos, rtol=1e-11, atol=1e-12)
    # the bf16 cast points move the sublayer's output by about bf16 precision only
    f_c = oracle.ffn_residual(x, Wg, Wu, Wd, gain) - x
    f_e = oracle.ffn_residual(x, Wg, Wu, Wd, gain, emulate_casts=False) - x
    rel = np.linalg.norm(f_c - f_e) / np.linalg.norm(f_e)
    assert 0 < rel < 2e-2


# ------------------------------------------- Gated DeltaNet details (optional)
def test_short_conv_against_library_convolution():
    """Per sequence and channel, the causal convolution is numpy's full convolution with the
    taps reversed, cut to the sequence (zero history), then silu."""
    lengths = [7, 0, 1, 12]
    C, W = 5, 4
    x = rng.standard_normal((sum(lengths), C))
    w = rng.standard_normal((C, W))
    cu = np.cumsum([0] + lengths)
    y = oracle.short_conv(x, w, cu)
    for s_ in range(len(lengths)):
        a, b = cu[s_], cu[s_ + 1]
        if a == b:
            continue
        for c in range(C):
            ref = np.convolve(x[a:b, c], w[c, ::-1])[:b - a]
            np.testing.assert_allclose(y[a:b, c], torch.nn.functional.silu(
                torch.from_numpy(ref)).numpy(), rtol=1e-13, atol=1e-15)


def test_short_conv_taps_and_state():
    """The current-token tap alone is pointwise; the oldest tap alone shifts by W-1 with zeros
    at each sequence start; continuing a sequence from its convolution state gives the same
    outputs as convolving it whole (the state holds the last W-1 inputs, oldest first)."""
    lengths = [9, 2, 6]
    C, W = 3, 4
    x = rng.standard_normal((sum(lengths), C))
    cu = np.cumsum([0] + lengths)
    cur = np.zeros((C, W)); cur[:, W - 1] = 1.5
    np.testing.assert_allclose(oracle.short_conv(x, cur, cu), oracle.silu(1.5 * x), rtol=1e-15)
    old = np.zeros((C, W)); old[:, 0] = 1.0
    y = oracle.short_conv(x, old, cu)
    for s_ in range(3):
        a, b = cu[s_], cu[s_ + 1]
        want = np.zeros((b - a, C))
        want[W - 1:] = x[a:b - (W - 1)] if b - a > W - 1 else want[W - 1:]
        np.testing.assert_allclose(y[a:b], oracle.silu(want), rtol=1e-15, atol=0)
    st = oracle.conv_state(x, W, cu)
    assert st.shape == (3, W - 1, C)
    np.testing.assert_array_equal(st[0], x[6:9])
    np.testing.assert_array_equal(st[1, 0], 0.0)           # length 2 < W - 1: zero-padded
    np.testing.assert_array_equal(st[1, 1:], x[9:11])
    # continuation: [x_0 .. x_8] split at 5; state of the head + tail == whole
    w = rng.standard_normal((C, W))
    whole = oracle.short_conv(x[:9], w, [0, 9])
    head_state = oracle.conv_state(x[:5], W, [0, 5])[0]
    cont = oracle.short_conv(np.concatenate([head_state, x[5:9]]), w, [0, W - 1 + 4])
    np.testing.assert_allclose(cont[W - 1:], whole[5:], rtol=1e-14)
    assert not oracle.conv_state(np.zeros((0, C)), W, [0, 0]).any()


def test_gated_rmsnorm_library_and_identities():
    T, H, dv = 4, 3, 8
    o = rng.standard_normal((T, H, dv))
    z = rng.standard_normal((T, H, dv))
    g = 1.0 + 0.1 * rng.standard_normal(dv)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (dv,), torch.from_numpy(g), eps=1e-6)
    ref = ref * torch.nn.functional.silu(torch.from_numpy(z))
    np.testing.assert_allclose(oracle.gated_rmsnorm(o, z, g, 1e-6), ref.numpy(), rtol=1e-12)
    assert not oracle.gated_rmsnorm(o, np.zeros_like(z), g).any()           # silu(0) = 0
    np.testing.assert_allclose(oracle.gated_rmsnorm(4.0 * o, z, g, 0.0),
                               oracle.gated_rmsnorm(o, z, g, 0.0), rtol=1e-14)
    c = np.full((1, 1, dv), -2.5)                                          # RMS = 2.5
    np.testing.assert_allclose(oracle.gated_rmsnorm(c, np.ones_like(c), None, 0.0),
                               -np.full_like(c, math.e / (1 + math.e)), rtol=1e-15)


def test_gate_parameters():
    """dt_bias shifts the softplus argument, exp(A_log) scales log alpha, zeros change nothing."""
    T, H = 6, 4
    a, b = rng.standard_normal((T, H)) * 3, rng.standard_normal((T, H))
    la0, b0 = oracle.gates(a, b)
    la1, b1 = oracle.gates(a, b, np.zeros(H), np.zeros(H))
    np.testing.assert_array_equal(la0, la1)
    np.testing.assert_array_equal(b0, b1)
    bias = np.array([-3.0, 0.5, 2.0, -7.0])
    np.testing.assert_allclose(oracle.gates(a, b, None, bias)[0], oracle.gates(a + bias, b)[0],
                               rtol=1e-15)
    A_log = np.log(np.array([1.0, 2.0, 3.0, 16.0]))
    np.testing.assert_allclose(oracle.gates(a, b, A_log)[0], la0 * np.exp(A_log), rtol=1e-15)
    assert np.all(oracle.gates(a, b, A_log, bias)[0] < 0)                   # alpha in (0, 1)


def _tiny_gdn_group(lengths, D=48, H=2, dk=8, dv=8, L=2, seed=17, **kw):
    layers = synth.la_layers(L, D, H, dk, dv, seed=seed, std=0.2, with_gain=True, **kw)
    h = torch.cat([synth.hidden_prefix(n, D, seed + i) for i, n in enumerate(lengths)])
    return h, layers, synth.cu_seqlens_of(lengths)


def test_replay_short_conv_zero_history_and_state():
    """With the convolution the tail replay gives layer 0 the same keys as the full replay
    except for the first W-1 tail tokens, whose history the zero start drops; with the
    current-token tap alone it drops nothing and the first layer's error identity of the
    reading notes (section 2.3) holds again.  Each layer's returned convolution state is the
    last W-1 rows of its bf16 pre-convolution projection."""
    m, H, dk, W = 30, 2, 8, 4
    kk = oracle.tail_len(m, 30, 100)                   # 9
    a = m - kk
    h, layers, _ = _tiny_gdn_group([m], conv_width=W)
    lw = layers[0]
    x_hat = oracle.bf16_round(oracle.rmsnorm(h, lw.rms_gain))
    q, k, v, _, _ = oracle.in_projection(x_hat, lw.W_in, H, dk, dk)
    pre = oracle.bf16_round(np.concatenate([q.reshape(m, -1), k.reshape(m, -1),
                                            v.reshape(m, -1)], 1))
    y_full = oracle.short_conv(pre, lw.conv_w, [0, m])
    y_tail = oracle.short_conv(pre[a:], lw.conv_w, [0, kk])
    np.testing.assert_array_equal(y_tail[W - 1:], y_full[a + W - 1:])
    assert np.abs(y_tail[:W - 1] - y_full[a:a + W - 1]).max() > 1e-3
    states = []
    oracle.replay_group(h[a:], [0, kk], layers, H, dk, dk, conv_states=states)
    assert len(states) == 2
    np.testing.assert_array_equal(states[0][0], pre[m - (W - 1):])
    # current-token tap only: the first layer's error identity holds
    cur = [synth.LALayerWeights(l.W_in, l.W_o, l.rms_gain, conv_w=torch.zeros_like(l.conv_w))
           for l in layers]
    for l in cur:
        l.conv_w[:, W - 1] = 0.8
    S_full, _ = oracle.replay_group(h, [0, m], cur, H, dk, dk)
    S_tail, _ = oracle.replay_group(h[a:], [0, kk], cur, H, dk, dk)
    S_a, _ = oracle.replay_group(h[:a], [0, a], cur, H, dk, dk)
    k0 = oracle.bf16_round(oracle.l2_normalize(oracle.silu(0.8 * pre[:, H * dk:2 * H * dk])
                                               .reshape(m, H, dk)))
    _, _, _, aa, ab = oracle.in_projection(x_hat, lw.W_in, H, dk, dk)
    la, b = oracle.gates(aa, ab)
    for hh in range(H):
        P = np.eye(dk)
        for i in range(a, m):
            P = _explicit_T(math.exp(la[i, hh]), b[i, hh], k0[i, hh]) @ P
        np.testing.assert_allclose(S_full[0, 0, hh] - S_tail[0, 0, hh], P @ S_a[0, 0, hh],
                                   rtol=1e-9, atol=1e-12)


def test_replay_output_gate_and_gate_parameters():
    """The output gate acts after the scan: layer 0's states do not see it, layer 1's do; a
    zero output-norm gain silences the attention sublayer (x passes unchanged); the gate
    parameters change the first layer's states through alpha only."""
    lengths = [11, 0, 6]
    H, dk = 2, 8
    h, layers, cu = _tiny_gdn_group(lengths, output_gate=True, gate_params=True)
    S, x = oracle.replay_group(h, cu, layers, H, dk, dk, output_gate=True)
    no_gp = [synth.LALayerWeights(l.W_in, l.W_o, l.rms_gain, o_norm_gain=l.o_norm_gain)
             for l in layers]
    S_ng, _ = oracle.replay_group(h, cu, no_gp, H, dk, dk, output_gate=True)
    assert np.abs(S[0] - S_ng[0]).max() > 1e-6
    # the z rows removed: the same layers without the output gate
    n_plain = synth.in_features(H, dk, dk)
    plain = []
    for l in layers:
        W = l.W_in
        W_no_z = torch.cat([W[:2 * H * dk + H * dk], W[2 * H * dk + 2 * H * dk:]])
        assert W_no_z.shape[0] == n_plain
        plain.append(synth.LALayerWeights(W_no_z, l.W_o, l.rms_gain, A_log=l.A_log,
                                          dt_bias=l.dt_bias))
    S_p, _ = oracle.replay_group(h, cu, plain, H, dk, dk)
    np.testing.assert_array_equal(S[0], S_p[0])
    assert np.abs(S[1] - S_p[1]).max() > 1e-6
    silent = [synth.LALayerWeights(l.W_in, l.W_o, l.rms_gain, A_log=l.A_log, dt_bias=l.dt_bias,
                                   o_norm_gain=torch.zeros_like(l.o_norm_gain)) for l in layers]
    _, x_s = oracle.replay_group(h[:11], [0, 11], silent[:1], H, dk, dk, output_gate=True)
    np.testing.assert_array_equal(x_s, h[:11].double().numpy())


def test_replay_ffn_with_gdn_options():
    """With the FFN and every Gated DeltaNet option in one group: layer 0's states see no
    FFN, the last FFN changes no state, and zero down weights give the FFN-free group."""
    lengths = [14, 5]
    H, dk = 2, 8
    h, layers, cu = _tiny_gdn_group(lengths, L=3, conv_width=3, gate_params=True,
                                    output_gate=True, d_ff=32)
    S_f, x_f = oracle.replay_group(h, cu, layers, H, dk, dk, output_gate=True,
                                   skip_last_ffn=False)
    S_s, _ = oracle.replay_group(h, cu, layers, H, dk, dk, output_gate=True)
    no_ffn = [synth.LALayerWeights(l.W_in, l.W_o, l.rms_gain, conv_w=l.conv_w, A_log=l.A_log,
                                   dt_bias=l.dt_bias, o_norm_gain=l.o_norm_gain) for l in layers]
    S_n, x_n = oracle.replay_group(h, cu, no_ffn, H, dk, dk, output_gate=True)
    np.testing.assert_array_equal(S_f, S_s)
    np.testing.assert_array_equal(S_f[0], S_n[0])
    assert np.abs(S_f[1] - S_n[1]).max() > 1e-6
    zero = [synth.LALayerWeights(l.W_in, l.W_o, l.rms_gain, l.W_gate, l.W_up,
                                 torch.zeros_like(l.W_down), None, l.conv_w, l.A_log, l.dt_bias,
                                 l.o_norm_gain) for l in layers]
    S_z, x_z = oracle.replay_group(h, cu, zero, H, dk, dk, output_gate=True, skip_last_ffn=False)
    np.testing.assert_array_equal(S_z, S_n)
    np.testing.assert_array_equal(x_z, x_n)


# ---------------------------------------------------------------- a8 state error
def test_state_error_cases():
    S = rng.standard_normal((3, 4, 5))
    per, tot = oracle.state_error(S, S)
    assert tot == 0 and not per.any()
    per, tot = oracle.state_error(S, np.zeros_like(S))
    np.testing.assert_allclose(per, 1.0); assert abs(tot - 1.0) < 1e-15
    Z = np.zeros((2, 4, 5))
    per, tot = oracle.state_error(Z, Z)
    assert tot == 0.0 and not per.any()
    Y = Z.copy(); Y[1, 0, 0] = 1e-3
    per, _ = oracle.state_error(Z, Y)
    assert per[0] == 0.0 and per[1] == np.inf
    per, tot = oracle.state_error(S, 0.5 * S)
    np.testing.assert_allclose(per, 0.5, rtol=1e-15)


# ------------------------------------------------------------ group replay (a2-a7)
def _tiny_group(lengths, D=48, H=2, dk=8, dv=8, L=3, seed=11):
    layers = synth.la_layers(L, D, H, dk, dv, seed=seed, std=0.2, with_gain=True)
    h = torch.cat([synth.hidden_prefix(n, D, seed + i) for i, n in enumerate(lengths)])
    return h, layers, synth.cu_seqlens_of(lengths)


def test_replay_first_layer_error_identity():
    """In the replay of a group, the first LA layer sees exact inputs (reading notes section 2.4),
    so for it E_m = (T_m ... T_{a+1}) S_a holds with the gates and keys that layer computes; the
    later layers see the replayed layers' outputs (the cross-layer recurrence of section 2.3) and
    only have to stay finite."""
    m, D, H, dk, dv = 30, 48, 2, 8, 8
    kk = oracle.tail_len(m, 30, 100)                  # 9
    a = m - kk
    h, layers, _ = _tiny_group([m], D, H, dk, dv)
    S_full, _ = oracle.replay_group(h, [0, m], layers, H, dk, dv)
    S_tail, _ = oracle.replay_group(h[a:], [0, kk], layers, H, dk, dv)
    S_a, _ = oracle.replay_group(h[:a], [0, a], layers, H, dk, dv)
    # rebuild layer 0's keys and gates independently from the pieces
    lw = layers[0]
    x_hat = oracle.bf16_round(oracle.rmsnorm(h, lw.rms_gain))
    _, k, _, aa, ab = oracle.in_projection(x_hat, lw.W_in, H, dk, dv)
    k = oracle.bf16_round(oracle.l2_normalize(k))
    la, b = oracle.gates(aa, ab)
    for hh in range(H):
        P = np.eye(dk)
        for i in range(a, m):
            P = _explicit_T(math.exp(la[i, hh]), b[i, hh], k[i, hh]) @ P
        np.testing.assert_allclose(S_full[0, 0, hh] - S_tail[0, 0, hh], P @ S_a[0, 0, hh],
                                   rtol=1e-9, atol=1e-12)
    assert np.all(np.isfinite(S_full - S_tail))


def test_replay_zero_and_full_and_skip():
    lengths = [13, 0, 21]
    h, layers, cu = _tiny_group(lengths)
    S, x = oracle.replay_group(h, cu, layers, 2, 8, 8)
    assert S.shape == (3, 3, 2, 8, 8)
    assert not S[:, 1].any()                         # k = 0: Zero-only state
    S2, x2 = oracle.replay_group(h, cu, layers, 2, 8, 8, skip_last_output=True)
    assert x2 is None and np.array_equal(S, S2)      # the skipped output feeds no state
    # packed requests equal separate replays (groups, heads and requests are independent)
    Sa, xa = oracle.replay_group(h[:13], [0, 13], layers, 2, 8, 8)
    Sb, xb = oracle.replay_group(h[13:], [0, 21], layers, 2, 8, 8)
    np.testing.assert_allclose(S[:, 0], Sa[:, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S[:, 2], Sb[:, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(x, np.concatenate([xa, xb]), rtol=1e-12, atol=1e-12)


def test_replay_cast_points_are_small():
    """The bf16 cast points of the boundary move the states by about bf16 precision only."""
    h, layers, cu = _tiny_group([40, 25], D=64, H=2, dk=16, dv=16)
    S_c, _ = oracle.replay_group(h, cu, layers, 2, 16, 16, emulate_casts=True)
    S_e, _ = oracle.replay_group(h, cu, layers, 2, 16, 16, emulate_casts=False)
    _, tot = oracle.state_error(S_e, S_c)
    assert 0 < tot < 2e-2


def test_folded_norm_cast_point_is_the_same_math():
    """The layers after a group's first take RMSNorm(x) W_in^T as (1/rms) ((x * gain) W_in^T),
    the bf16 rounding on x * gain: in exact arithmetic (no casts) that is the plain RMSNorm
    and projection to fp64 rounding, with the gain and the 1/rms both in play; with the
    casts the two orders differ by bf16 rounding only."""
    h, layers, cu = _tiny_group([40, 25], D=64, H=2, dk=16, dv=16)
    lw = layers[1]
    x = synth.normal((65, 64), 17, 3).double() * 3.0     # rows of very different rms
    gain = torch.linspace(0.5, 1.5, 64, dtype=torch.float64)
    for g in (None, gain):
        S_a, x_a = oracle.replay_layer(x, lw.W_in, lw.W_o, g, cu, 2, 16, 16, emulate_casts=False)
        S_b, x_b = oracle.replay_layer(x, lw.W_in, lw.W_o, g, cu, 2, 16, 16, emulate_casts=False,
                                       fold_norm=True)
        np.testing.assert_allclose(S_b, S_a, rtol=1e-10, atol=1e-13)
        np.testing.assert_allclose(x_b, x_a, rtol=1e-10, atol=1e-12)
        S_c, _ = oracle.replay_layer(x, lw.W_in, lw.W_o, g, cu, 2, 16, 16, fold_norm=True)
        _, tot = oracle.state_error(S_a, S_c)
        assert 0 < tot < 2e-2


def _tiny_ffn_group(lengths, D=48, H=2, dk=8, dv=8, L=3, F=64, seed=11):
    layers = synth.la_layers(L, D, H, dk, dv, seed=seed, std=0.2, with_gain=True, d_ff=F)
    h = torch.cat([synth.hidden_prefix(n, D, seed + i) for i, n in enumerate(lengths)])
    return h, layers, synth.cu_seqlens_of(lengths)


def _without_ffn(layers):
    return [synth.LALayerWeights(lw.W_in, lw.W_o, lw.rms_gain) for lw in layers]


def test_replay_group_ffn_placement_and_tail_skip():
    """RN section 2.5: the FFNs between a group's LA layers feed the next LA layer; the last
    layer's FFN feeds no state and is skipped.  So: the first layer's state sees no FFN; the
    last layer's FFN changes no state; an FFN with zero down weights is no FFN; the skipped
    FFN, applied to the skip's x_out, gives the unskipped x_out."""
    lengths = [17, 0, 9]
    H, dk = 2, 8
    h, layers, cu = _tiny_ffn_group(lengths)
    plain = _without_ffn(layers)
    S_f, x_skip = oracle.replay_group(h, cu, layers, H, dk, dk)               # tail skip (default)
    S_n, x_n = oracle.replay_group(h, cu, plain, H, dk, dk)
    S_u, x_full = oracle.replay_group(h, cu, layers, H, dk, dk, skip_last_ffn=False)
    np.testing.assert_array_equal(S_f[0], S_n[0])                # layer 0's state: no FFN before it
    assert np.abs(S_f[1] - S_n[1]).max() > 1e-3                  # the layer-0 FFN feeds layer 1
    np.testing.assert_array_equal(S_u, S_f)                      # the last FFN feeds no state
    last = layers[-1]
    np.testing.assert_allclose(x_full, oracle.ffn_residual(x_skip, last.W_gate, last.W_up,
                                                           last.W_down, last.ffn_gain),
                               rtol=1e-13, atol=1e-13)
    S_o, _ = oracle.replay_group(h, cu, layers, H, dk, dk, skip_last_output=True)
    np.testing.assert_array_equal(S_o, S_f)
    # zero down weights: the FFN adds nothing
    zeroed = [synth.LALayerWeights(lw.W_in, lw.W_o, lw.rms_gain, lw.W_gate, lw.W_up,
                                   torch.zeros_like(lw.W_down), lw.ffn_gain) for lw in layers]
    S_z, x_z = oracle.replay_group(h, cu, zeroed, H, dk, dk, skip_last_ffn=False)
    np.testing.assert_array_equal(S_z, S_n)
    np.testing.assert_array_equal(x_z, x_n)
    # a one-layer group with the tail skip is the plain LA layer
    S1, x1 = oracle.replay_group(h, cu, layers[:1], H, dk, dk)
    S1n, x1n = oracle.replay_group(h, cu, plain[:1], H, dk, dk)
    np.testing.assert_array_equal(S1, S1n)
    np.testing.assert_array_equal(x1, x1n)
    assert not S_f[:, 1].any()                                   # k = 0: zero state
    # packed requests equal separate replays
    Sa, xa = oracle.replay_group(h[:17], [0, 17], layers, H, dk, dk, skip_last_ffn=False)
    np.testing.assert_allclose(S_u[:, 0], Sa[:, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(x_full[:17], xa, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------- transition product (HYPIC operator)
def test_transition_product_explicit_matrices():
    """Reading notes section 2.3: the tail's operator is the product T_t ... T_1 of the
    explicit d_k x d_k matrices T_i = alpha_i (I - beta_i k_i k_i^T); varlen sequences are
    independent and an empty one gives the identity."""
    q, k, v, la, b = _rand_scan(17, 2, 6, 3, seed=31)
    cu = [0, 9, 9, 17]
    P = oracle.transition_product(k, la, b, cu)
    for n in range(3):
        for h in range(2):
            want = np.eye(6)
            for t in range(cu[n], cu[n + 1]):
                want = _explicit_T(math.exp(la[t, h]), b[t, h], k[t, h]) @ want
            np.testing.assert_allclose(P[n, h], want, atol=1e-14)


def test_transition_product_is_the_scans_linear_part():
    """Eq. (1) is affine in the state: scan(S0) - scan(0) = P S0 (in the M = S^T layout),
    checked against the plain C recurrence, which never forms P."""
    q, k, v, la, b = _rand_scan(40, 3, 8, 5, seed=32)
    S0 = rng.standard_normal((2, 3, 8, 5))
    cu = [0, 25, 40]
    _, S1 = oracle.gdn_scan(q, k, v, la, b, cu, S0=S0, want_o=False)
    _, Sz = oracle.gdn_scan(q, k, v, la, b, cu, want_o=False)
    P = oracle.transition_product(k, la, b, cu)
    np.testing.assert_allclose(S1 - Sz, np.einsum('nhij,nhjk->nhik', P, S0), atol=1e-12)


def test_transition_product_identity_and_bound():
    """alpha = 1, beta = 0 gives P = I; with unit keys and beta in (0, 1) every T_i is a
    contraction times alpha_i, so ||P||_2 <= prod alpha_i (reading notes section 2.3)."""
    q, k, v, la, b = _rand_scan(30, 2, 8, 4, seed=33)
    P0 = oracle.transition_product(k, np.zeros_like(la), np.zeros_like(b), [0, 30])
    np.testing.assert_allclose(P0[0], np.broadcast_to(np.eye(8), (2, 8, 8)), atol=0)
    P = oracle.transition_product(k, la, b, [0, 30])
    for h in range(2):
        assert np.linalg.norm(P[0, h], 2) <= math.exp(la[:, h].sum()) * (1 + 1e-12)


def test_transition_product_composes():
    """The operator of a span is the later part's times the earlier part's, for any split
    (T_m ... T_1 = (T_m ... T_{c+1})(T_c ... T_1)), and a packed batch of two spans gives
    each span's operator."""
    q, k, v, la, b = _rand_scan(30, 2, 8, 4, seed=35)
    P_all = oracle.transition_product(k, la, b, [0, 30])[0]
    for c in (1, 12, 29):
        P_pair = oracle.transition_product(k, la, b, [0, c, 30])
        for h in range(2):
            np.testing.assert_allclose(P_pair[1, h] @ P_pair[0, h], P_all[h], rtol=1e-12,
                                       atol=1e-15)
        np.testing.assert_allclose(P_pair[0], oracle.transition_product(
            k[:c], la[:c], b[:c], [0, c])[0], rtol=1e-15, atol=0)


def test_transition_product_repairs_the_tail():
    """The repair the operator makes possible: with an exact earlier state S_a, the full
    state is S_m = P S_a + S_hat_m exactly (reading notes section 2.3, E_m = P S_a)."""
    m, kk = 60, 22
    q, k, v, la, b = _rand_scan(m, 2, 8, 6, seed=34)
    a = m - kk
    _, S_m = oracle.gdn_scan(q, k, v, la, b, [0, m], want_o=False)
    _, S_a = oracle.gdn_scan(q[:a], k[:a], v[:a], la[:a], b[:a], [0, a], want_o=False)
    _, S_hat = oracle.gdn_scan(q[a:], k[a:], v[a:], la[a:], b[a:], [0, kk], want_o=False)
    P = oracle.transition_product(k[a:], la[a:], b[a:], [0, kk])
    np.testing.assert_allclose(S_m, np.einsum('nhij,nhjk->nhik', P, S_a) + S_hat, atol=1e-12)
