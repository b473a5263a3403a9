"""Pins of the oracle against what the pages and the mathematics fix (CPU only).

Each test ties an oracle function to something other than the oracle itself:
hand-computed or closed-form values, exact rational arithmetic, textbook attention
from a library, or invariants. A plausible slip (a dropped 1/2, a wrong 1/sqrt(d),
a transposed operand, a wrong tie rule, an off-by-one block range) fails one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import cobs_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- exact mass, OSA

def test_exact_mass_hand_computed():
    """COBS §2.1 mass m_b = sum_r exp(q.k_r/sqrt(d)) on a case computed by hand."""
    rows = _golden_rows("exact_mass_tiny.txt")
    L, d = 4, 2
    K = np.zeros((L * len(rows), d))
    expected = []
    for j, r in enumerate(rows):
        a = [float(x) for x in r[1:5]]
        K[j * L:(j + 1) * L, 0] = np.log(a)
        K[j * L:(j + 1) * L, 1] = [0.3, -1.0, 2.0, 5.0]   # orthogonal to q: must not matter
        expected.append(float(r[5]))
    q = np.array([math.sqrt(2.0), 0.0])
    got = O.exact_log_mass(q, K, L)
    np.testing.assert_allclose(got, expected, rtol=0, atol=1e-12)
    # oracle sparse attention picks the blocks of largest mass (block 3, then the tie 0/2 -> 0)
    assert list(O.osa_top_k(q[None], K, L, len(rows), 2)) == [0, 3]


# ---------------------------------------------------------------- summaries

def test_summaries_linear_rows_closed_form():
    """Rows k_r = r + c0: mean (L-1)/2 + c0, population variance (L^2-1)/12 (COBS §2.2 kappa_1, kappa_2)."""
    L, d = 64, 8
    r = np.arange(2 * L, dtype=np.float64)
    K = r[:, None] + np.arange(d)[None, :] * 0.5
    mu, var = O.block_summaries(K, L)
    for b in range(2):
        np.testing.assert_allclose(mu[b], b * L + (L - 1) / 2 + np.arange(d) * 0.5, rtol=0, atol=1e-12)
        np.testing.assert_allclose(var[b], (L * L - 1) / 12.0, rtol=0, atol=1e-9)
    s32 = O.canonical_summaries(K.astype(np.float32), L)
    # every step is exact in float32 here, so the canonical summaries equal the closed form exactly
    assert np.array_equal(s32[:, 0], mu.astype(np.float32))
    assert np.all(s32[:, 1] == np.float32((L * L - 1) / 12.0))


def test_summaries_identical_rows_and_shift():
    rng = np.random.default_rng(0)
    L, d = 64, 16
    # bf16-valued row (as in the cache): 64 copies sum exactly in float32
    row = synth.bf16_to_f32(synth.f32_to_bf16(rng.standard_normal(d).astype(np.float32)))
    K = np.tile(row, (L, 1)).astype(np.float64)
    mu, var = O.block_summaries(K, L)
    s32 = O.canonical_summaries(K.astype(np.float32), L)
    assert np.array_equal(s32[0, 0], row) and np.all(s32[0, 1] == 0)
    np.testing.assert_allclose(mu[0], row, atol=1e-15)
    assert np.all(var[0] == 0)
    # variance is shift invariant, mean shifts
    K2 = rng.standard_normal((3 * L, d))
    c = rng.standard_normal(d) * 10
    m1, v1 = O.block_summaries(K2, L)
    m2, v2 = O.block_summaries(K2 + c, L)
    np.testing.assert_allclose(v1, v2, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(m2 - m1, np.tile(c, (3, 1)), atol=1e-12)
    # and agree with numpy's own mean/var(ddof=0)
    np.testing.assert_allclose(v1, K2.reshape(3, L, d).var(axis=1, ddof=0), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- scores

def test_identical_key_block_score_equals_exact_mass():
    """Zero spread: the cumulant series stops after kappa_1, so score = ln m_b - ln L (COBS §2.2)."""
    rng = np.random.default_rng(1)
    L, d = 64, 32
    rows = rng.standard_normal((5, d)) * 0.7
    K = np.repeat(rows, L, axis=0)
    mu, var = O.block_summaries(K, L)
    for _ in range(4):
        q = rng.standard_normal(d)
        s = O.head_scores(q, mu, var, alpha=1.0)
        np.testing.assert_allclose(s, O.exact_log_mass(q, K, L) - np.log(L), rtol=0, atol=1e-12)


def test_gaussian_keys_lognormal_closed_form():
    """Golden closed form: for Gaussian keys the second-order estimate is exact in the limit."""
    (d, qs, ms, ss, exp) = _golden_rows("lognormal_closed_form.txt")[0]
    d = int(d)
    q = np.array([float(x) for x in qs.split(",")])
    m = np.array([float(x) for x in ms.split(",")])
    s = np.array([float(x) for x in ss.split(",")])
    # the oracle's score with the population summaries (mean m, variance s^2)
    got = O.head_scores(q, m[None], (s * s)[None], alpha=1.0)[0]
    assert abs(got - float(exp)) < 1e-12
    # and the exact mass of sampled blocks converges to it, error ~ L^(-1/2)
    rng = np.random.default_rng(2)
    errs = []
    for logL in (10, 14, 18):
        L = 1 << logL
        K = m + s * rng.standard_normal((L, d))
        errs.append(abs(O.exact_log_mass(q, K, L)[0] - np.log(L) - float(exp)))
    assert errs[2] < 0.01, errs
    assert errs[2] < errs[0], errs
    # with alpha = 0 the estimate keeps a constant bias of variance/2 = 0.0925
    first = O.head_scores(q, m[None], (s * s)[None], alpha=0.0)[0]
    assert abs(first - float(exp)) > 0.09


def test_gaussian_blocks_empirical_summaries_converge():
    """Per-channel variance weighting: the score from the block's own summaries tracks ln(m_b/L)."""
    rng = np.random.default_rng(3)
    d = 8
    q = rng.standard_normal(d)
    m = rng.standard_normal(d) * 0.3
    s = np.linspace(0.1, 0.5, d)
    prev = None
    for logL in (10, 14, 18):
        L = 1 << logL
        K = m + s * rng.standard_normal((L, d))
        mu, var = O.block_summaries(K, L)
        err = abs(O.exact_log_mass(q, K, L)[0] - np.log(L) - O.head_scores(q, mu, var, 1.0)[0])
        err0 = abs(O.exact_log_mass(q, K, L)[0] - np.log(L) - O.head_scores(q, mu, var, 0.0)[0])
        assert err < err0
        prev = err
    assert prev < 2e-3


def test_alpha_zero_is_first_order_mean_pool():
    """alpha = 0 ranks blocks by the mean-pooled key against the summed group query (NSA mean-pool)."""
    rng = np.random.default_rng(4)
    L, d, G, nB = 64, 64, 4, 40
    K = rng.standard_normal((nB * L, d)) * rng.uniform(0.2, 2.0, size=(nB * L, 1))
    qs = rng.standard_normal((G, d))
    pooled = K.reshape(nB, L, d).mean(axis=1)
    ref = np.sort(np.argsort(-(pooled @ qs.sum(axis=0)), kind="stable")[:8])
    mu, var = O.block_summaries(K, L)
    assert list(O.top_k(O.group_scores(qs, mu, var, 0.0), nB, 8)) == list(ref)
    summ = O.canonical_summaries(K.astype(np.float32), L)
    a, b = O.canonical_group_query(qs.astype(np.float32))
    S = O.canonical_scores(a[None], b[None], summ, 0.0)[0]
    assert list(O.top_k(S, nB, 8)) == list(ref)


@pytest.mark.parametrize("G", [2, 4, 16])
def test_group_score_identical_key_blocks_equal_exact_group_mass(G):
    """Zero spread, several heads: every form's group score equals the exact group log-mass
    sum_h (ln m_{h,b} - ln L) (COBS §2.1 mass, §2.2 series ending at kappa_1). A group score
    that averaged, took the max, or dropped a head would miss it."""
    rng = np.random.default_rng(11 + G)
    L, d, nB = 64, 32, 6
    rows = rng.standard_normal((nB, d)) * 0.7
    K = np.repeat(rows, L, axis=0)
    qs = rng.standard_normal((G, d))
    exact = O.exact_group_score(qs, K, L)
    mu, var = O.block_summaries(K, L)
    tol = 1e-12 * G
    np.testing.assert_allclose(O.group_scores(qs, mu, var, 1.0), exact, rtol=0, atol=tol)
    np.testing.assert_allclose(O.group_scores_iso(qs, mu, var.mean(axis=1), 1.0), exact, rtol=0, atol=tol)
    m2, u, lam = O.block_eigenpairs(K, L, 2)
    np.testing.assert_allclose(O.group_scores_lowrank(qs, m2, u, lam, 1.0), exact, rtol=0, atol=1e-10 * G)
    # the same blocks ranked by the exact group mass and by the group score
    assert list(O.top_k(O.group_scores(qs, mu, var, 1.0), nB, 3)) == list(O.osa_top_k(qs, K, L, nB, 3))


def test_group_score_gaussian_blocks_converge_to_exact_group_mass():
    """Gaussian keys N(m, diag s^2), G = 4: the exact group log-mass of sampled blocks converges
    (error ~ L^-1/2) to sum_h [q_h.m/sqrt(d) + 1/2 sum_c q_{h,c}^2 s_c^2 / d] (lognormal mean per
    head, COBS §2.2), which is the group score of the population summaries; the first-order
    group score keeps the bias sum_h 1/2 sum_c q_{h,c}^2 s_c^2 / d."""
    rng = np.random.default_rng(21)
    d, G = 8, 4
    qs = rng.standard_normal((G, d)) * 0.8
    m = rng.standard_normal(d) * 0.3
    s = np.linspace(0.1, 0.45, d)
    closed = sum(q @ m / np.sqrt(d) + 0.5 * (q * q) @ (s * s) / d for q in qs)
    got = O.group_scores(qs, m[None], (s * s)[None], 1.0)[0]
    assert abs(got - closed) < 1e-12
    bias = sum(0.5 * (q * q) @ (s * s) / d for q in qs)
    assert abs(O.group_scores(qs, m[None], (s * s)[None], 0.0)[0] - closed) == pytest.approx(bias, abs=1e-12)
    errs, errs_emp = [], []
    for logL in (10, 14, 18):
        L = 1 << logL
        K = m + s * rng.standard_normal((L, d))
        exact = O.exact_group_score(qs, K, L)[0]
        errs.append(abs(exact - closed))
        mu, var = O.block_summaries(K, L)
        errs_emp.append(abs(exact - O.group_scores(qs, mu, var, 1.0)[0]))
    assert errs[2] < errs[0], errs
    assert errs[2] < 0.01 and errs_emp[2] < 5e-3, (errs, errs_emp)
    assert bias > 0.05 and errs_emp[2] < bias / 10


def test_near_tie_gap_reports_only_float_level_disagreements():
    """near_tie_gap: None when the float32 and float64 choices agree; otherwise the float64 gap
    between the swapped blocks, relative to the largest score."""
    S64 = np.array([3.0, 1.0, 2.0, 2.0 + 1e-9, 0.5])
    assert O.near_tie_gap(S64, np.array([0, 3], np.int32), 5, 2) is None
    gap = O.near_tie_gap(S64, np.array([0, 2], np.int32), 5, 2)   # float32 took 2 over 3
    assert gap == pytest.approx(1e-9 / 3.0, rel=1e-6)
    assert O.near_tie_gap(S64, np.array([0, 1], np.int32), 5, 2) == pytest.approx((2.0 + 1e-9 - 1.0) / 3.0)


def test_float32_selection_agrees_with_float64_ranking_on_the_decode_workload():
    """On seeded decode-workload units the float32 canonical choice equals the float64 top-k of
    the same definition, or differs only at a float64 gap below 1e-5 relative."""
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=8192)
    K, V = synth.kv_cache(w)
    Q, g = synth.queries_decode(w), synth.gates_decode(w)
    Pk, Pv = synth.projections(w)
    res = O.decode(w, K, V, Q, g, Pk, Pv)
    for (_, _, gap) in res["near_ties"]:
        assert gap < 1e-5


def test_group_sum_reading_internal_consistency():
    """Group score = sum of head scores = collapsed form (reading; parity unpinned by the pages)."""
    rng = np.random.default_rng(5)
    L, d, G, nB = 64, 128, 4, 10
    K = rng.standard_normal((nB * L, d))
    qs = rng.standard_normal((G, d))
    mu, var = O.block_summaries(K, L)
    collapsed = (mu @ qs.sum(0)) / np.sqrt(d) + 0.7 * 0.5 * (var @ (qs * qs).sum(0)) / d
    np.testing.assert_allclose(O.group_scores(qs, mu, var, 0.7), collapsed, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- canonical float32 arithmetic

def _dot4_exact(F, x, y):
    """The canonical channel sum: four partial chains (channels c = j mod 4, ascending, one
    rounded fma per term) combined as (s0 + s1) + (s2 + s3), every step rounded once."""
    s = [Fraction(0)] * 4
    for c in range(len(x)):
        s[c % 4] = _rn32(F(x[c]) * F(y[c]) + s[c % 4])
    return _rn32(_rn32(s[0] + s[1]) + _rn32(s[2] + s[3]))


def _rn32(x: Fraction) -> Fraction:
    """Round an exact rational to the nearest binary32 value, ties to even (normal range)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    n, rem = divmod(a, ulp)
    n = int(n)
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    return sign * n * ulp


def test_canonical_selector_matches_exact_rational_emulation():
    """Brute force: each canonical step as exact rational arithmetic rounded once to float32."""
    rng = np.random.default_rng(6)
    L, d, G, nB = 64, 32, 3, 3
    K = synth.bf16_to_f32(synth.f32_to_bf16((rng.standard_normal((nB * L, d)) * 1.3).astype(np.float32)))
    q = rng.standard_normal((G, d)).astype(np.float32)
    alpha = np.float32(0.83)
    summ = O.canonical_summaries(K, L)
    qsum, q2 = O.canonical_group_query(q)
    S = O.canonical_scores(qsum[None], q2[None], summ, float(alpha))[0]
    F = lambda v: Fraction(float(v))
    for b in range(nB):
        for c in range(d):
            s = Fraction(0)
            for r in range(L):
                s = _rn32(s + F(K[b * L + r, c]))
            mu = _rn32(s / L)
            a = Fraction(0)
            for r in range(L):
                t = _rn32(F(K[b * L + r, c]) - mu)
                a = _rn32(t * t + a)
            assert F(summ[b, 0, c]) == mu
            assert F(summ[b, 1, c]) == _rn32(a / L)
    for c in range(d):
        s, s2 = Fraction(0), Fraction(0)
        for h in range(G):
            s = _rn32(s + F(q[h, c]))
            s2 = _rn32(F(q[h, c]) * F(q[h, c]) + s2)
        assert F(qsum[c]) == s and F(q2[c]) == s2
    isd = _rn32(Fraction(1.0 / math.sqrt(d)))
    c2 = _rn32(F(alpha) / (2 * d))
    for b in range(nB):
        a = _dot4_exact(F, qsum, summ[b, 0])
        v = _dot4_exact(F, q2, summ[b, 1])
        assert F(S[b]) == _rn32(c2 * v + _rn32(a * isd)), b


def test_canonical_scores_exact_on_dyadic_inputs():
    """Dyadic inputs make every float32 step exact: canonical == float64 definition, bit for bit."""
    rng = np.random.default_rng(7)
    L, d, G, nB = 64, 64, 4, 12
    # rows = centre + balanced deviations: mean = centre exactly, deviations in {0, +-1/2, +-1}
    centre = rng.integers(-8, 9, size=(nB, 1, d)) / 4.0
    half = rng.integers(-2, 3, size=(nB, L // 2, d)) / 2.0
    dev = np.concatenate([half, -half], axis=1)
    dev = np.take_along_axis(dev, rng.permuted(np.tile(np.arange(L)[None, :, None], (nB, 1, d)), axis=1), axis=1)
    K = (centre + dev).reshape(nB * L, d)
    qs = rng.integers(-1, 2, size=(G, d)).astype(np.float64)
    mu, var = O.block_summaries(K, L)
    ref = O.group_scores(qs, mu, var, 1.0)
    summ = O.canonical_summaries(K.astype(np.float32), L)
    a, b = O.canonical_group_query(qs.astype(np.float32))
    S = O.canonical_scores(a[None], b[None], summ, 1.0)[0]
    assert np.array_equal(S.astype(np.float64), ref)


# ---------------------------------------------------------------- top-k

def test_topk_tie_rule_padding_and_order():
    S = np.array([1.0, 3.0, 3.0, -0.0, 0.0, 3.0, 2.0], np.float32)
    assert list(O.top_k(S, 7, 2)) == [1, 2]            # equal scores: lower index wins
    assert list(O.top_k(S, 7, 4)) == [1, 2, 5, 6]        # returned ascending
    assert list(O.top_k(S, 5, 4)) == [0, 1, 2, 3]        # -0 == +0, lower index wins
    assert list(O.top_k(S, 3, 5)) == [0, 1, 2, -1, -1]   # fewer candidates than k: -1 padding
    assert list(O.top_k(S, 0, 2)) == [-1, -1]
    # duplicated summaries: identical scores, the lower block index is kept
    L, d = 64, 16
    rng = np.random.default_rng(8)
    blk = rng.standard_normal((L, d))
    K = np.concatenate([rng.standard_normal((L, d)) * 0.1, blk, blk, rng.standard_normal((L, d)) * 0.1])
    summ = O.canonical_summaries(K.astype(np.float32), L)
    q = rng.standard_normal((2, d)).astype(np.float32)
    a, b = O.canonical_group_query(q)
    S = O.canonical_scores(a[None], b[None], summ, 1.0)[0]
    assert S[1] == S[2]
    sel = O.top_k(S, 4, 1)
    assert sel[0] in (0, 1, 3) and sel[0] != 2


def test_candidates_are_complete_blocks_before_position():
    assert O.n_candidates(62, 64) == 0
    assert O.n_candidates(63, 64) == 1
    assert O.n_candidates(64, 64) == 1
    assert O.n_candidates(32767, 64) == 512


# ---------------------------------------------------------------- branches

def _sdpa(q, K, V):
    """Textbook attention from torch (float64, CPU)."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q[None]), t(K), t(V))[0, 0, 0].numpy()


def test_branches_reduce_to_dense_attention():
    rng = np.random.default_rng(9)
    L, d, T = 64, 32, 512
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    q = rng.standard_normal((1, d)) * 2
    dense = _sdpa(q[0], K, V)
    nB = T // L
    Kc = O.compressed_tokens(K, None, 1, 1, "f32")
    Vc = O.compressed_tokens(V, None, 1, 1, "f32")
    all_blocks = np.arange(nB)
    t = T - 1
    # top-k = all blocks: the selected branch is dense attention
    o = O.position_output(q, [[0, 1, 0]], K, V, Kc, Vc, all_blocks, t, L, 128, 1, 1)
    np.testing.assert_allclose(o[0], dense, rtol=0, atol=1e-12)
    # window covering the whole context: dense
    o = O.position_output(q, [[0, 0, 1]], K, V, Kc, Vc, all_blocks[:1], t, L, T + 5, 1, 1)
    np.testing.assert_allclose(o[0], dense, rtol=0, atol=1e-12)
    # compression with block = stride = 1 and identity map: dense
    o = O.position_output(q, [[1, 0, 0]], K, V, Kc, Vc, all_blocks[:1], t, L, 128, 1, 1)
    np.testing.assert_allclose(o[0], dense, rtol=0, atol=1e-12)
    # gates mix linearly
    o1 = O.position_output(q, [[0.2, 0.3, 0.5]], K, V, Kc, Vc, all_blocks, t, L, T, 1, 1)
    np.testing.assert_allclose(o1[0], dense, rtol=0, atol=1e-12)


def test_window_and_selection_token_sets():
    slc, win, cmp_ = O.branch_tokens(200, np.array([0, 2, -1]), 64, 128, 32, 16, 100)
    assert list(slc) == list(range(0, 64)) + list(range(128, 192))
    assert list(win) == list(range(73, 201))
    # compressed token i covers rows 16i .. 16i+31 and is visible when 16i+31 <= t
    assert list(cmp_) == list(range(0, 11))          # 16*10+31 = 191 <= 200 < 16*11+31
    slc, win, cmp_ = O.branch_tokens(20, np.array([-1]), 64, 128, 32, 16, 100)
    assert len(slc) == 0 and list(win) == list(range(0, 21)) and len(cmp_) == 0


def test_attention_shift_invariance_and_empty_branch():
    rng = np.random.default_rng(10)
    K = rng.standard_normal((50, 16))
    V = rng.standard_normal((50, 16))
    q = rng.standard_normal(16)
    o1 = O.attend(q, K, V)
    o2 = O.attend(q, K + rng.standard_normal(16), V)     # q.k shifts by a constant
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    assert np.all(O.attend(q, K[:0], V[:0]) == 0)


def test_compressed_tokens_mean_pool_closed_form():
    T, d = 256, 4
    X = np.arange(T, dtype=np.float64)[:, None] * np.ones((1, d))
    C = O.compressed_tokens(X, None, 32, 16, "f32")
    assert C.shape == ((T - 32) // 16 + 1, d)
    np.testing.assert_allclose(C[:, 0], 16 * np.arange(C.shape[0]) + 15.5, atol=0)
    P = np.diag([1.0, 2.0, -1.0, 0.5])
    Cp = O.compressed_tokens(X, P, 32, 16, "f32")
    np.testing.assert_allclose(Cp, C * np.array([1.0, 2.0, -1.0, 0.5]), atol=0)


def test_round_bf16_matches_bit_rounding():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-3, 4, 100000)).astype(np.float32)
    # halfway cases: ties to even
    x[:4] = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 1.0 + 2 ** -9], np.float32)
    ref = synth.bf16_to_f32(synth.f32_to_bf16(x)).astype(np.float64)
    assert np.array_equal(O.round_bf16(x.astype(np.float64)), ref)
    assert list(ref[:4]) == [1.0, 1.015625, -1.0, 1.0]


# ---------------------------------------------------------------- whole path

def test_decode_equals_prefill_last_row():
    w = synth.WORKLOADS["tiny"]
    K, V = synth.kv_cache(w)
    Q = synth.queries_decode(w)
    g = synth.gates_decode(w)
    dec = O.decode(w, K, V, Q, g, None, None)
    Qp = synth.queries_prefill(w, positions=[w.T - 1])
    gp = synth.gates_prefill(w, positions=[w.T - 1])
    assert np.array_equal(Qp[0, 0], Q[0])
    Op, idxp = O.prefill_positions(w, K, V, Qp[0], gp[0], None, None, [w.T - 1])
    assert np.array_equal(idxp[0], dec["idx"][0])
    np.testing.assert_allclose(Op[0], dec["O"][0], rtol=0, atol=1e-13)


def test_needle_recall_second_order_beats_first_order():
    """Method claim (COBS §2.2/§2.3): the variance term finds high-spread blocks the mean misses."""
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=8192)
    K, V = synth.kv_cache(w)
    Q = synth.queries_decode(w)
    r1, r0 = [], []
    for h in range(w.Hkv):
        Kf = synth.to_f64(K[0, h], w.dtype)
        qs = synth.to_f64(Q[0, h * w.G:(h + 1) * w.G], w.dtype)
        summ = O.canonical_summaries(Kf.astype(np.float32), w.block)
        a, b = O.canonical_group_query(qs.astype(np.float32))
        ref = O.osa_top_k(qs, Kf, w.block, w.nB, w.topk)
        s1 = O.top_k(O.canonical_scores(a[None], b[None], summ, 1.0)[0], w.nB, w.topk)
        s0 = O.top_k(O.canonical_scores(a[None], b[None], summ, 0.0)[0], w.nB, w.topk)
        r1.append(O.recall(s1, ref))
        r0.append(O.recall(s0, ref))
    assert np.mean(r1) > np.mean(r0), (r1, r0)


def test_projection_orientation():
    """Compressed token = P @ pooled (row j of the output is P[j] . m): constant rows e_0 give P[:, 0]."""
    rng = np.random.default_rng(12)
    d = 8
    P = rng.standard_normal((d, d))
    X = np.zeros((64, d))
    X[:, 0] = 1.0
    C = O.compressed_tokens(X, P, 32, 16, "f32")
    np.testing.assert_allclose(C[0], P[:, 0], rtol=0, atol=1e-15)


def test_gate_order_isolates_each_branch():
    """Gates (cmp, slc, win): each unit gate picks exactly its branch, checked against library attention."""
    rng = np.random.default_rng(13)
    L, d, T, W = 64, 16, 1024, 96
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    P = rng.standard_normal((d, d)) / np.sqrt(d)
    Kc = O.compressed_tokens(K, P, 32, 16, "f32")
    Vc = O.compressed_tokens(V, P.T, 32, 16, "f32")
    q = rng.standard_normal((1, d)) * 2
    idx = np.array([1, 4, 9])
    t = 700
    sel_tok = np.concatenate([np.arange(b * L, (b + 1) * L) for b in idx])
    n_vis = (t - 32 + 1) // 16 + 1
    expect = {
        0: _sdpa(q[0], Kc[:n_vis], Vc[:n_vis]),
        1: _sdpa(q[0], K[sel_tok], V[sel_tok]),
        2: _sdpa(q[0], K[t - W + 1:t + 1], V[t - W + 1:t + 1]),
    }
    for j in range(3):
        g = np.zeros((1, 3))
        g[0, j] = 1.0
        o = O.position_output(q, g, K, V, Kc, Vc, idx, t, L, W, 32, 16)
        np.testing.assert_allclose(o[0], expect[j], rtol=0, atol=1e-12)
    assert not np.allclose(expect[0], expect[1]) and not np.allclose(expect[1], expect[2])


# ---------------------------------------------------------------- isotropic scalar variant

def test_iso_summaries_match_library_variance():
    """sigma2_b = mean over channels of numpy's population variance (ddof=0) of the block."""
    rng = np.random.default_rng(21)
    L, d, nB = 64, 64, 6
    K = synth.bf16_to_f32(synth.f32_to_bf16((rng.standard_normal((nB * L, d)) *
                                              rng.uniform(0.2, 2.0, (nB * L, 1))).astype(np.float32)))
    s = O.canonical_summaries_iso(K, L)
    blocks = K.astype(np.float64).reshape(nB, L, d)
    assert np.allclose(s[:, :d], blocks.mean(axis=1), rtol=0, atol=1e-6)
    assert np.allclose(s[:, d], np.var(blocks, axis=1, ddof=0).mean(axis=1), rtol=1e-5, atol=0)


def test_iso_score_equals_diagonal_score_for_equal_channel_variances():
    """When every channel of a block has the same variance, Sigma_b = sigma2 I and the two
    second-order terms agree: sigma2 |q|^2 = sum_c q_c^2 sigma2 (float64 definitions)."""
    rng = np.random.default_rng(22)
    L, d, nB, G = 64, 32, 5, 3
    centre = rng.standard_normal((nB, 1, d))
    amp = rng.uniform(0.3, 2.0, size=(nB, 1, 1))
    signs = np.where(rng.permuted(np.tile((np.arange(L) % 2)[None, :, None], (nB, 1, d)), axis=1) == 0, 1.0, -1.0)
    K = (centre + amp * signs).reshape(nB * L, d)          # every channel: variance amp^2 exactly
    mu, var = O.block_summaries(K, L)
    assert np.allclose(var, np.repeat(amp[:, 0, :] ** 2, d, axis=1))
    qs = rng.standard_normal((G, d))
    iso = O.group_scores_iso(qs, mu, var.mean(axis=1), 1.0)
    diag = O.group_scores(qs, mu, var, 1.0)
    assert np.allclose(iso, diag, rtol=0, atol=1e-12)
    # and with unequal channel variances they differ
    K2 = K * np.linspace(0.5, 1.5, d)
    mu2, var2 = O.block_summaries(K2, L)
    assert not np.allclose(O.group_scores_iso(qs, mu2, var2.mean(axis=1), 1.0), O.group_scores(qs, mu2, var2, 1.0))


def test_iso_score_exact_for_isotropic_gaussian_keys():
    """Closed form: keys N(m, s^2 I) give ln E exp(q.k/sqrt(d)) = q.m/sqrt(d) + s^2 |q|^2 / (2 d),
    which the isotropic score reproduces with the population summaries, and sampled blocks
    converge to it."""
    rng = np.random.default_rng(23)
    d = 16
    q = rng.standard_normal(d)
    m = rng.standard_normal(d) * 0.4
    s = 0.45
    exact = q @ m / math.sqrt(d) + s * s * (q @ q) / (2 * d)
    assert abs(O.head_scores_iso(q, m[None], np.array([s * s]), 1.0)[0] - exact) < 1e-12
    errs = []
    for logL in (10, 14, 18):
        L = 1 << logL
        K = m + s * rng.standard_normal((L, d))
        errs.append(abs(O.exact_log_mass(q, K, L)[0] - math.log(L) - exact))
    assert errs[-1] < 0.01 and errs[-1] < errs[0], errs


def test_iso_alpha_zero_equals_first_order():
    """alpha = 0: the isotropic and the per-channel selectors both reduce to mean-pool ranking."""
    rng = np.random.default_rng(24)
    L, d, G, nB = 64, 64, 4, 40
    K = (rng.standard_normal((nB * L, d)) * rng.uniform(0.2, 2.0, size=(nB * L, 1))).astype(np.float32)
    qs = rng.standard_normal((G, d)).astype(np.float32)
    a, b = O.canonical_group_query(qs)
    S_iso = O.canonical_scores_iso(a[None], b[None], O.canonical_summaries_iso(K, L), 0.0)[0]
    S_diag = O.canonical_scores(a[None], b[None], O.canonical_summaries(K, L), 0.0)[0]
    assert np.array_equal(S_iso, S_diag)
    pooled = K.astype(np.float64).reshape(nB, L, d).mean(axis=1)
    ref = np.sort(np.argsort(-(pooled @ qs.astype(np.float64).sum(axis=0)), kind="stable")[:8])
    assert list(O.top_k(S_iso, nB, 8)) == list(ref)


def test_iso_canonical_matches_exact_rational_emulation():
    """Brute force: the isotropic canonical steps as exact rationals rounded once to float32."""
    rng = np.random.default_rng(25)
    L, d, G, nB = 64, 16, 3, 3
    K = synth.bf16_to_f32(synth.f32_to_bf16((rng.standard_normal((nB * L, d)) * 1.1).astype(np.float32)))
    q = rng.standard_normal((G, d)).astype(np.float32)
    alpha = np.float32(0.77)
    summ = O.canonical_summaries(K, L)
    iso = O.canonical_summaries_iso(K, L)
    qsum, q2 = O.canonical_group_query(q)
    S = O.canonical_scores_iso(qsum[None], q2[None], iso, float(alpha))[0]
    F = lambda v: Fraction(float(v))
    for b in range(nB):
        acc = Fraction(0)
        for c in range(d):
            assert F(iso[b, c]) == F(summ[b, 0, c])
            acc = _rn32(acc + F(summ[b, 1, c]))
        assert F(iso[b, d]) == _rn32(acc / d)
    q2tot = Fraction(0)
    for c in range(d):
        q2tot = _rn32(q2tot + F(q2[c]))
    isd = _rn32(Fraction(1.0 / math.sqrt(d)))
    c2 = _rn32(F(alpha) / (2 * d))
    for b in range(nB):
        a = _dot4_exact(F, qsum, iso[b, :d])
        v = _rn32(q2tot * F(iso[b, d]))
        assert F(S[b]) == _rn32(c2 * v + _rn32(a * isd)), b


# ---------------------------------------------------------------- low-rank covariance variant

def _aniso_blocks(rng, nB, L, d, spectrum, noise):
    U, _ = np.linalg.qr(rng.standard_normal((d, len(spectrum))))
    mu = rng.standard_normal((nB, 1, d)) * 0.5
    Z = rng.standard_normal((nB, L, len(spectrum))) * np.asarray(spectrum)
    return (mu + Z @ U.T + noise * rng.standard_normal((nB, L, d))).reshape(nB * L, d)


def test_lowrank_solver_matches_library_eigh():
    """The fixed float32 subspace iteration reaches numpy's eigh on well-separated spectra."""
    rng = np.random.default_rng(31)
    L, d, R, nB = 64, 128, 4, 8
    K = _aniso_blocks(rng, nB, L, d, [3.0, 2.2, 1.6, 1.2, 0.5, 0.3], 0.05).astype(np.float32)
    mu32, u32, lam32 = O.canonical_summaries_lowrank(K, L, R)
    mu, u, lam = O.block_eigenpairs(K.astype(np.float64), L, R)
    assert np.allclose(mu32, mu, atol=1e-6)
    assert np.abs(lam32 / lam - 1).max() < 1e-4
    cos = np.abs(np.einsum("brd,brd->br", u32.astype(np.float64), u))
    assert cos.min() > 0.9999
    assert np.all(np.diff(lam32, axis=1) <= 0)   # descending


def test_lowrank_score_is_the_covariance_quadratic_form_for_low_rank_blocks():
    """Blocks whose keys span an R-dimensional affine subspace: sum_j lam_j (q.u_j)^2 = q^T Sigma q,
    so the low-rank score equals the full second-order score (float64 definitions)."""
    rng = np.random.default_rng(32)
    L, d, R, nB, G = 64, 32, 3, 5, 4
    K = _aniso_blocks(rng, nB, L, d, [2.0, 1.0, 0.5], 0.0)
    mu, u, lam = O.block_eigenpairs(K, L, R)
    qs = rng.standard_normal((G, d))
    full = np.zeros(nB)
    for b in range(nB):
        Y = K[b * L:(b + 1) * L] - mu[b]
        S = Y.T @ Y / L
        full[b] = sum(q @ mu[b] / math.sqrt(d) + 0.5 * (q @ S @ q) / d for q in qs)
    assert np.allclose(O.group_scores_lowrank(qs, mu, u, lam, 1.0), full, rtol=0, atol=1e-10)
    # a rank-R truncation of a rank-(R+2) block loses the smallest directions
    K2 = _aniso_blocks(rng, nB, L, d, [2.0, 1.0, 0.5, 0.4, 0.3], 0.0)
    mu2, u2, lam2 = O.block_eigenpairs(K2, L, R)
    mu5, u5, lam5 = O.block_eigenpairs(K2, L, R + 2)
    assert np.all(O.group_scores_lowrank(qs, mu2, u2, lam2, 1.0) <= O.group_scores_lowrank(qs, mu5, u5, lam5, 1.0) + 1e-12)


def test_lowrank_axis_aligned_block_equals_per_channel_score():
    """Variance in R channels only (a diagonal covariance): the eigenvectors are those axes and
    the low-rank score equals the per-channel-variance score."""
    rng = np.random.default_rng(33)
    L, d, R, nB, G = 64, 16, 3, 4, 3
    # deviations along R channels by mutually orthogonal, zero-mean +-1 patterns (rows of a
    # Sylvester-Hadamard matrix other than the first): the block covariance is exactly diagonal
    H = np.array([[1.0]])
    while H.shape[0] < L:
        H = np.block([[H, H], [H, -H]])
    K = np.repeat(rng.standard_normal((nB, 1, d)), L, axis=1)
    for b in range(nB):
        chans = rng.choice(d, size=R, replace=False)
        amps = np.sort(rng.uniform(0.5, 2.0, size=R))[::-1] + np.arange(R)[::-1] * 0.3  # distinct
        for i, c in enumerate(chans):
            K[b][:, c] += amps[i] * H[1 + 3 * i]
    K = K.reshape(nB * L, d)
    mu, var = O.block_summaries(K, L)
    mu2, u, lam = O.block_eigenpairs(K, L, R)
    qs = rng.standard_normal((G, d))
    assert np.allclose(O.group_scores_lowrank(qs, mu2, u, lam, 1.0), O.group_scores(qs, mu, var, 1.0), atol=1e-10)


def test_lowrank_alpha_zero_is_first_order():
    rng = np.random.default_rng(34)
    L, d, R, nB, G = 64, 64, 4, 24, 4
    K = _aniso_blocks(rng, nB, L, d, [2.0, 1.5, 1.0, 0.7, 0.4], 0.1).astype(np.float32)
    q = rng.standard_normal((G, d)).astype(np.float32)
    S = O.canonical_scores_lowrank(q, O.canonical_summaries_lowrank(K, L, R), 0.0)
    pooled = K.astype(np.float64).reshape(nB, L, d).mean(axis=1)
    ref = np.sort(np.argsort(-(pooled @ q.astype(np.float64).sum(axis=0)), kind="stable")[:8])
    assert list(O.top_k(S, nB, 8)) == list(ref)


def test_lowrank_scores_match_exact_rational_emulation():
    """Brute force: the low-rank score's float32 steps as exact rationals rounded once each."""
    rng = np.random.default_rng(35)
    L, d, R, nB, G = 64, 16, 2, 3, 3
    K = _aniso_blocks(rng, nB, L, d, [2.0, 1.0, 0.4], 0.05).astype(np.float32)
    summ = O.canonical_summaries_lowrank(K, L, R)
    mu, u, lam = summ
    q = rng.standard_normal((G, d)).astype(np.float32)
    alpha = np.float32(0.9)
    S = O.canonical_scores_lowrank(q, summ, float(alpha))
    qsum, _ = O.canonical_group_query(q)
    F = lambda v: Fraction(float(v))
    isd = _rn32(Fraction(1.0 / math.sqrt(d)))
    c2 = _rn32(F(alpha) / (2 * d))
    for b in range(nB):
        a = _dot4_exact(F, qsum, mu[b])
        v = Fraction(0)
        for j in range(R):
            e = Fraction(0)
            for h in range(G):
                pj = _dot4_exact(F, q[h], u[b, j])
                e = _rn32(pj * pj + e)
            v = _rn32(F(lam[b, j]) * e + v)
        assert F(S[b]) == _rn32(c2 * v + _rn32(a * isd)), b


# ---------------------------------------------------------------- FP4 (E2M1) low-rank variant

_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_rounding_is_nearest_with_ties_to_even_and_saturation():
    """Brute force over a fine grid (and every tie point): the code's magnitude is the nearest
    of the eight E2M1 magnitudes, ties go to the even index, |x| > 6 saturates, the sign is bit 3."""
    grid = list(np.linspace(-8, 8, 3201)) + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -1.75, -5.0]
    for x in grid:
        code = O.e2m1_code(x)
        a = abs(x)
        d = [abs(a - m) for m in _E2M1]
        best = min(range(8), key=lambda i: (d[i], i % 2))
        if a > 6:
            best = 7
        assert code & 7 == best, (x, code)
        assert (code >> 3) == (1 if (x < 0 and best > 0) else 0), (x, code)


def test_fp4_mean_is_bf16_round_to_nearest_even():
    rng = np.random.default_rng(41)
    K = (rng.standard_normal((4 * 64, 32)) * 3).astype(np.float32)
    fp4 = O.canonical_summaries_lowrank_fp4(K, 64, 2)
    mu = O.canonical_summaries(K, 64)[:, 0, :]
    ref = torch.from_numpy(mu).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(fp4[0], ref)


def test_fp4_vectors_within_the_e2m1_grid_bound():
    """Dequantized eigenvectors: u'_c = code * s with s = max|u| / 6; the error is at most half
    the E2M1 gap at that magnitude (at most s), and the largest entry is exact up to rounding of s."""
    rng = np.random.default_rng(42)
    L, d, R, nB = 64, 128, 4, 6
    K = _aniso_blocks(rng, nB, L, d, [3.0, 2.0, 1.4, 1.0, 0.5], 0.05).astype(np.float32)
    mu, u, lam = O.canonical_summaries_lowrank(K, L, R)
    mu_q, codes, scales, lam_q, u_q = O.canonical_summaries_lowrank_fp4(K, L, R)
    assert np.array_equal(lam_q, lam)
    s = scales[..., None].astype(np.float64)
    err = np.abs(u_q.astype(np.float64) - u.astype(np.float64))
    half_gap = np.where(np.abs(u) / s > 4, 1.0, np.where(np.abs(u) / s > 2, 0.5, 0.25))
    assert np.all(err <= half_gap * s * (1 + 1e-6) + 1e-12)
    assert np.allclose(scales, np.abs(u).max(axis=-1) / 6, rtol=1e-7)


def test_fp4_selection_tracks_float32_low_rank_selection():
    """On anisotropic blocks the FP4 summaries select nearly the same blocks as float32 ones."""
    rng = np.random.default_rng(43)
    L, d, R, nB, G, k = 64, 128, 4, 96, 4, 16
    K = _aniso_blocks(rng, nB, L, d, [3.0, 2.0, 1.4, 1.0, 0.6, 0.4], 0.05).astype(np.float32)
    K += (rng.standard_normal((nB, 1, d)) * rng.uniform(0.2, 1.5, (nB, 1, 1))).repeat(L, axis=1).reshape(nB * L, d).astype(np.float32)
    q = rng.standard_normal((G, d)).astype(np.float32)
    s32 = O.canonical_scores_lowrank(q, O.canonical_summaries_lowrank(K, L, R), 1.0)
    s4 = O.canonical_scores_lowrank(q, O.canonical_summaries_lowrank_fp4(K, L, R).dequantized(), 1.0)
    a, b = set(O.top_k(s32, nB, k).tolist()), set(O.top_k(s4, nB, k).tolist())
    assert len(a & b) >= 13


# ---------------------------------------------------------------- query-subspace variant

def _orthonormal(rng, d, s):
    Pm, _ = np.linalg.qr(rng.standard_normal((d, s)))
    return Pm


def test_subspace_with_the_identity_basis_is_the_low_rank_selector():
    """P = I (s = d): every projection is exact, so the subspace scores equal the low-rank scores
    bit for bit in float32."""
    rng = np.random.default_rng(51)
    L, d, R, nB, G = 64, 32, 3, 10, 4
    K = _aniso_blocks(rng, nB, L, d, [2.0, 1.2, 0.7, 0.4], 0.05).astype(np.float32)
    q = rng.standard_normal((G, d)).astype(np.float32)
    I = np.eye(d, dtype=np.float32)
    S_sub = O.canonical_scores_subspace(q, O.canonical_summaries_subspace(K, L, R, I), 1.0)
    S_lr = O.canonical_scores_lowrank(q, O.canonical_summaries_lowrank(K, L, R), 1.0)
    assert np.array_equal(S_sub, S_lr)


def test_subspace_score_is_exact_for_queries_in_the_subspace():
    """Queries in span(P): (P^T q).(P^T u) = q^T P P^T u = q.u, so the float64 subspace score equals
    the low-rank score; queries outside it lose their out-of-subspace part."""
    rng = np.random.default_rng(52)
    L, d, R, nB, G, s = 64, 32, 3, 6, 3, 12
    K = _aniso_blocks(rng, nB, L, d, [2.0, 1.2, 0.7, 0.4], 0.05)
    mu, u, lam = O.block_eigenpairs(K, L, R)
    P = _orthonormal(rng, d, s)
    qs = (P @ rng.standard_normal((s, G))).T
    assert np.allclose(O.group_scores_subspace(qs, mu, u, lam, P, 1.0), O.group_scores_lowrank(qs, mu, u, lam, 1.0),
                       atol=1e-10)
    q_out = rng.standard_normal((G, d))
    assert not np.allclose(O.group_scores_subspace(q_out, mu, u, lam, P, 1.0),
                           O.group_scores_lowrank(q_out, mu, u, lam, 1.0))


def test_subspace_canonical_matches_exact_rational_emulation():
    rng = np.random.default_rng(53)
    L, d, R, nB, G, s = 64, 16, 2, 3, 2, 8
    K = _aniso_blocks(rng, nB, L, d, [2.0, 1.0, 0.4], 0.05).astype(np.float32)
    P = _orthonormal(rng, d, s).astype(np.float32)
    summ = O.canonical_summaries_subspace(K, L, R, P)
    mu, ut, lam, _ = summ
    _, u, _ = O.canonical_summaries_lowrank(K, L, R)
    q = rng.standard_normal((G, d)).astype(np.float32)
    S = O.canonical_scores_subspace(q, summ, 0.8)
    F = lambda v: Fraction(float(v))
    for b in range(nB):
        for j in range(R):
            for i in range(s):
                assert F(ut[b, j, i]) == _dot4_exact(F, P[:, i], u[b, j])
    qsum, _ = O.canonical_group_query(q)
    qt = [[_dot4_exact(F, P[:, i], q[h]) for i in range(s)] for h in range(G)]
    isd = _rn32(Fraction(1.0 / math.sqrt(d)))
    c2 = _rn32(F(np.float32(0.8)) / (2 * d))
    for b in range(nB):
        a = _dot4_exact(F, qsum, mu[b])
        v = Fraction(0)
        for j in range(R):
            e = Fraction(0)
            for h in range(G):
                pj = _dot4_exact(lambda x: x, qt[h], [F(x) for x in ut[b, j]])
                e = _rn32(pj * pj + e)
            v = _rn32(F(lam[b, j]) * e + v)
        assert F(S[b]) == _rn32(c2 * v + _rn32(a * isd)), b


def test_subspace_decode_with_identity_basis_is_low_rank_decode():
    """The oracle's decode driver: with P = I the query-subspace selection and output are the
    low-rank ones."""
    import synth
    w = synth.WORKLOADS["tiny"]
    K, V = synth.kv_cache(w)
    Q, g = synth.queries_decode(w), synth.gates_decode(w)
    Pk, Pv = synth.projections(w)
    a = O.decode(w, K, V, Q, g, Pk, Pv, variance="lowrank", rank=4)
    b = O.decode(w, K, V, Q, g, Pk, Pv, variance="subspace", rank=4, basis=np.eye(w.d, dtype=np.float32))
    assert np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["O"], b["O"])


# ---------------------------------------------------------------- query subspace with FP4 coordinates

def test_subspace_fp4_with_the_identity_basis_is_the_fp4_low_rank_form():
    """P = I (s = d): the projected coordinates are the eigenvectors exactly, so every stored field
    (bf16 mean, codes, scales, eigenvalues, dequantized vectors) and every score equal the FP4
    low-rank form's, bit for bit."""
    rng = np.random.default_rng(61)
    L, d, R, nB, G = 64, 32, 3, 12, 4
    K = _aniso_blocks(rng, nB, L, d, [2.0, 1.2, 0.7, 0.4], 0.05).astype(np.float32)
    I = np.eye(d, dtype=np.float32)
    sub = O.canonical_summaries_subspace_fp4(K, L, R, I)
    lr = O.canonical_summaries_lowrank_fp4(K, L, R)
    for x, y in zip(sub[:5], lr):
        assert np.array_equal(x, y)
    q = rng.standard_normal((G, d)).astype(np.float32)
    assert np.array_equal(O.canonical_scores_subspace(q, sub.dequantized(), 1.0),
                          O.canonical_scores_lowrank(q, lr.dequantized(), 1.0))


def test_fp4_vectors_are_exact_on_the_e2m1_grid():
    """Rows whose entries are E2M1 magnitudes times a power of two whose largest magnitude is 6:
    the scale is that power of two exactly and every entry round-trips exactly, with the code of
    its magnitude index and sign (worked by hand from the E2M1 table 0, .5, 1, 1.5, 2, 3, 4, 6)."""
    x = np.array([[6.0, -3.0, 0.5, 0.0, 1.5, -6.0, 4.0, -0.5],
                  [0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0]], np.float32)
    x[0] *= 0.125
    codes, scales, xq = O.fp4_vectors(x)
    assert scales.tolist() == [0.125, 0.0]
    assert codes[0].tolist() == [7, 8 | 5, 1, 0, 3, 8 | 7, 6, 8 | 1]
    assert codes[1].tolist() == [0] * 8
    assert np.array_equal(xq, x)


def test_subspace_fp4_coordinates_within_the_e2m1_grid_bound():
    """The dequantized subspace coordinates differ from the float32 ones by at most half the E2M1
    gap at their magnitude (0.25, 0.5 or 1 times the scale); the scale is max |u~| / 6; the mean is
    the bf16 rounding of the float32 mean (8 significant bits: relative error at most half an ulp,
    2^-8); eigenvalues unchanged."""
    rng = np.random.default_rng(62)
    L, d, R, nB, s = 64, 128, 4, 8, 84
    K = _aniso_blocks(rng, nB, L, d, [3.0, 2.0, 1.4, 1.0, 0.5], 0.05).astype(np.float32)
    P = _orthonormal(rng, d, s).astype(np.float32)
    mu, ut, lam, _ = O.canonical_summaries_subspace(K, L, R, P)
    mu_q, codes, scales, lam_q, ut_q, _ = O.canonical_summaries_subspace_fp4(K, L, R, P)
    assert np.array_equal(lam_q, lam)
    assert codes.shape == (nB, R, s) and codes.max() <= 15
    sc = scales[..., None].astype(np.float64)
    err = np.abs(ut_q.astype(np.float64) - ut.astype(np.float64))
    half_gap = np.where(np.abs(ut) / sc > 4, 1.0, np.where(np.abs(ut) / sc > 2, 0.5, 0.25))
    assert np.all(err <= half_gap * sc * (1 + 1e-6) + 1e-12)
    assert np.allclose(scales, np.abs(ut).max(axis=-1) / 6, rtol=1e-7)
    rel = np.abs(mu_q.astype(np.float64) - mu) / np.maximum(np.abs(mu.astype(np.float64)), 1e-30)
    assert np.all(rel <= 2.0 ** -8)


def test_subspace_fp4_canonical_scores_match_float64_of_the_stored_form():
    """The float32 canonical scores of the stored (dequantized) form agree with the float64 score of
    the same stored numbers to float32 rounding (a relative bound on the summed terms)."""
    rng = np.random.default_rng(63)
    L, d, R, nB, G, s = 64, 128, 4, 40, 4, 84
    K = _aniso_blocks(rng, nB, L, d, [3.0, 2.0, 1.4, 1.0, 0.5], 0.05).astype(np.float32)
    P = _orthonormal(rng, d, s).astype(np.float32)
    summ = O.canonical_summaries_subspace_fp4(K, L, R, P)
    q = rng.standard_normal((G, d)).astype(np.float32)
    S32 = O.canonical_scores_subspace(q, summ.dequantized(), 1.0).astype(np.float64)
    mu_q, _, _, lam, ut_q, _ = summ
    S64 = O.group_scores_subspace_coords(q.astype(np.float64), mu_q.astype(np.float64), ut_q.astype(np.float64),
                                         lam.astype(np.float64), P.astype(np.float64), 1.0)
    # magnitude of the summed terms: |q||mu| / sqrt(d) per head + the covariance term
    scale = np.abs(S64) + np.linalg.norm(q, axis=1).sum() * np.linalg.norm(mu_q, axis=1) / np.sqrt(d) + 1.0
    assert np.all(np.abs(S32 - S64) <= 64 * 2.0 ** -24 * scale)


def test_subspace_fp4_selection_tracks_the_float32_subspace_selection():
    """On anisotropic blocks with queries in the subspace, the FP4 coordinates select nearly the same
    blocks as the float32 subspace coordinates."""
    rng = np.random.default_rng(64)
    L, d, R, nB, G, k, s = 64, 128, 4, 96, 4, 16, 84
    K = _aniso_blocks(rng, nB, L, d, [3.0, 2.0, 1.4, 1.0, 0.6, 0.4], 0.05).astype(np.float32)
    K += (rng.standard_normal((nB, 1, d)) * rng.uniform(0.2, 1.5, (nB, 1, 1))).repeat(L, axis=1).reshape(nB * L, d).astype(np.float32)
    P = _orthonormal(rng, d, s).astype(np.float32)
    q = (P @ rng.standard_normal((s, G))).T.astype(np.float32)
    s32 = O.canonical_scores_subspace(q, O.canonical_summaries_subspace(K, L, R, P), 1.0)
    s4 = O.canonical_scores_subspace(q, O.canonical_summaries_subspace_fp4(K, L, R, P).dequantized(), 1.0)
    a, b = set(O.top_k(s32, nB, k).tolist()), set(O.top_k(s4, nB, k).tolist())
    assert len(a & b) >= 13


# ---------------------------------------------------------------- query-subspace basis from queries

def test_query_basis_recovers_an_exactly_diagonal_second_moment():
    """Rows +-c_k u_k of an orthonormal U: M = (1/n) sum_k 2 c_k^2 u_k u_k^T exactly, so the basis is
    the u_k of the s largest c_k (each with its largest-magnitude entry made positive) and the
    eigenvalues are 2 c_k^2 / n."""
    rng = np.random.default_rng(71)
    d, s = 16, 5
    U, _ = np.linalg.qr(rng.standard_normal((d, d)))
    c = np.linspace(3.0, 0.5, d)
    rows = np.concatenate([c[:, None] * U.T, -c[:, None] * U.T])   # [2d, d]
    rows = rows[rng.permutation(2 * d)]
    P, lam = O.query_basis(rows, s)
    n = 2 * d
    assert np.allclose(lam, 2 * c[:s] ** 2 / n, rtol=1e-12)
    for k in range(s):
        u = U[:, k] * np.sign(U[np.argmax(np.abs(U[:, k])), k])
        assert np.allclose(P[:, k], u, atol=1e-10), k


def test_query_basis_two_dimensional_closed_form():
    """d = 2: the leading eigenvalue of [[a, b], [b, c]] is (a + c)/2 + sqrt(((a - c)/2)^2 + b^2) and
    its eigenvector is at angle atan2(2b, a - c)/2."""
    Q = np.array([[1.0, 2.0], [3.0, -1.0], [0.5, 0.25], [-2.0, 1.5]])
    a, b, c = (Q[:, 0] ** 2).mean(), (Q[:, 0] * Q[:, 1]).mean(), (Q[:, 1] ** 2).mean()
    P, lam = O.query_basis(Q, 1)
    assert lam[0] == pytest.approx((a + c) / 2 + math.sqrt(((a - c) / 2) ** 2 + b * b), rel=1e-12)
    th = 0.5 * math.atan2(2 * b, a - c)
    v = np.array([math.cos(th), math.sin(th)])
    v = v * np.sign(v[np.argmax(np.abs(v))])
    assert np.allclose(P[:, 0], v, atol=1e-12)


def test_query_basis_planted_subspace_and_invariances():
    """Queries drawn in a planted s-dimensional subspace with distinct scales plus small isotropic
    noise: the basis spans the planted subspace (projectors agree to sampling error); permuting the
    rows leaves the basis unchanged and scaling them by 2 multiplies the eigenvalues by 4; the
    columns are orthonormal with the sign rule."""
    rng = np.random.default_rng(72)
    d, s, n = 64, 12, 40000
    P0, _ = np.linalg.qr(rng.standard_normal((d, s)))
    sig = np.linspace(3.0, 1.5, s)
    Q = (rng.standard_normal((n, s)) * sig) @ P0.T + 0.05 * rng.standard_normal((n, d))
    P, lam = O.query_basis(Q, s)
    assert np.abs(P @ P.T - P0 @ P0.T).max() < 0.02
    assert np.allclose(lam, sig ** 2 + 0.05 ** 2, rtol=0.05)
    assert np.allclose(P.T @ P, np.eye(s), atol=1e-12)
    for k in range(s):
        assert P[np.argmax(np.abs(P[:, k])), k] > 0
    P2, lam2 = O.query_basis(Q[rng.permutation(n)], s)
    assert np.allclose(P2, P, atol=1e-9) and np.allclose(lam2, lam, rtol=1e-12)
    P3, lam3 = O.query_basis(2 * Q, s)
    assert np.allclose(P3, P, atol=1e-9) and np.allclose(lam3, 4 * lam, rtol=1e-12)
