"""Pins for the sampler oracle: brute force on tiny vocabularies and closed forms.

The brute-force checks restate each rule in a second, independent form
(top-k as "fewer than k tokens strictly greater", top-p as an explicit double
loop with math.exp) so that a dropped term, a wrong inequality, a wrong tie
rule or a transposed operand in the oracle fails here.
"""
import math

import numpy as np
import pytest

from oracle import sampler as S
from oracle.philox import token_uniforms


def _brute_kept(l, T, k, p):
    """Kept set by explicit loops over the definitions (Python floats)."""
    V = len(l)
    x = [float(np.float32(np.float32(v) / np.float32(T)) + np.float32(0)) for v in l]
    finite = [math.isfinite(float(v)) for v in l]
    keep = list(finite)
    if 0 < k < V:
        for i in range(V):
            greater = sum(1 for j in range(V) if x[j] > x[i])
            keep[i] = keep[i] and greater < k
    if p < 1:
        K = [i for i in range(V) if keep[i]]
        m = max(x[i] for i in K)
        Z = sum(math.exp(x[j] - m) for j in K)
        new = [False] * V
        for i in K:
            mass = sum(math.exp(x[j] - m) / Z for j in K if x[j] > x[i])
            new[i] = mass < float(np.float32(p))
        keep = new
    return np.array(keep)


def _random_row(rng, V, ties=False, neg_inf=False):
    l = rng.normal(0.0, rng.uniform(0.3, 3.0), V).astype(np.float32)
    if ties:
        l = (np.round(l * 4) / 4).astype(np.float32)
    if neg_inf and V > 2:
        l[rng.choice(V, rng.integers(1, V - 1), replace=False)] = -np.inf
    return l


@pytest.mark.parametrize("case", range(400))
def test_kept_set_matches_brute_force(case):
    rng = np.random.default_rng(case)
    V = int(rng.integers(1, 13))
    l = _random_row(rng, V, ties=case % 3 == 0, neg_inf=case % 5 == 0)
    if not np.any(np.isfinite(l)):
        l[0] = 0.0
    T = float(np.float32(rng.choice([0.25, 0.7, 1.0, 1.3, 2.0])))
    k = int(rng.integers(0, V + 2))
    p = float(np.float32(rng.choice([0.05, 0.3, 0.5, 0.9, 0.99, 1.0])))
    r = S.sample_row(l, T, k, p, 1, 2, 3, 0)
    if r.cut_tie:
        pytest.skip("boundary mass within the cut-tie tolerance")
    expect = _brute_kept(l, T, k, p)
    assert np.array_equal(r.kept, expect)
    assert r.kept[r.token]


@pytest.mark.parametrize("case", range(100))
def test_draw_matches_enumeration(case):
    """token = argmax over the kept set of x + Gumbel noise, lowest id on ties."""
    rng = np.random.default_rng(1000 + case)
    V = int(rng.integers(2, 40))
    l = _random_row(rng, V, ties=case % 2 == 0)
    T, k, p = 0.9, int(rng.integers(0, V)), 0.8
    req, pos, seed = int(rng.integers(0, 1 << 20)), int(rng.integers(0, 9000)), int(rng.integers(0, 1 << 40))
    r = S.sample_row(l, T, k, p, req, pos, seed, 0)
    best, best_id = -math.inf, -1
    for i in range(V):
        if not r.kept[i]:
            continue
        u = float(token_uniforms(i, req, pos, seed))
        s = float(np.float32(np.float32(l[i]) / np.float32(T))) - math.log(-math.log(u))
        if s > best:
            best, best_id = s, i
    assert r.token == best_id


def test_greedy_is_argmax_lowest_id():
    l = np.array([0.5, 3.0, -1.0, 3.0, 2.9], np.float32)
    for k, p in [(0, 1.0), (2, 0.1), (1, 0.5)]:
        r = S.sample_row(l, 0.0, k, p, 0, 0, 0, 3)
        assert r.token == 1
    assert list(S.top_n(l, 3)) == [1, 3, 4]


@pytest.mark.parametrize("seed", range(20))
def test_top_k_one_is_argmax(seed):
    rng = np.random.default_rng(seed)
    l = rng.normal(0, 2, 300).astype(np.float32)
    r = S.sample_row(l, 0.8, 1, 1.0, seed, 5, seed, 0)
    assert r.token == int(np.argmax(l)) and r.kept.sum() == 1


@pytest.mark.parametrize("seed", range(20))
def test_tiny_top_p_is_argmax(seed):
    rng = np.random.default_rng(seed)
    l = rng.normal(0, 2, 300).astype(np.float32)
    r = S.sample_row(l, 1.1, 0, 1e-7, seed, 5, seed, 0)
    assert r.token == int(np.argmax(l)) and r.kept.sum() == 1


def test_top_p_one_and_k_off_keep_all_finite():
    rng = np.random.default_rng(5)
    l = rng.normal(0, 1, 500).astype(np.float32)
    l[::7] = -np.inf
    for k in (0, 500, 501, 10_000):
        r = S.sample_row(l, 1.0, k, 1.0, 0, 0, 0, 0)
        assert np.array_equal(r.kept, np.isfinite(l))
    r_off = S.sample_row(l, 1.0, 0, 0.7, 4, 4, 4, 0)
    r_big = S.sample_row(l, 1.0, 500, 0.7, 4, 4, 4, 0)
    assert np.array_equal(r_off.kept, r_big.kept) and r_off.token == r_big.token


def test_top_k_keeps_ties_at_boundary():
    l = np.array([5, 4, 4, 4, 1, 0], np.float32)
    r = S.sample_row(l, 1.0, 2, 1.0, 0, 0, 0, 0)
    assert r.kept.tolist() == [True, True, True, True, False, False]


def test_top_p_keeps_ties_at_cut():
    # x = [1, 0, 0]: p = [e/(e+2), 1/(e+2), 1/(e+2)] ~ [0.576, 0.212, 0.212]
    l = np.array([1, 0, 0], np.float32)
    r = S.sample_row(l, 1.0, 0, 0.6, 0, 0, 0, 0)
    assert r.kept.tolist() == [True, True, True]
    r = S.sample_row(l, 1.0, 0, 0.5, 0, 0, 0, 0)
    assert r.kept.tolist() == [True, False, False]


def test_top_p_renormalises_over_top_k_survivors():
    # l = [2, 1, 0], k = 2: survivors {0, 1} with renormalised masses
    # e/(e+1) ~ 0.731 and 0.269; over the full row token 0 would carry
    # e^2/(e^2+e+1) ~ 0.665.  With top_p = 0.7 token 1 is dropped under the
    # renormalised reading and kept under the full-row one.
    l = np.array([2, 1, 0], np.float32)
    r = S.sample_row(l, 1.0, 2, 0.7, 0, 0, 0, 0)
    assert r.kept.tolist() == [True, False, False]
    r_full = S.sample_row(l, 1.0, 0, 0.7, 0, 0, 0, 0)
    assert r_full.kept.tolist() == [True, True, False]


def test_logprobs_normalise_and_sort():
    rng = np.random.default_rng(9)
    l = rng.normal(0, 3, 2000).astype(np.float32)
    l[:50] = -np.inf
    lp = S.log_softmax(l)
    assert abs(np.sum(np.exp(lp[np.isfinite(lp)])) - 1.0) < 1e-12
    r = S.sample_row(l, 1.0, 0, 1.0, 0, 0, 0, 20)
    assert np.all(np.diff(r.topn_logprob) <= 0)
    assert set(r.topn_ids.tolist()) == set(np.argsort(-l, kind="stable")[:20].tolist())
    # the sampled token's logprob is its raw log-softmax value
    assert r.token_logprob == lp[r.token]


def test_logprob_closed_form_uniform_row():
    l = np.zeros(1024, np.float32)
    lp = S.log_softmax(l)
    assert np.allclose(lp, -math.log(1024), atol=1e-14, rtol=0)


def test_temperature_is_a_true_division():
    # scaling l and T by the same power of two leaves x = fl(l / T) unchanged
    rng = np.random.default_rng(3)
    l = rng.normal(0, 2, 700).astype(np.float32)
    a = S.sample_row(l, 0.7, 30, 0.9, 2, 3, 4, 0)
    b = S.sample_row(l * np.float32(4), 2.8, 30, 0.9, 2, 3, 4, 0)
    assert a.token == b.token and np.array_equal(a.kept, b.kept)
    # and a different temperature changes the kept set for this row
    c = S.sample_row(l, 0.3, 30, 0.9, 2, 3, 4, 0)
    assert not np.array_equal(a.kept, c.kept)


def test_flags():
    good = np.array([0.0, 1.0, 2.0], np.float32)
    assert S.sample_row(np.array([0, np.nan, 1], np.float32), 1, 0, 1, 0, 0, 0, 2).flags == S.FLAG_NONFINITE
    assert S.sample_row(np.array([0, np.inf, 1], np.float32), 1, 0, 1, 0, 0, 0, 2).flags == S.FLAG_NONFINITE
    assert S.sample_row(np.full(3, -np.inf, np.float32), 1, 0, 1, 0, 0, 0, 2).flags == S.FLAG_ALL_NEG_INF
    assert S.sample_row(good, -1.0, 0, 1, 0, 0, 0, 2).flags == S.FLAG_BAD_TEMPERATURE
    assert S.sample_row(good, float("nan"), 0, 1, 0, 0, 0, 2).flags == S.FLAG_BAD_TEMPERATURE
    assert S.sample_row(good, 1.0, 0, 0.0, 0, 0, 0, 2).flags == S.FLAG_BAD_TOP_P
    assert S.sample_row(good, 1.0, -1, 1.0, 0, 0, 0, 2).flags == S.FLAG_BAD_TOP_K
    big = np.array([3e38, 1.0], np.float32)
    r = S.sample_row(big, 0.5, 0, 1.0, 0, 0, 0, 2)
    assert r.flags == S.FLAG_SCALE_OVERFLOW and r.token == -1
    assert S.sample_row(big, 0.0, 0, 1.0, 0, 0, 0, 2).flags == 0   # greedy does not scale


def test_negative_zero_ties_positive_zero():
    l = np.array([-0.0, 0.0, -1.0], np.float32)
    assert list(S.top_n(l, 2)) == [0, 1]
    r = S.sample_row(l, 1.0, 1, 1.0, 0, 0, 0, 0)
    assert r.kept.tolist() == [True, True, False]
