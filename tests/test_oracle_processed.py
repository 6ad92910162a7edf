"""Pins of the oracle's processed logprobs (the distribution the draw samples
from, after temperature, top-k and top-p): normalisation, the special cases
that reduce to a library log-softmax or to a point mass, ratio invariance,
the order of the top-n, agreement with the kept set of the draw, and the
frequencies of the oracle's own Gumbel-max draws."""
import numpy as np
import pytest
from scipy import special, stats

from oracle.sampler import processed_logprobs, sample_row, scale


def _row(V, seed, spread=2.0, neg_inf=0):
    rng = np.random.default_rng(seed)
    l = (rng.standard_normal(V) * spread).astype(np.float32)
    if neg_inf:
        l[rng.choice(V, neg_inf, replace=False)] = -np.inf
    return l


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("T,k,p", [(1.0, 0, 0.9), (0.7, 50, 0.95), (1.3, 5, 1.0), (0.5, 0, 0.3), (2.0, 300, 0.99)])
def test_normalised_on_the_kept_set(seed, T, k, p):
    l = _row(257, seed, neg_inf=seed % 3)
    r = processed_logprobs(l, T, k, p, 20)
    assert r.flags == 0
    assert abs(np.sum(np.exp(r.logprob[r.kept])) - 1.0) < 1e-12
    assert np.all(r.logprob[~r.kept] == -np.inf)
    assert np.all(np.isfinite(r.logprob[r.kept]))


@pytest.mark.parametrize("T", [0.5, 1.0, 1.7])
def test_full_vocabulary_is_the_library_log_softmax_of_x(T):
    l = _row(1000, 3, neg_inf=7)
    r = processed_logprobs(l, T, 0, 1.0, 5)
    x = scale(l, T).astype(np.float64)
    fin = np.isfinite(x)
    ref = special.log_softmax(x[fin])
    assert np.max(np.abs(r.logprob[fin] - ref)) < 1e-12
    assert np.all(r.logprob[~fin] == -np.inf) and np.array_equal(r.kept, fin)


def test_point_masses():
    l = _row(64, 5)
    am = int(np.argmax(l))
    for r in (processed_logprobs(l, 0.0, 7, 0.5, 4),    # greedy ignores k and p
              processed_logprobs(l, 1.0, 1, 1.0, 4),    # top_k = 1, no ties
              processed_logprobs(l, 1.0, 0, 1e-6, 4)):  # top_p -> 0
        assert r.topn_ids.tolist() == [am, -1, -1, -1]
        assert r.topn_logprob[0] == 0.0 and np.all(r.topn_logprob[1:] == -np.inf)
        assert r.kept.sum() == 1 and r.logprob[am] == 0.0


def test_ratios_of_kept_tokens_are_exp_of_x_differences():
    l = _row(300, 9)
    r = processed_logprobs(l, 0.8, 40, 0.9, 20)
    x = scale(l, 0.8).astype(np.float64)
    ids = np.nonzero(r.kept)[0]
    d_lp = r.logprob[ids][:, None] - r.logprob[ids][None, :]
    d_x = x[ids][:, None] - x[ids][None, :]
    assert np.max(np.abs(d_lp - d_x)) < 1e-12


def test_topn_order_ties_and_padding():
    # equal x from equal logits: lower id first; fewer kept tokens than n: padded
    l = np.array([1.0, 3.0, 3.0, -np.inf, 2.0, 3.0, 0.5], np.float32)
    r = processed_logprobs(l, 1.0, 3, 1.0, 6)
    assert r.topn_ids.tolist() == [1, 2, 5, -1, -1, -1]
    assert np.allclose(r.topn_logprob[:3], np.log(1.0 / 3.0)) and np.all(r.topn_logprob[3:] == -np.inf)
    # equal x from different logits (the division maps two adjacent floats to one
    # float32): by id, where the raw order would put the larger logit first
    T = np.float32(0.51)
    a = np.float32(1.5)
    while True:
        b = np.nextafter(a, np.float32(2.0))
        if scale(np.array([a]), T)[0] == scale(np.array([b]), T)[0]:
            break
        a = b
    r = processed_logprobs(np.array([a, b, -1.0], np.float32), T, 0, 1.0, 2)
    assert r.topn_ids.tolist() == [0, 1]


@pytest.mark.parametrize("seed", range(4))
def test_kept_set_is_the_draws(seed):
    l = _row(500, 20 + seed, neg_inf=3)
    for T, k, p in [(1.0, 0, 0.8), (0.6, 30, 0.9), (1.5, 200, 1.0)]:
        r = processed_logprobs(l, T, k, p, 5)
        s = sample_row(l, T, k, p, 3, 11, seed, 5)
        assert np.array_equal(r.kept, s.kept)
        assert np.isfinite(r.logprob[s.token])


def test_flagged_rows():
    l = _row(32, 1)
    l[4] = np.nan
    r = processed_logprobs(l, 1.0, 0, 0.9, 3)
    assert r.flags != 0 and r.topn_ids.tolist() == [-1, -1, -1] and np.all(np.isnan(r.topn_logprob))
    r = processed_logprobs(_row(32, 1), -1.0, 0, 0.9, 3)
    assert r.flags != 0 and np.all(np.isnan(r.logprob))


def test_frequencies_of_the_oracles_draws():
    """20,000 Gumbel-max draws of the oracle (swept seeds) fall on the tokens
    with the processed probabilities (chi-square, alpha = 1e-3), and not with
    the raw softmax over the whole row."""
    l = np.array([2.0, 1.5, 1.4, 1.0, 0.9, 0.2, -0.5, -1.0, 0.0, 1.2, -3.0, 0.7], np.float32)
    T, k, p = 0.8, 8, 0.9
    r = processed_logprobs(l, T, k, p, 3)
    N = 20000
    counts = np.zeros(l.size)
    for s in range(N):
        counts[sample_row(l, T, k, p, 5, 17, s, 0).token] += 1
    q = np.exp(r.logprob)
    kept = r.kept
    assert counts[~kept].sum() == 0
    chi2 = np.sum((counts[kept] - N * q[kept]) ** 2 / (N * q[kept]))
    assert stats.chi2.sf(chi2, kept.sum() - 1) > 1e-3
    raw = special.softmax(l.astype(np.float64))
    chi2_raw = np.sum((counts - N * raw) ** 2 / (N * raw))
    assert stats.chi2.sf(chi2_raw, l.size - 1) < 1e-3
    # a plausible mistake, the probabilities at the wrong temperature, is rejected too
    q1 = np.exp(processed_logprobs(l, 1.0, k, p, 3).logprob)
    with np.errstate(divide="ignore", invalid="ignore"):
        terms = np.where(counts > 0, (counts - N * q1) ** 2 / (N * q1), N * q1)
    assert stats.chi2.sf(np.sum(terms), l.size - 1) < 1e-3
