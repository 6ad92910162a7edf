"""Statistical pin for the oracle's draw: Gumbel-max over the kept set samples
the kept set's renormalised softmax.  Frequencies of >= 10**6 draws over swept
(position, seed) are compared with the closed-form probabilities by a
chi-square test at a fixed significance of 1e-3 with fixed seeds."""
import numpy as np
import pytest
from scipy import stats

from oracle import sampler as S


def _draw_frequencies(x, kept_ids, request_id, positions, seeds):
    counts = np.zeros(kept_ids.size, np.int64)
    for seed in seeds:
        for lo in range(0, positions.size, 50_000):
            pos = positions[lo:lo + 50_000, None]
            s = S.gumbel_scores(x[kept_ids][None, :], kept_ids[None, :], request_id, pos, seed)
            counts += np.bincount(np.argmax(s, axis=1), minlength=kept_ids.size)
    return counts


def _chi2_pvalue(counts, probs):
    expect = probs * counts.sum()
    order = np.argsort(expect)
    # merge the smallest expected cells until every cell expects >= 5 draws
    obs_m, exp_m, acc_o, acc_e = [], [], 0, 0.0
    for i in order:
        acc_o += counts[i]
        acc_e += expect[i]
        if acc_e >= 5:
            obs_m.append(acc_o)
            exp_m.append(acc_e)
            acc_o, acc_e = 0, 0.0
    if acc_e > 0:
        obs_m[-1] += acc_o
        exp_m[-1] += acc_e
    return stats.chisquare(obs_m, exp_m).pvalue


@pytest.mark.parametrize("T,k,p", [(1.0, 50, 0.9), (0.7, 0, 0.6), (1.3, 20, 1.0)])
def test_draw_frequencies_match_truncated_softmax(T, k, p):
    rng = np.random.default_rng(4242)
    V = 1024
    l = rng.normal(0, 1.4, V).astype(np.float32)
    if k == 0:       # keep the kept set small enough for 10**6 vectorised draws
        l[:800] -= 6
    r = S.sample_row(l, T, k, p, 17, 0, 0, 0)
    ids = np.nonzero(r.kept)[0]
    x = S.scale(l, T).astype(np.float64)
    w = np.exp(x[ids] - x[ids].max())
    probs = w / w.sum()
    counts = _draw_frequencies(S.scale(l, T), ids, 17, np.arange(250_000), seeds=[0, 1, 2, 3])
    assert counts.sum() == 1_000_000
    assert _chi2_pvalue(counts, probs) > 1e-3


def test_chi2_detects_a_wrong_temperature():
    """The same test rejects draws made at the wrong temperature."""
    rng = np.random.default_rng(7)
    l = rng.normal(0, 1.4, 64).astype(np.float32)
    ids = np.arange(64)
    x_true = S.scale(l, 1.0).astype(np.float64)
    probs = np.exp(x_true - x_true.max())
    probs /= probs.sum()
    counts = _draw_frequencies(S.scale(l, 1.15), ids, 3, np.arange(200_000), seeds=[0])
    assert _chi2_pvalue(counts, probs) < 1e-3
