"""The pruning rule a sampler can apply with tile statistics, checked on the CPU
with the oracle: for a row with top-k (or a greedy row) and n logprobs, let
R = max(n, k) (greedy: max(n, 1)) and t0 the R-th largest block maximum.  R
blocks hold a value >= t0, so the R-th largest logit is >= t0; x = fl(l / T)
is non-decreasing in l, so every token top-k keeps (x >= theta_k) and every
top-n logit lies in a quarter whose largest x is >= fl(t0 / T).  Only those
quarters need to be read."""
import numpy as np
import pytest

from oracle.sampler import scale, top_k_threshold, top_n
from oracle.tile_stats import tile_stats


def selected_quarters(rec, R, T):
    qmax = rec[:, :4].reshape(-1)
    bmax = rec[:, :4].max(axis=1)
    if R > bmax.size:
        return np.ones(qmax.size, bool)
    t0 = np.sort(bmax)[::-1][R - 1]
    if T == 0.0:
        return qmax >= t0
    return scale(qmax, T) >= scale(np.float32(t0), T)


def quarter_of(ids, S, V_s):
    B = -(-V_s // 128)
    s, j = np.divmod(ids, V_s)
    return (s * B + j // 128) * 4 + (j % 128) // 32


def rows(kind, rng, V):
    if kind == "gauss":
        return rng.normal(0.0, 1.3, V).astype(np.float32)
    if kind == "zipf":
        l = (-1.1 * np.log(np.arange(1, V + 1))).astype(np.float32)
        l = l[rng.permutation(V)]
        l[rng.integers(0, V, 2)] = 12.0
        return l
    if kind == "quantised":  # many exact ties
        return np.round(rng.normal(0.0, 1.0, V) * 16.0).astype(np.float32) / 16.0
    raise KeyError(kind)


@pytest.mark.parametrize("kind", ["gauss", "zipf", "quantised"])
@pytest.mark.parametrize("T,k,n", [(0.8, 40, 20), (1.0, 1000, 20), (0.37, 1, 0), (0.0, 0, 20), (1e-3, 20, 5)])
def test_pruned_quarters_hold_kept_set_and_top_n(kind, T, k, n):
    rng = np.random.default_rng(hash((kind, T, k, n)) & 0xFFFF)
    S, V_s = 4, 2500  # ragged last block (2500 = 19 * 128 + 68)
    V = S * V_s
    for _ in range(3):
        l = rows(kind, rng, V)
        rec = tile_stats([l[None, s * V_s:(s + 1) * V_s] for s in range(S)])[0]
        R = max(n, k) if T > 0 else max(n, 1)
        sel = selected_quarters(rec, R, T)
        need = set(top_n(l, n).tolist()) if n else set()
        if T > 0:
            x = scale(l, T)
            need |= set(np.flatnonzero(x >= top_k_threshold(x, k)).tolist())
        else:
            need.add(int(top_n(l, 1)[0]))
        q = quarter_of(np.array(sorted(need)), S, V_s)
        assert sel[q].all()
        # and the rule prunes: about R quarters when R is well below the block count
        if 4 * R <= rec.shape[0] and kind == "gauss":
            assert sel.sum() <= 2 * R + 8
