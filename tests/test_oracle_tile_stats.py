"""Pins of the tile-statistics oracle: closed forms, special values, the record
layout, and the merge of the blocks' sums against a library logsumexp."""
import numpy as np
import pytest
from scipy.special import logsumexp

from oracle.tile_stats import BLOCK, blocks_per_slice, block_record, row_logsumexp, tile_stats


def geometric(n, d):
    """sum_{k=0}^{n-1} exp(-d k) in closed form."""
    return (1.0 - np.exp(-d * n)) / (1.0 - np.exp(-d))


@pytest.mark.parametrize("n", [128, 100, 33, 1])
def test_arithmetic_progression_closed_form(n):
    a, d = -3.25, 0.015625
    vals = a + d * np.arange(n)
    rec = block_record(vals)
    for q in range(4):
        last = min(32 * q + 31, n - 1)
        want = a + d * last if 32 * q < n else -np.inf
        assert rec[q] == want
    # c is the largest value a + d (n - 1): terms exp(-d k), k = 0 .. n - 1
    assert rec[4] == pytest.approx(geometric(n, d), rel=1e-14)
    assert rec[5] == a
    # every term is negative (a + d (n - 1) < 0): the smallest |l| is the last one
    assert rec[6] == -(a + d * (n - 1))
    assert rec[7] == 0.0


def test_decreasing_progression_quarters():
    vals = 10.0 - 0.5 * np.arange(128)
    rec = block_record(vals)
    assert list(rec[:4]) == [10.0, 10.0 - 16.0, 10.0 - 32.0, 10.0 - 48.0]
    assert rec[4] == pytest.approx(geometric(128, 0.5), rel=1e-14)
    assert rec[5] == 10.0 - 0.5 * 127


def test_constant_block_sums_to_its_size():
    assert block_record(np.full(77, 4.5))[4] == 77.0


def test_smallest_nonzero_magnitude():
    vals = np.array([0.0, -0.0, -2.5, 1e-30, -3e-38, np.nan, 7.0] + [0.0] * 20)
    assert block_record(vals)[6] == 3e-38
    assert block_record(np.zeros(40))[6] == np.inf
    assert block_record(np.array([0.0, -np.inf, 0.0]))[6] == np.inf      # only an infinity: +inf
    assert block_record(np.array([0.0, -np.inf, -5.0]))[6] == 5.0


def test_negative_infinity_entries():
    vals = np.full(128, -np.inf)
    rec = block_record(vals)
    assert np.all(rec[:4] == -np.inf) and rec[4] == 0.0 and rec[5] == np.inf and rec[6] == np.inf
    vals[40] = 2.0
    vals[100] = -7.0
    rec = block_record(vals)
    assert rec[0] == -np.inf and rec[1] == 2.0 and rec[2] == -np.inf and rec[3] == -7.0
    assert rec[4] == pytest.approx(1.0 + np.exp(-9.0), rel=1e-15)
    assert rec[5] == -7.0


def test_nan_and_positive_infinity():
    vals = np.zeros(128)
    vals[5] = np.nan
    assert np.isnan(block_record(vals)[4])
    vals[5] = np.inf
    rec = block_record(vals)
    assert rec[0] == np.inf and rec[4] == np.inf and rec[5] == 0.0


def test_layout_one_hot():
    # one large value per row at a known global id: only its record's quarter shows it
    R, S, V_s = 3, 2, 300
    B = blocks_per_slice(V_s)
    assert B == 3
    rng = np.random.default_rng(5)
    slices = [rng.uniform(-1.0, 0.0, (R, V_s)) for _ in range(S)]
    ids = [0, 299 + 1, 2 * V_s - 1]  # slice 0 id 0; slice 1 id 0; slice 1 last id (partial block)
    for r, g in enumerate(ids):
        slices[g // V_s][r, g % V_s] = 50.0
    st = tile_stats(slices)
    assert st.shape == (R, S * B, 8)
    for r, g in enumerate(ids):
        s, j = divmod(g, V_s)
        b, q = j // BLOCK, (j % BLOCK) // 32
        hits = np.argwhere(st[r, :, :4] == 50.0)
        assert hits.tolist() == [[s * B + b, q]]
    # quarters past the slice's end are empty: V_s = 300 leaves 44 ids in block 2
    assert np.all(st[:, B - 1, 2:4] == -np.inf) and np.all(st[:, 2 * B - 1, 2:4] == -np.inf)


def test_merged_sums_equal_library_logsumexp():
    rng = np.random.default_rng(11)
    for V_s, S in [(512, 2), (300, 3), (1000, 1)]:
        slices = [rng.normal(0.0, 3.0, (4, V_s)) for _ in range(S)]
        slices[0][1, :V_s // 2] = -np.inf  # whole blocks of -inf
        st = tile_stats(slices)
        row = np.concatenate(slices, axis=1)
        for r in range(4):
            assert row_logsumexp(st[r]) == pytest.approx(logsumexp(row[r]), abs=1e-12)
            # the maxima of the quarters give the row maximum
            assert st[r, :, :4].max() == row[r].max()
