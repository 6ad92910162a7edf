"""Tile statistics on the GPU (the statistics kernel and the projection's
epilogue) against the oracle, and the sampler's tile mode: the same tokens,
kept sets, top-n and flags as the oracle (and as the sampler without the
statistics), raw logprobs within 1e-4."""
import numpy as np
import pytest
import torch

import vocab_sharded_logits_b200 as vsl
import workloads as W
from oracle.gemm import logits_local as ref_logits
from oracle.tile_stats import tile_stats as ref_tile_stats
from parity_helpers import compare, run_sampler

pytestmark = pytest.mark.gpu

SUM_RTOL = 2e-6  # block sums: float32 terms from a fast exp2, summed in float32


def check_records(got, want):
    """Maxima and minima exact (a quarter holding a NaN excepted), sums within
    SUM_RTOL (NaN and +inf where the oracle has them), reserved words 0."""
    got = np.asarray(got, np.float64)
    assert got.shape == want.shape
    nan_block = np.isnan(want[..., 4])
    q = got[..., :4][~nan_block]
    assert np.array_equal(q, want[..., :4][~nan_block]), np.argwhere(got[..., :4][~nan_block] != want[..., :4][~nan_block])[:5]
    assert np.array_equal(got[..., 5:7], want[..., 5:7])
    assert np.all(got[..., 7] == 0)
    s, w = got[..., 4], want[..., 4]
    assert np.array_equal(np.isnan(s), np.isnan(w))
    fin = np.isfinite(w)
    assert np.array_equal(s[~fin & ~np.isnan(w)], w[~fin & ~np.isnan(w)])
    assert np.all(np.abs(s[fin] - w[fin]) <= SUM_RTOL * np.abs(w[fin])), np.max(np.abs(s[fin] - w[fin]) / np.abs(w[fin]))


def special_logits(R, V, rng):
    l = rng.normal(0.0, 2.0, (R, V)).astype(np.float32)
    l[0, :] = -np.inf                       # a row of -inf
    l[1, : V // 2] = -np.inf                # whole blocks of -inf
    l[2, 7] = np.nan                        # NaN
    l[2, V - 3] = -np.nan                   # negative NaN
    l[3, 100 % V] = np.inf                  # +inf
    l[4, :] = np.round(l[4, :] * 2) / 2     # ties across quarters
    l[5, 3] = 3e38                          # huge finite
    l[5, 4] = -3e38
    return l


@pytest.mark.parametrize("R,S,V_s", [(6, 2, 300), (8, 4, 2500), (6, 4, 37984)])
def test_statistics_kernel_matches_oracle(cuda_device, R, S, V_s):
    rng = np.random.default_rng(V_s)
    l = special_logits(R, S * V_s, rng)
    slices = [torch.from_numpy(l[:, s * V_s:(s + 1) * V_s].copy()).to(cuda_device) for s in range(S)]
    got = vsl.tile_stats(slices)
    torch.cuda.synchronize()
    assert tuple(got.shape) == vsl.tile_stats_shape(R, S, V_s)
    want = ref_tile_stats([l[:, s * V_s:(s + 1) * V_s] for s in range(S)])
    check_records(got.cpu().numpy(), want)


@pytest.mark.parametrize("R,H,S,V_s", [
    (3, 64, 2, 300),     # BN = 16, ragged block
    (17, 128, 2, 1000),  # BN = 32
    (64, 256, 1, 2052),  # BN = 64
    (100, 128, 2, 260),  # BN = 128
    (300, 64, 1, 388),   # two batch tiles of 256, ragged
])
def test_projection_statistics_match_oracle(cuda_device, R, H, S, V_s):
    """Integer inputs make the projection exact, so the oracle's records of the
    oracle's own logits must match the epilogue's (maxima and minima exactly)."""
    g = torch.Generator(device=cuda_device)
    g.manual_seed(R + H + V_s)
    hidden = torch.randint(-3, 4, (R, H), generator=g, device=cuda_device).to(torch.bfloat16)
    ws = [torch.randint(-3, 4, (V_s, H), generator=g, device=cuda_device).to(torch.bfloat16) for _ in range(S)]
    out, stats = vsl.logits_local(hidden, ws, tile_stats=True)
    torch.cuda.synchronize()
    ref = ref_logits(hidden.float().cpu().numpy(), [w.float().cpu().numpy() for w in ws])
    for o, r in zip(out, ref):
        assert np.array_equal(o.cpu().numpy().astype(np.float64), r)
    check_records(stats.cpu().numpy(), ref_tile_stats(ref))


@pytest.mark.parametrize("name", ["decode", "spec", "peaked"])
def test_projection_statistics_full_size(cuda_device, name):
    """At a full configuration's shape, on integer inputs (weights in steps of
    1/64, so the projection is exact): three rows' logits and records equal
    the oracle's computed from the same inputs."""
    w = W.WORKLOADS[name]
    g = torch.Generator(device=cuda_device)
    g.manual_seed(w.data_seed + 17)
    hidden = torch.randint(-3, 4, (w.R, w.H), generator=g, device=cuda_device).to(torch.bfloat16)
    ws = [(torch.randint(-3, 4, (w.V_s, w.H), generator=g, device=cuda_device).float() / 64).to(torch.bfloat16)
          for _ in range(w.S)]
    out, stats = vsl.logits_local(hidden, ws, tile_stats=True)
    torch.cuda.synchronize()
    rows = [0, w.R // 2, w.R - 1]
    ref = ref_logits(hidden[rows].float().cpu().numpy(), [x.float().cpu().numpy() for x in ws])
    for o, r in zip(out, ref):
        assert np.array_equal(o[rows].cpu().numpy().astype(np.float64), r)
    check_records(stats[rows].cpu().numpy(), ref_tile_stats(ref))


@pytest.mark.parametrize("name", ["decode", "spec", "peaked"])
def test_projection_and_kernel_statistics_agree(cuda_device, name):
    """On the workloads' own inputs the epilogue's records equal the statistics
    kernel's of the same logits (maxima and minima bit-exact, sums within 2 x
    SUM_RTOL): the two producers of the records agree."""
    w = W.WORKLOADS[name]
    hidden, ws = W.gemm_inputs(w, cuda_device)
    out, stats = vsl.logits_local(hidden, ws, tile_stats=True)
    again = vsl.tile_stats(out)
    torch.cuda.synchronize()
    a, b = stats.cpu().numpy(), again.cpu().numpy()
    assert np.array_equal(a[..., :4], b[..., :4]) and np.array_equal(a[..., 5:], b[..., 5:])
    assert np.all(np.abs(a[..., 4] - b[..., 4]) <= 2 * SUM_RTOL * np.abs(b[..., 4]))


def _same_as_without(a, b):
    for key in ("token", "topn_ids", "flags", "theta", "p_topn_ids"):
        assert np.array_equal(a[key], b[key], equal_nan=True), key
    for key in ("token_lp", "topn_lp"):
        assert np.allclose(a[key], b[key], atol=2e-5, rtol=0, equal_nan=True), key


@pytest.mark.parametrize("name", ["decode", "spec", "peaked", "tiny", "large"])
def test_tile_mode_small_vocab_all_rows(cuda_device, name):
    w = W.scaled(W.WORKLOADS[name], V=8 * 1500, requests=max(4, 64 // W.WORKLOADS[name].rows_per_request)) \
        if name != "tiny" else W.WORKLOADS[name]
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    got = run_sampler(logits, params, 0, w.n_logprobs, w.S, cuda_device, tiles=True)
    ref = run_sampler(logits, params, 0, w.n_logprobs, w.S, cuda_device)
    _same_as_without(got, ref)
    st = compare(got, logits.cpu().numpy(), params, 0, w.n_logprobs, range(w.R))
    assert st["mismatch_allowed"] <= max(1, st["rows"] // 50)


@pytest.mark.parametrize("name,nrows", [("decode", 48), ("spec", 64), ("peaked", 32), ("large", 8), ("wide", 32)])
def test_tile_mode_full_size(cuda_device, name, nrows):
    w = W.WORKLOADS[name]
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    got = run_sampler(logits, params, 7, w.n_logprobs, w.S, cuda_device, tiles=True)
    ref = run_sampler(logits, params, 7, w.n_logprobs, w.S, cuda_device)
    _same_as_without(got, ref)
    rows = sorted(np.random.default_rng(9).choice(w.R, min(nrows, w.R), replace=False).tolist())
    compare(got, logits.cpu().numpy(), params, 7, w.n_logprobs, rows)


def test_tile_mode_peaked_seed_sweep(cuda_device):
    w = W.WORKLOADS["peaked"]
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    logits_np = logits.cpu().numpy()
    for seed in range(0, 16, 3):
        got = run_sampler(logits, params, seed, w.n_logprobs, w.S, cuda_device, tiles=True)
        rows = sorted(np.random.default_rng(200 + seed).choice(w.R, 8, replace=False).tolist())
        compare(got, logits_np, params, seed, w.n_logprobs, rows)


@pytest.mark.parametrize("V,S", [(1024, 2), (12000, 4), (151936, 8)])
def test_tile_mode_edge_cases(cuda_device, V, S):
    from test_sample_gpu import _edge_rows
    rng = np.random.default_rng(V + 1)
    logits, prm = _edge_rows(V, rng)
    R = logits.shape[0]
    params = (np.array([p[0] for p in prm], np.float32), np.array([p[1] for p in prm], np.int32),
              np.array([p[2] for p in prm], np.float32), np.arange(R), np.arange(R) * 3 + 1)
    n = min(20, V)
    t = torch.from_numpy(logits)
    got = run_sampler(t, params, 99, n, S, cuda_device, tiles=True)
    ref = run_sampler(t, params, 99, n, S, cuda_device)
    _same_as_without(got, ref)
    compare(got, logits, params, 99, n, range(R))


def test_tile_mode_large_batch_mixed(cuda_device):
    """A large batch (one CTA per row, top-k-off rows streamed as before) whose
    top-k and greedy rows take the tile mode."""
    w = W.scaled(W.WORKLOADS["decode"], V=4 * 5000, requests=400)
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    got = run_sampler(logits, params, 3, w.n_logprobs, w.S, cuda_device, tiles=True)
    ref = run_sampler(logits, params, 3, w.n_logprobs, w.S, cuda_device)
    _same_as_without(got, ref)
    rows = sorted(np.random.default_rng(4).choice(w.R, 40, replace=False).tolist())
    compare(got, logits.cpu().numpy(), params, 3, w.n_logprobs, rows)
    assert vsl.device_error() == (0, 0)


@pytest.mark.parametrize("V,S", [(12000, 4), (151936, 8)])
def test_tile_mode_large_batch_top_k_off(cuda_device, V, S):
    """Top-k-off rows of a large batch take their statistics, smallest nonzero
    |l| (the division's domain check) and top-n candidates from the records
    and stream their row for the top-p passes only: the same results as
    without the records, and the oracle's."""
    from test_sample_gpu import _koff_rows
    R = 300
    rng = np.random.default_rng(V + 5)
    logits, params = _koff_rows(V, R, rng)
    t = torch.from_numpy(logits)
    got = run_sampler(t, params, 4243, 20, S, cuda_device, tiles=True)
    ref = run_sampler(t, params, 4243, 20, S, cuda_device)
    _same_as_without(got, ref)
    rows = range(R) if V <= 12000 else sorted(set(range(12)) | set(rng.choice(R, 28, replace=False).tolist()))
    st = compare(got, logits, params, 4243, 20, rows)
    assert st["mismatch_allowed"] <= 2


@pytest.mark.parametrize("S,V_s", [(16, 32768), (15, 34952)])
def test_tile_mode_at_the_record_limit(cuda_device, S, V_s):
    """4,096 blocks of 128 (the quarter maxima fill the streaming kernel's ring
    exactly) and 4,110 (above the limit: the sampler ignores the records), at
    vocabularies of about 524k: the same results as without the records, and
    the oracle's.  Such vocabularies need clusters of 16 CTAs; a device that
    does not schedule them rejects the size and the test is skipped."""
    R = 6
    rng = np.random.default_rng(S)
    logits = rng.normal(0.0, 1.5, (R, S * V_s)).astype(np.float32)
    params = (np.array([0.0, 0.8, 1.0, 0.7, 1.2, 0.9], np.float32), np.array([0, 40, 1000, 20, 1, 64], np.int32),
              np.array([1.0, 0.9, 0.95, 1.0, 0.5, 0.8], np.float32), np.arange(R), np.arange(R))
    t = torch.from_numpy(logits)
    try:
        ref = run_sampler(t, params, 5, 20, S, cuda_device)
    except vsl.VslError as e:
        if e.status == 3:
            pytest.skip("the device does not schedule the clusters this vocabulary needs")
        raise
    got = run_sampler(t, params, 5, 20, S, cuda_device, tiles=True)
    _same_as_without(got, ref)
    compare(got, logits, params, 5, 20, range(R))
