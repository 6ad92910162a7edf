"""Parity of the CUDA sampler with the oracle (GPU), on the same seeded fp32
logits: flags and token ids bit-exact (except near-ties / cut-ties, counted),
top-n ids exact, logprobs within 1e-4."""
import numpy as np
import pytest
import torch

import vocab_sharded_logits_b200 as vsl
import workloads as W
from parity_helpers import compare, run_sampler

pytestmark = pytest.mark.gpu


def _case(w, device, seed_offset=0, rows=None, S=None, seed=0):
    logits = W.sampler_logits(w, device, seed_offset)
    params = W.row_params(w, seed_offset)
    gpu = run_sampler(logits, params, seed, w.n_logprobs, S or w.S, device)
    rows = range(w.R) if rows is None else rows
    return compare(gpu, logits.cpu().numpy(), params, seed, w.n_logprobs, rows), gpu


def test_tiny_config_all_rows(cuda_device):
    st, _ = _case(W.WORKLOADS["tiny"], cuda_device)
    assert st["rows"] == 4


@pytest.mark.parametrize("name", ["decode", "spec", "large", "peaked", "wide"])
def test_small_vocab_versions_all_rows(cuda_device, name):
    # the configs' parameter recipes at a vocabulary the oracle handles in seconds,
    # still several CTAs per row and a ragged tail
    w = W.scaled(W.WORKLOADS[name], V=8 * 1500, requests=max(4, 64 // W.WORKLOADS[name].rows_per_request))
    st, _ = _case(w, cuda_device)
    assert st["mismatch_allowed"] <= max(1, st["rows"] // 50)


@pytest.mark.parametrize("name,nrows", [("decode", 64), ("spec", 48), ("large", 24), ("peaked", 24), ("wide", 32)])
def test_full_size_configs_sampled_rows(cuda_device, name, nrows):
    w = W.WORKLOADS[name]
    rows = np.random.default_rng(5).choice(w.R, min(nrows, w.R), replace=False)
    st, _ = _case(w, cuda_device, rows=sorted(rows.tolist()))
    assert st["rows"] == len(rows)


def test_peaked_full_size_seed_sweep(cuda_device):
    """The peaked / long-tail configuration at full size, draw seeds 0..15: the
    whole batch sampled per seed, 12 rows per seed compared with the oracle
    (tokens, kept sets, thresholds, top-n)."""
    w = W.WORKLOADS["peaked"]
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    logits_np = logits.cpu().numpy()
    total = {"rows": 0, "mismatch_allowed": 0}
    for seed in range(16):
        gpu = run_sampler(logits, params, seed, w.n_logprobs, w.S, cuda_device)
        rows = sorted(np.random.default_rng(100 + seed).choice(w.R, 12, replace=False).tolist())
        st = compare(gpu, logits_np, params, seed, w.n_logprobs, rows)
        total["rows"] += st["rows"]
        total["mismatch_allowed"] += st["mismatch_allowed"]
    assert total["rows"] == 16 * 12
    assert total["mismatch_allowed"] <= 4


@pytest.mark.parametrize("S", [1, 2, 4, 8])
def test_results_do_not_depend_on_slicing(cuda_device, S):
    w = W.scaled(W.WORKLOADS["decode"], V=8 * 1024, requests=32)
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    ref = run_sampler(logits, params, 3, w.n_logprobs, 1, cuda_device)
    got = run_sampler(logits, params, 3, w.n_logprobs, S, cuda_device)
    for key in ref:
        assert np.array_equal(ref[key], got[key], equal_nan=True), key


def test_run_twice_bitwise_equal(cuda_device):
    w = W.WORKLOADS["decode"]
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    a = run_sampler(logits, params, 11, 20, w.S, cuda_device)
    b = run_sampler(logits, params, 11, 20, w.S, cuda_device)
    for key in a:
        assert np.array_equal(a[key], b[key], equal_nan=True), key


def _edge_rows(V, rng):
    rows, params = [], []
    base = lambda: rng.normal(0, 1.5, V).astype(np.float32)
    add = lambda l, T, k, p: (rows.append(l), params.append((T, k, p)))
    add(base(), 0.0, 0, 1.0)                           # greedy
    add(base(), 1.0, 1, 1.0)                           # top_k = 1
    add(base(), 1.0, V, 1.0)                           # k >= V: off
    add(base(), 1.0, V + 7, 0.5)                       # k > V with top-p
    add(base(), 1.0, 0, 1.0)                           # pure sampling, full vocab
    add(base(), 0.7, 0, 0.3)                           # top-p only
    add(base(), 1.3, 3000, 0.9)                        # large k: narrowing path
    add(base(), 0.05, 0, 0.9)                          # very peaked
    add(base(), 50.0, 0, 0.95)                         # very flat
    add(np.zeros(V, np.float32), 1.0, 10, 0.5)         # all equal: ties everywhere
    add(np.zeros(V, np.float32), 0.0, 0, 1.0)          # all equal, greedy
    l = base(); l[::3] = -np.inf; add(l, 1.0, 50, 0.9)  # -inf mixed in
    l = np.full(V, -np.inf, np.float32); l[min(17, V - 1)] = 2.0; add(l, 1.0, 5, 0.9)  # one finite token
    l = np.full(V, -np.inf, np.float32); l[5:9] = 1.0; add(l, 1.0, 100, 1.0)  # k > #finite
    l = np.round(base() * 4) / 4; add(l.astype(np.float32), 1.0, 40, 0.8)    # quantised ties
    l = base(); l[min(100, V - 1)] = np.nan; add(l, 1.0, 0, 1.0)   # NaN -> flagged
    l = base(); l[3] = np.inf; add(l, 1.0, 0, 1.0)     # +inf -> flagged
    add(np.full(V, -np.inf, np.float32), 1.0, 0, 1.0)  # all -inf -> flagged
    add(base(), -1.0, 0, 1.0)                          # bad temperature
    add(base(), float("nan"), 0, 1.0)                  # bad temperature
    add(base(), 1.0, 0, 0.0)                           # bad top_p
    add(base(), 1.0, -3, 1.0)                          # bad top_k
    l = base(); l[0] = 3e38; add(l, 0.5, 0, 1.0)       # l / T overflows
    l = base(); l[::2] = -0.0; l[1::2] = 0.0; add(l, 1.0, 2, 1.0)  # signed zeros tie
    add(base() * np.float32(1e35) - np.float32(3e37), 1.0, 0, 0.9)  # finite, all far below -1e30
    l = base(); l[1] = -3.0e38; add(l, 1.0, 0, 0.9)        # |l| > 2.4e38: l log2(e) would overflow
    l = base(); l[2] = 3.0e38; add(l, 1.0, 0, 0.9)         # a huge finite maximum (x finite at T = 1)
    return np.stack(rows), params


@pytest.mark.parametrize("V,S", [(1024, 2), (12000, 4), (151936, 8), (8, 2)])
def test_edge_cases(cuda_device, V, S):
    rng = np.random.default_rng(V)
    logits, prm = _edge_rows(V, rng)
    R = logits.shape[0]
    T = np.array([p[0] for p in prm], np.float32)
    k = np.array([p[1] for p in prm], np.int32)
    p = np.array([p[2] for p in prm], np.float32)
    req = np.arange(R)
    pos = np.arange(R) * 3 + 1
    n = min(20, V)
    params = (T, k, p, req, pos)
    gpu = run_sampler(torch.from_numpy(logits), params, 1234, n, S, cuda_device)
    compare(gpu, logits, params, 1234, n, range(R))


def test_no_logprobs_requested(cuda_device):
    w = W.scaled(W.WORKLOADS["decode"], V=4 * 2048, requests=16)
    logits = W.sampler_logits(w, cuda_device)
    params = W.row_params(w)
    gpu = run_sampler(logits, params, 5, 0, w.S, cuda_device)
    compare(gpu, logits.cpu().numpy(), params, 5, 0, range(w.R))


def test_outputs_fully_written_over_poison(cuda_device):
    w = W.scaled(W.WORKLOADS["spec"], V=4 * 2048, requests=16)
    logits = W.sampler_logits(w, cuda_device)
    T, k, p, req, pos = W.row_params(w)
    slices = [t.contiguous() for t in torch.tensor_split(logits, w.S, dim=1)]
    prm = vsl.make_row_params(T, k, p, req, pos, cuda_device)
    out = vsl.SampleResult(torch.full((w.R,), -7, dtype=torch.int32, device=cuda_device),
                           torch.full((w.R,), float("nan"), device=cuda_device),
                           torch.full((w.R, w.n_logprobs), -7, dtype=torch.int32, device=cuda_device),
                           torch.full((w.R, w.n_logprobs), float("nan"), device=cuda_device),
                           torch.full((w.R,), 0x7777, dtype=torch.int32, device=cuda_device))
    vsl.sample(slices, prm, 0, w.n_logprobs, out=out)
    torch.cuda.synchronize()
    assert bool((out.token_ids >= 0).all()) and bool(torch.isfinite(out.token_logprob).all())
    assert bool((out.topn_ids >= 0).all()) and bool(torch.isfinite(out.topn_logprob).all())
    assert bool((out.row_flags == 0).all())
    assert vsl.device_error() == (0, 0)


def test_draw_frequencies_chi_square(cuda_device):
    """GPU draw frequencies over many positions match the oracle's truncated,
    renormalised distribution (chi-square, significance 1e-3, fixed seeds)."""
    from scipy import stats
    from oracle import sampler as S
    rng = np.random.default_rng(77)
    V = 1024
    l = rng.normal(0, 1.4, V).astype(np.float32)
    T, k, p = 0.9, 30, 0.9
    ref = S.sample_row(l, T, k, p, 0, 0, 0, 0)
    ids = np.nonzero(ref.kept)[0]
    x = S.scale(l, T).astype(np.float64)
    probs = np.exp(x[ids] - x[ids].max())
    probs /= probs.sum()
    R = 1 << 17
    logits = torch.from_numpy(np.tile(l, (R, 1)))
    params = (np.full(R, T, np.float32), np.full(R, k, np.int32), np.full(R, p, np.float32),
              np.full(R, 9), np.arange(R))
    counts = np.zeros(V, np.int64)
    for seed in (0, 1, 2, 3, 4, 5, 6, 7):
        gpu = run_sampler(logits, params, seed, 0, 2, cuda_device)
        counts += np.bincount(gpu["token"], minlength=V)
    assert counts[~ref.kept].sum() == 0
    obs = counts[ids]
    exp = probs * obs.sum()
    big = exp >= 5
    obs_m = np.append(obs[big], obs[~big].sum())
    exp_m = np.append(exp[big], exp[~big].sum())
    if exp_m[-1] == 0:
        obs_m, exp_m = obs_m[:-1], exp_m[:-1]
    assert stats.chisquare(obs_m, exp_m).pvalue > 1e-3


@pytest.mark.parametrize("R", [8, 80, 150, 300])
def test_streaming_geometries(cuda_device, R):
    """The streaming kernel's CTAs per row (8, 4, 2, 1 for these batch sizes on a
    148-SM part) and the cluster kernel's rows in one batch: greedy, small and
    large top-k (several compactions), top-k off with and without top-p (taken
    by the streaming kernel's three-pass path at one CTA per row, R = 300),
    sampled rows vs the oracle."""
    V, S = 151936, 4
    rng = np.random.default_rng(R)
    logits = torch.from_numpy((rng.standard_normal((R, V)) * 1.3).astype(np.float32))
    kinds = np.arange(R) % 5
    T = np.where(kinds == 0, 0.0, rng.uniform(0.3, 1.5, R)).astype(np.float32)
    k = np.choose(kinds, [0, 20, 900, 0, 0]).astype(np.int32)
    p = np.choose(kinds, [1.0, 0.9, 0.95, 0.7, 1.0]).astype(np.float32)
    params = (T, k, p, np.arange(R), np.arange(R) * 7 + 3)
    gpu = run_sampler(logits, params, 99, 20, S, cuda_device)
    rows = sorted(set(np.random.default_rng(1).choice(R, min(R, 12), replace=False).tolist()) | {0, 1, 2, 3, 4})
    compare(gpu, logits.numpy(), params, 99, 20, rows)


def _koff_rows(V, R, rng):
    """Top-k-off top-p rows for the streaming kernel's one-CTA-per-row path: a
    maximum at the end of the row, huge logits (the IEEE quotient instead of
    the fused one), very flat rows (a top-p window larger than the list: the
    cluster kernel takes the row), a cut ~18 units below the maximum, -inf
    mixes, two finite tokens, ties, values on a 5/256 grid, all equal."""
    rows, prm = [], []
    add = lambda l, T, p: (rows.append(np.asarray(l, np.float32)), prm.append((T, p)))
    base = lambda s=1.4: rng.normal(0, s, V).astype(np.float32)
    add(base() + np.linspace(0, 30, V, dtype=np.float32), 0.7, 0.9)      # max at the end
    add(base() + np.linspace(0, 300, V, dtype=np.float32), 1.0, 0.95)    # a steep trend
    add(base() * 1e30, 1.0, 0.9)                                         # |l| > 2^100: the IEEE quotient
    add(base(), 50.0, 0.95)                                              # very flat: window too large
    add(base(1.43), 0.3, 0.99999)                                        # cut ~18 below the max
    add(base(4.0), 0.05, 0.5)                                            # very peaked
    l = base(); l[::3] = -np.inf; add(l, 0.8, 0.8)                       # -inf mixed in
    l = np.full(V, -np.inf, np.float32); l[7] = 1.0; l[V // 2] = 1.5; add(l, 1.0, 0.5)  # two finite
    add(np.round(base() * 4) / 4, 0.9, 0.7)                              # ties
    add(rng.integers(-300, 300, V).astype(np.float32) * np.float32(5 / 256), 1.0, 0.9)  # a coarse grid
    l = base(); l[::5] = 1e-30; add(l, 0.9, 0.8)                         # tiny |l|: the IEEE quotient
    add(np.zeros(V, np.float32), 1.0, 0.5)                               # all equal
    while len(rows) < R:
        add(base(rng.uniform(0.5, 3.0)), float(rng.uniform(0.3, 1.5)), float(rng.uniform(0.3, 0.999)))
    T = np.array([p[0] for p in prm], np.float32)
    p = np.array([p[1] for p in prm], np.float32)
    return np.stack(rows), (T, np.zeros(R, np.int32), p, np.arange(R), np.arange(R) * 5 + 11)


@pytest.mark.parametrize("V,S", [(12000, 4), (151936, 8)])
def test_large_batch_top_k_off_all_rows(cuda_device, V, S):
    """A batch of more rows than SMs, every row top-k off with top_p < 1: the
    streaming kernel's one-CTA-per-row path (both quotients) and the rows it
    passes on, every row (V = 12,000) or 40 rows (V = 151,936) compared with
    the oracle: tokens, thresholds and kept sets, top-n."""
    R = 300
    rng = np.random.default_rng(V)
    logits, params = _koff_rows(V, R, rng)
    gpu = run_sampler(torch.from_numpy(logits), params, 4242, 20, S, cuda_device)
    rows = range(R) if V <= 12000 else sorted(set(range(12)) | set(rng.choice(R, 28, replace=False).tolist()))
    st = compare(gpu, logits, params, 4242, 20, rows)
    assert st["mismatch_allowed"] <= 2


def test_streaming_tie_flood_defers(cuda_device):
    """Rows whose top-k ties overflow the streaming kernel's candidate list (a few
    distinct values over the whole vocabulary) are resolved by the cluster kernel."""
    V, S, R = 151936, 4, 6
    rng = np.random.default_rng(3)
    logits = np.round(rng.standard_normal((R, V)) * 2).astype(np.float32) / 2  # ~16 distinct values
    T = np.full(R, 1.0, np.float32)
    k = np.array([5, 50, 1000, 300, 1, 20], np.int32)
    p = np.array([0.9, 1.0, 0.99, 0.5, 1.0, 0.8], np.float32)
    params = (T, k, p, np.arange(R), np.arange(R))
    gpu = run_sampler(torch.from_numpy(logits), params, 5, 20, S, cuda_device)
    compare(gpu, logits, params, 5, 20, range(R))


def test_deferred_rows_of_a_large_batch(cuda_device):
    """A large batch whose every row floods the streaming kernel's list with ties:
    the cluster kernel's deferred-row pass (a fixed number of clusters, each
    taking every G-th row and, past 256 rows per cluster, a second block of
    marks) samples them all."""
    R, V, S = 9600, 90112, 4
    g = torch.Generator(device=cuda_device)
    g.manual_seed(17)
    # integer logits: the top 1000 of a row reach into a tie of ~5,500 values at 2.0
    logits = torch.round(torch.randn(R, V, generator=g, device=cuda_device))
    T = np.full(R, 1.0, np.float32)
    k = np.full(R, 1000, np.int32)
    p = np.full(R, 0.99, np.float32)
    params = (T, k, p, np.arange(R), np.arange(R))
    gpu = run_sampler(logits, params, 9, 20, S, cuda_device)
    assert np.all(gpu["flags"] == 0)
    assert np.all((gpu["token"] >= 0) & (gpu["token"] < V))
    sel = np.array([0, 1, 36, 37, 500, 4095, 9471, 9472, 9500, R - 1])
    sub = {key: val[sel] for key, val in gpu.items()}
    sub_params = tuple(np.asarray(x)[sel] for x in params)
    del gpu
    compare(sub, logits[torch.from_numpy(sel).to(cuda_device)].cpu().numpy(), sub_params, 9, 20, range(len(sel)))


@pytest.mark.parametrize("requests", [64, 200])
def test_cuda_graph_capture_replays_the_step(cuda_device, requests):
    """The projection and the sampler captured into one CUDA graph (side-by-side
    launches with their fork / join events at 64 rows, the serial pair at 200)
    replay to the same outputs as the eager calls."""
    w = W.scaled(W.WORKLOADS["decode"], V=4 * 4096, requests=requests)
    hidden, ws = W.gemm_inputs(w, cuda_device)
    T, k, p, req, pos = W.row_params(w)
    params = vsl.make_row_params(T, k, p, req, pos, cuda_device)
    logits = [torch.empty(w.R, w.V_s, device=cuda_device) for _ in range(w.S)]
    n = w.n_logprobs

    def fresh():
        return vsl.SampleResult(torch.full((w.R,), -7, dtype=torch.int32, device=cuda_device),
                                torch.zeros(w.R, device=cuda_device),
                                torch.full((w.R, n), -7, dtype=torch.int32, device=cuda_device),
                                torch.zeros(w.R, n, device=cuda_device),
                                torch.full((w.R,), 7, dtype=torch.int32, device=cuda_device))

    eager = fresh()
    vsl.logits_local(hidden, ws, out=logits)
    vsl.sample(logits, params, 21, n, out=eager)
    torch.cuda.synchronize()
    ref_logits = [t.clone() for t in logits]
    for t in logits:
        t.fill_(float("nan"))
    out = fresh()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(cuda_device)
    side.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(side):
        with torch.cuda.graph(g):
            vsl.logits_local(hidden, ws, out=logits)
            vsl.sample(logits, params, 21, n, out=out)
    torch.cuda.current_stream(cuda_device).wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(logits, ref_logits):
        assert torch.equal(a, b)
    for key in ("token_ids", "token_logprob", "topn_ids", "topn_logprob", "row_flags"):
        assert torch.equal(getattr(out, key), getattr(eager, key)), key
    del g
    assert vsl.device_error() == (0, 0)


def test_sample_launch_count(cuda_device):
    """Small batches (at most one row per SM) run the sampler's kernels side by side
    (3 launches), large ones in order (2): the decode and speculative-verify sizes."""
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    assert vsl.sample_launches(64, 4, 37984) == (3 if 64 <= sms else 2)
    assert vsl.sample_launches(64, 8, 31040) == (3 if 64 <= sms else 2)
    assert vsl.sample_launches(512, 4, 37984) == 2
