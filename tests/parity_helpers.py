"""Shared checks of the CUDA sampler against the oracle, row by row."""
import os

import numpy as np
import torch

import vocab_sharded_logits_b200 as vsl
from oracle import sampler as S

LOGPROB_TOL = 1e-4      # raw logprobs: fp32 online log-sum-exp vs float64
LOGIT_TOL = 2e-2        # projection: bf16 inputs, fp32 accumulation vs float64

# per-test counts of the allowed exceptions, printed in pytest's terminal summary
REPORT = []


def run_sampler(logits, params_np, seed, n, S_slices, device, tiles=False):
    """Runs the CUDA sampler on [R, V] fp32 logits split into S_slices slices,
    with the kept-set thresholds requested (tiles: with the tile statistics of
    the logits, from the library's statistics kernel)."""
    T, k, p, req, pos = params_np
    slices = [t.contiguous() for t in torch.tensor_split(logits.to(device), S_slices, dim=1)]
    prm = vsl.make_row_params(T, k, p, req, pos, device)
    stats = vsl.tile_stats(slices) if tiles else None
    out = vsl.sample(slices, prm, seed, n, processed=True, tile_stats=stats)
    torch.cuda.synchronize()
    return {
        "p_token": out.processed_logprob.cpu().numpy(),
        "p_topn_ids": out.processed_topn_ids.cpu().numpy(),
        "p_topn_lp": out.processed_topn_logprob.cpu().numpy(),
        "token": out.token_ids.cpu().numpy(),
        "token_lp": out.token_logprob.cpu().numpy(),
        "topn_ids": out.topn_ids.cpu().numpy(),
        "topn_lp": out.topn_logprob.cpu().numpy(),
        "flags": out.row_flags.cpu().numpy().astype(np.uint32),
        "theta": out.kept_theta.cpu().numpy(),
    }


def _expected_theta(v):
    return np.float32(-np.inf) if v is None else np.float32(v)


def compare(gpu, logits_np, params_np, seed, n, rows):
    """Element-by-element comparison on ``rows``: flags, top-n ids (exact) and
    logprobs (1e-4), the kept-set thresholds theta_k and theta_p (bit-exact) and
    the kept set they define (every element), the token (exact), and the
    processed logprobs (the token's and the top-n's: ids exact, values 1e-4).
    Returns counts of the allowed exceptions: near-ties of the draw (the token
    only) and cut-ties of top-p (theta_p, the kept set, the token and the
    processed logprobs)."""
    T, k, p, req, pos = params_np
    stats = {"rows": 0, "near_tie": 0, "cut_tie": 0, "mismatch_allowed": 0, "kept_checked": 0}
    for r in rows:
        o = S.sample_row(logits_np[r], T[r], int(k[r]), p[r], int(req[r]), int(pos[r]), seed, n)
        stats["rows"] += 1
        th = gpu["theta"][r]
        assert int(gpu["flags"][r]) == o.flags, (r, gpu["flags"][r], o.flags)
        if o.flags:
            assert gpu["token"][r] == -1 and np.isnan(gpu["token_lp"][r])
            assert np.isnan(th).all(), (r, th)
            assert np.isnan(gpu["p_token"][r])
            if n:
                assert np.all(gpu["topn_ids"][r] == -1)
                assert np.all(gpu["p_topn_ids"][r] == -1) and np.isnan(gpu["p_topn_lp"][r]).all()
            continue
        if n:
            assert np.array_equal(gpu["topn_ids"][r], o.topn_ids), (r, gpu["topn_ids"][r], o.topn_ids)
            assert np.allclose(gpu["topn_lp"][r], o.topn_logprob, atol=LOGPROB_TOL, rtol=0), r
        stats["near_tie"] += int(o.near_tie)
        stats["cut_tie"] += int(o.cut_tie)
        if np.float32(T[r]) == 0:
            assert np.isnan(th).all(), (r, th)          # greedy: no kept set
        else:
            assert th[0] == _expected_theta(o.theta_k), (r, "theta_k", th[0], o.theta_k)
            if not o.cut_tie:
                assert th[1] == _expected_theta(o.theta_p), (r, "theta_p", th[1], o.theta_p)
                l = logits_np[r]
                x = S.scale(l, T[r])
                kept = np.isfinite(l) & (x >= max(th[0], th[1]))
                assert np.array_equal(kept, o.kept), (r, int(kept.sum()), int(o.kept.sum()))
                stats["kept_checked"] += 1
        tok = int(gpu["token"][r])
        if tok != o.token:
            assert o.near_tie or o.cut_tie, (r, tok, o.token, o.score_gap, o.cut_margin)
            stats["mismatch_allowed"] += 1
            # the GPU's token must still be a valid draw: inside the kept set
            if o.kept is not None:
                assert o.kept[tok]
        ref_lp = S.log_softmax(logits_np[r])[tok]
        assert abs(float(gpu["token_lp"][r]) - ref_lp) <= LOGPROB_TOL, (r, gpu["token_lp"][r], ref_lp)
        if not o.cut_tie:
            pr = S.processed_logprobs(logits_np[r], T[r], int(k[r]), p[r], n)
            assert abs(float(gpu["p_token"][r]) - pr.logprob[tok]) <= LOGPROB_TOL, (r, gpu["p_token"][r], pr.logprob[tok])
            if n:
                assert np.array_equal(gpu["p_topn_ids"][r], pr.topn_ids), (r, gpu["p_topn_ids"][r], pr.topn_ids)
                got, want = gpu["p_topn_lp"][r].astype(np.float64), pr.topn_logprob
                assert np.array_equal(np.isinf(got), np.isinf(want)), r
                fin = np.isfinite(want)
                assert np.allclose(got[fin], want[fin], atol=LOGPROB_TOL, rtol=0), r
    REPORT.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], dict(stats)))
    return stats
