"""Shared checks of the CUDA sampler against the oracle, row by row."""
import numpy as np
import torch

import vocab_sharded_logits_b200 as vsl
from oracle import sampler as S

LOGPROB_TOL = 1e-4      # raw logprobs: fp32 online log-sum-exp vs float64
LOGIT_TOL = 2e-2        # projection: bf16 inputs, fp32 accumulation vs float64


def run_sampler(logits, params_np, seed, n, S_slices, device):
    """Runs the CUDA sampler on [R, V] fp32 logits split into S_slices slices."""
    T, k, p, req, pos = params_np
    slices = [t.contiguous() for t in torch.tensor_split(logits.to(device), S_slices, dim=1)]
    prm = vsl.make_row_params(T, k, p, req, pos, device)
    out = vsl.sample(slices, prm, seed, n)
    torch.cuda.synchronize()
    return {
        "token": out.token_ids.cpu().numpy(),
        "token_lp": out.token_logprob.cpu().numpy(),
        "topn_ids": out.topn_ids.cpu().numpy(),
        "topn_lp": out.topn_logprob.cpu().numpy(),
        "flags": out.row_flags.cpu().numpy().astype(np.uint32),
    }


def compare(gpu, logits_np, params_np, seed, n, rows):
    """Element-by-element comparison on ``rows``; returns counts of the
    allowed exceptions (near-ties of the draw, cut-ties of top-p)."""
    T, k, p, req, pos = params_np
    stats = {"rows": 0, "near_tie": 0, "cut_tie": 0, "mismatch_allowed": 0}
    for r in rows:
        o = S.sample_row(logits_np[r], T[r], int(k[r]), p[r], int(req[r]), int(pos[r]), seed, n)
        stats["rows"] += 1
        assert int(gpu["flags"][r]) == o.flags, (r, gpu["flags"][r], o.flags)
        if o.flags:
            assert gpu["token"][r] == -1 and np.isnan(gpu["token_lp"][r])
            if n:
                assert np.all(gpu["topn_ids"][r] == -1)
            continue
        if n:
            assert np.array_equal(gpu["topn_ids"][r], o.topn_ids), (r, gpu["topn_ids"][r], o.topn_ids)
            assert np.allclose(gpu["topn_lp"][r], o.topn_logprob, atol=LOGPROB_TOL, rtol=0), r
        stats["near_tie"] += int(o.near_tie)
        stats["cut_tie"] += int(o.cut_tie)
        tok = int(gpu["token"][r])
        if tok != o.token:
            assert o.near_tie or o.cut_tie, (r, tok, o.token, o.score_gap, o.cut_margin)
            stats["mismatch_allowed"] += 1
            # the GPU's token must still be a valid draw: inside the kept set
            if o.kept is not None:
                assert o.kept[tok]
        ref_lp = S.log_softmax(logits_np[r])[tok]
        assert abs(float(gpu["token_lp"][r]) - ref_lp) <= LOGPROB_TOL, (r, gpu["token_lp"][r], ref_lp)
    return stats
