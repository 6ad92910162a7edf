"""Parity of the CUDA speculative verification (vsl_verify_drafts) with the
oracle (oracle/verify.py), bit for bit: on random target / draft arrays with
matches planted at every position, and end to end on the sampler's own draws
for the speculative-verify recipe (drafts equal to the draws, then each
position changed in turn)."""
import numpy as np
import pytest
import torch

import vocab_sharded_logits_b200 as vsl
import workloads as W
from oracle.verify import verify

pytestmark = pytest.mark.gpu


def _run(tokens, drafts, lps, device):
    t = torch.from_numpy(np.ascontiguousarray(tokens, np.int32)).to(device)
    d = torch.from_numpy(np.ascontiguousarray(drafts, np.int32)).to(device)
    lp = torch.from_numpy(np.ascontiguousarray(lps, np.float32)).to(device) if lps is not None else None
    out = vsl.verify_drafts(t, d, lp)
    torch.cuda.synchronize()
    return (out.accepted.cpu().numpy(), out.out_ids.cpu().numpy(),
            out.out_logprob.cpu().numpy() if lp is not None else None)


@pytest.mark.parametrize("spec,requests", [(0, 5), (1, 33), (3, 128), (7, 256), (64, 40)])
def test_random_arrays_match_the_oracle(cuda_device, spec, requests):
    rng = np.random.default_rng(spec * 1000 + requests)
    drafts = rng.integers(0, 50, (requests, spec)).astype(np.int32)
    target = rng.integers(0, 50, (requests, spec + 1)).astype(np.int32)
    # plant a prefix of matches of every length, and flagged rows
    for q in range(requests):
        a = int(rng.integers(0, spec + 1))
        target[q, :a] = drafts[q, :a]
        if rng.random() < 0.1:
            target[q, int(rng.integers(0, spec + 1))] = -1
    lps = rng.normal(size=(requests, spec + 1)).astype(np.float32)
    acc, out, olp = _run(target.reshape(-1), drafts, lps.reshape(-1), cuda_device)
    racc, rout, rolp = verify(target.reshape(-1), drafts, lps.reshape(-1).astype(np.float64))
    assert np.array_equal(acc, racc)
    assert np.array_equal(out, rout)
    assert np.array_equal(np.isnan(olp), np.isnan(rolp))
    assert np.array_equal(olp[~np.isnan(olp)], rolp[~np.isnan(rolp)].astype(np.float32))
    acc2, out2, _ = _run(target.reshape(-1), drafts, None, cuda_device)   # without logprobs
    assert np.array_equal(acc2, racc) and np.array_equal(out2, rout)


def test_end_to_end_on_the_samplers_draws(cuda_device):
    """The speculative-verify recipe (4 rows per request) at a small vocabulary:
    the sampler draws every row; drafts equal to the draws are all accepted,
    and changing draft j stops acceptance at j and emits the draw there."""
    w = W.scaled(W.WORKLOADS["spec"], V=4 * 2048, requests=32)
    logits = W.sampler_logits(w, cuda_device)
    T, k, p, req, pos = W.row_params(w)
    slices = [t.contiguous() for t in torch.tensor_split(logits, w.S, dim=1)]
    res = vsl.sample(slices, vsl.make_row_params(T, k, p, req, pos, cuda_device), 21, w.n_logprobs)
    spec = w.rows_per_request - 1
    toks = res.token_ids.view(w.requests, spec + 1)
    lps = res.token_logprob
    drafts = toks[:, :spec].contiguous().clone()
    for j in [None] + list(range(spec)):
        d = drafts.clone()
        if j is not None:
            d[:, j] = (d[:, j] + 1) % w.V
        out = vsl.verify_drafts(res.token_ids, d, lps)
        torch.cuda.synchronize()
        racc, rout, rolp = verify(res.token_ids.cpu().numpy(), d.cpu().numpy(), lps.cpu().numpy())
        assert np.array_equal(out.accepted.cpu().numpy(), racc)
        assert np.array_equal(out.out_ids.cpu().numpy(), rout)
        assert (racc == (spec if j is None else j)).all()
        got_lp = out.out_logprob.cpu().numpy()
        assert np.array_equal(np.isnan(got_lp), np.isnan(rolp))
