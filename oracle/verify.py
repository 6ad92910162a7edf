"""Speculative verification oracle: acceptance of deterministic draft tokens.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix ("Qwen4Exp batch-sharded sampling: inside vLLM PR #61018",
orcarouter.ai blog): the sampler runs over batch x (speculative tokens + 1) x
vocab logits (section "batch-sharded sampling in one paragraph"), the gain is
measured in requests per second and acceptance length (section "the 1.5 %
estimate"), and sharded draft logits are left as future work (section
"batch-sharded sampling in one paragraph").  Everything else below is a
reading, stated where it is used:

* a request has spec draft tokens d_0 .. d_{spec-1} proposed for positions
  0 .. spec - 1 and spec + 1 target rows; row j holds the target's draw t_j
  for position j (the sampler's token, -1 for a flagged row);
* the drafts are deterministic (a draft distribution that is a point mass on
  d_j: no draft logits, which the pages leave for later);
* draft j is accepted iff every earlier draft was accepted and t_j == d_j; the
  number accepted is a, and the request emits d_0 .. d_{a-1} followed by t_a
  (the correction when a < spec, the bonus token when a == spec), then -1.

With the draw keyed by (seed, request, position, token), accepting iff the
target's own draw equals the draft is the speculative-sampling rejection test
for a point-mass draft: the draft is accepted with probability p(d_j) (p the
distribution the draw samples, after temperature, top-k and top-p) and on
rejection the emitted token is distributed as p restricted to tokens != d_j,
renormalised, so each emitted token is distributed as p
(``tests/test_oracle_verify.py`` checks both by sampling).
"""
import numpy as np


def verify_request(target, drafts):
    """Accepted count and emitted tokens of one request.

    target: spec + 1 target tokens t_0 .. t_spec; drafts: spec draft tokens.
    Returns (a, out) with out of length spec + 1: d_0 .. d_{a-1}, t_a, then -1.
    """
    target = [int(t) for t in target]
    drafts = [int(d) for d in drafts]
    spec = len(drafts)
    assert len(target) == spec + 1
    a = 0
    while a < spec and target[a] >= 0 and target[a] == drafts[a]:
        a += 1
    out = drafts[:a] + [target[a]] + [-1] * (spec - a)
    return a, out


def verify(target_ids, draft_ids, logprobs=None):
    """All requests: target_ids [requests * (spec + 1)] (row-major by request),
    draft_ids [requests, spec], optional per-row logprobs [requests * (spec + 1)].
    Returns (accepted [requests], out_ids [requests, spec + 1], out_logprob or None)
    with out_logprob[q, j] the logprob of row j's token for j <= a, NaN after."""
    draft_ids = np.asarray(draft_ids)
    assert draft_ids.ndim == 2, "draft_ids is [requests, spec]"
    nreq, spec = draft_ids.shape
    target_ids = np.asarray(target_ids).reshape(nreq, spec + 1)
    acc = np.zeros(nreq, np.int64)
    out = np.full((nreq, spec + 1), -1, np.int64)
    olp = None
    if logprobs is not None:
        lp = np.asarray(logprobs, np.float64).reshape(nreq, spec + 1)
        olp = np.full((nreq, spec + 1), np.nan)
    for q in range(nreq):
        a, o = verify_request(target_ids[q], draft_ids[q])
        acc[q] = a
        out[q] = o
        if olp is not None:
            olp[q, :a + 1] = lp[q, :a + 1]
    return acc, out, olp
