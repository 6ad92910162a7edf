"""Pins of the speculative-verification oracle (oracle/verify.py): closed
forms, an independent formulation on random cases, and sampling checks that
accepting a draft iff the target's own draw equals it is the rejection rule
for a point-mass draft (acceptance probability p(d), and on rejection the
token distributed as p without d, renormalised)."""
import numpy as np
import pytest
from scipy import stats

from oracle import sampler as S
from oracle.verify import verify, verify_request


def test_all_accepted_emits_drafts_and_the_bonus_token():
    a, out = verify_request([5, 7, 9, 11], [5, 7, 9])
    assert a == 3 and out == [5, 7, 9, 11]


@pytest.mark.parametrize("j", [0, 1, 2])
def test_first_mismatch_emits_the_correction_then_nothing(j):
    drafts = [5, 7, 9]
    target = [5, 7, 9, 11]
    target[j] = 100 + j
    a, out = verify_request(target, drafts)
    assert a == j
    assert out == drafts[:j] + [100 + j] + [-1] * (3 - j)


def test_a_flagged_target_row_stops_acceptance():
    a, out = verify_request([5, -1, 9, 11], [5, -1, 9])  # a draft of -1 never matches
    assert a == 1 and out == [5, -1, -1, -1]


def test_no_speculative_tokens():
    assert verify_request([42], []) == (0, [42])


def test_independent_formulation_on_random_cases():
    rng = np.random.default_rng(0)
    for _ in range(300):
        spec = int(rng.integers(0, 9))
        nreq = int(rng.integers(1, 6))
        drafts = rng.integers(0, 4, (nreq, spec))
        target = rng.integers(-1, 4, (nreq, spec + 1))
        lp = rng.normal(size=(nreq, spec + 1))
        acc, out, olp = verify(target.reshape(-1), drafts, lp.reshape(-1))
        for q in range(nreq):
            eq = (target[q, :spec] == drafts[q]) & (target[q, :spec] >= 0)
            a = int(np.cumprod(eq).sum()) if spec else 0
            assert acc[q] == a
            want = np.concatenate([drafts[q, :a], target[q, a:a + 1], np.full(spec - a, -1)])
            assert np.array_equal(out[q], want)
            assert np.allclose(olp[q, :a + 1], lp[q, :a + 1]) and np.isnan(olp[q, a + 1:]).all()


def _p(l, T, k, p):
    return np.exp(S.processed_logprobs(l, T, k, p, 0).logprob)


def test_acceptance_is_the_rejection_rule_for_a_point_mass_draft():
    """Over many positions (independent Philox counters), the draft is accepted
    with frequency p(d) and the rejected draws follow p without d."""
    rng = np.random.default_rng(7)
    V = 10
    l = rng.normal(0, 1.2, V).astype(np.float32)
    T, k, p = 0.9, 8, 0.95
    prob = _p(l, T, k, p)
    d = int(np.argsort(prob)[-2])          # the second most likely token as the draft
    n = 20000
    draws = np.array([S.sample_row(l, T, k, p, 3, pos, 11, 0).token for pos in range(n)])
    accepted = [verify_request([t, -1], [d])[0] for t in draws]
    assert stats.binomtest(int(np.sum(accepted)), n, prob[d]).pvalue > 1e-3
    rej = draws[draws != d]
    q = prob.copy()
    q[d] = 0.0
    q /= q.sum()
    support = q > 0
    obs = np.bincount(rej, minlength=V)[support]
    assert np.bincount(rej, minlength=V)[~support].sum() == 0
    assert stats.chisquare(obs, q[support] * rej.size).pvalue > 1e-3


def test_two_drafts_are_accepted_with_the_product_of_their_probabilities():
    """Positions 0 and 1 draw with independent counters: P(a = 2) = p0(d0) p1(d1)."""
    rng = np.random.default_rng(8)
    V = 8
    l0 = rng.normal(0, 1.0, V).astype(np.float32)
    l1 = rng.normal(0, 1.0, V).astype(np.float32)
    p0, p1 = _p(l0, 1.0, 0, 0.9), _p(l1, 0.7, 0, 1.0)
    d0, d1 = int(np.argmax(p0)), int(np.argmax(p1))
    n = 12000
    full = 0
    for r in range(n):
        t0 = S.sample_row(l0, 1.0, 0, 0.9, r, 0, 5, 0).token
        t1 = S.sample_row(l1, 0.7, 0, 1.0, r, 1, 5, 0).token
        a, _ = verify_request([t0, t1, 0], [d0, d1])
        full += a == 2
    assert stats.binomtest(full, n, p0[d0] * p1[d1]).pvalue > 1e-3
