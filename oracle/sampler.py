"""Per-row sampler oracle: temperature, top-k, top-p, Gumbel-max draw, top-n logprobs.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix ("Qwen4Exp batch-sharded sampling: inside vLLM PR #61018",
orcarouter.ai blog, section "batch-sharded sampling in one paragraph"): the
sampler runs top-k and top-p per request over logits of size
batch x (speculative tokens + 1) x vocab, each rank holding a vocab slice, and
logprobs are requested through a non-negative ``max_logprobs``.  Everything
else below is a reading, stated where it is used:

* a row is the concatenation of its S equal, contiguous vocab slices, so the
  token with index j in slice s has global id s * V_s + j;
* temperature: x_i = fl(l_i / T) in float32 with IEEE round-to-nearest
  division (then -0 is read as +0); T == 0 means greedy, which ignores top-k
  and top-p and returns argmax l (lowest id on ties);
* top-k acts on x: theta_k is the k-th largest x (with multiplicity) and
  every x >= theta_k is kept, so ties at the boundary are all kept; k == 0 or
  k >= V means off;
* top-p acts on the top-k survivors K with probabilities renormalised over K:
  p_i = exp(x_i - m) / sum_{j in K} exp(x_j - m), m = max_K x, in float64; i is
  kept iff the mass of strictly greater values, sum_{j in K, x_j > x_i} p_j,
  is < top_p (ties at the cut all kept); top_p >= 1 means off;
* -inf logits are legal and have probability 0: they are never kept or drawn;
* the draw is Gumbel-max: token = argmax over kept i of
  double(x_i) - log(-log(u_i)), u_i from ``oracle.philox.token_uniforms``,
  lowest id on exact ties;
* logprobs are of the raw logits over the full vocabulary:
  lp_i = l_i - (M + log sum_j exp(l_j - M)), float64; top-n lists the n
  largest raw logits, lower id first on ties, sorted descending;
* a row with a NaN or +inf logit, with every logit -inf, or with an invalid
  parameter (T < 0, T NaN or inf, top_p <= 0 or NaN, top_k < 0), or whose
  l / T overflows float32, is flagged and returns token -1, NaN logprobs and
  top-n ids -1.
"""
from dataclasses import dataclass, field

import numpy as np

from .philox import token_uniforms

FLAG_NONFINITE = 1 << 0
FLAG_ALL_NEG_INF = 1 << 1
FLAG_BAD_TEMPERATURE = 1 << 2
FLAG_BAD_TOP_P = 1 << 3
FLAG_BAD_TOP_K = 1 << 4
FLAG_SCALE_OVERFLOW = 1 << 5

# Two perturbed scores closer than this (relative) may legitimately be ordered
# differently by a float32 evaluation of the Gumbel scores.
NEAR_TIE_REL = 1e-6
# A top-p cut whose boundary mass lies this close to top_p depends on the
# summation order of up to 2**18 float64 terms (worst case n * 2**-53 < 3e-11).
CUT_TIE_ABS = 1e-10


@dataclass
class RowResult:
    token: int
    token_logprob: float
    topn_ids: np.ndarray
    topn_logprob: np.ndarray
    flags: int
    kept: np.ndarray = None          # bool mask over V of the kept set (sampling rows)
    theta_k: float = None            # top-k threshold on x (None when off)
    theta_p: float = None            # top-p threshold on x (None when off)
    near_tie: bool = False           # top two perturbed scores within NEAR_TIE_REL
    cut_tie: bool = False            # top-p boundary mass within CUT_TIE_ABS of top_p
    score_gap: float = float("inf")  # relative gap between the two best scores
    cut_margin: float = float("inf")
    extra: dict = field(default_factory=dict)


def scale(l, temperature):
    """x = fl(l / T) in float32 (IEEE round-to-nearest), with -0 read as +0."""
    l32 = np.asarray(l, dtype=np.float32)
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        x = l32 / np.float32(temperature)
    return (x + np.float32(0.0)).astype(np.float32)


def validate(l, temperature, top_k, top_p):
    """Row flags for non-finite data, all -inf rows and invalid parameters."""
    l32 = np.asarray(l, dtype=np.float32)
    flags = 0
    if np.any(np.isnan(l32)) or np.any(l32 == np.inf):
        flags |= FLAG_NONFINITE
    elif np.all(l32 == -np.inf):
        flags |= FLAG_ALL_NEG_INF
    t = np.float32(temperature)
    if not (np.isfinite(t) and t >= 0):
        flags |= FLAG_BAD_TEMPERATURE
    if not (np.float32(top_p) > 0):          # NaN compares False
        flags |= FLAG_BAD_TOP_P
    if top_k < 0:
        flags |= FLAG_BAD_TOP_K
    if flags == 0 and t > 0:
        finite = np.isfinite(l32)
        x = scale(l32[finite], t)
        if np.any(np.isinf(x)):
            flags |= FLAG_SCALE_OVERFLOW
    return flags


def log_softmax(l):
    """lp_i = l_i - (M + log sum_j exp(l_j - M)) over the finite logits, float64."""
    l64 = np.asarray(l, dtype=np.float32).astype(np.float64)
    finite = np.isfinite(l64)
    M = l64[finite].max()
    lse = M + np.log(np.sum(np.exp(l64[finite] - M)))
    return l64 - lse


def top_n(l, n):
    """Ids of the n largest raw logits, descending, lower id first on ties."""
    l32 = np.asarray(l, dtype=np.float32)
    ids = np.arange(l32.size)
    order = np.lexsort((ids, -l32.astype(np.float64)))
    return order[:n]


def top_k_threshold(x, k):
    """theta_k = the k-th largest value of x, counted with multiplicity."""
    return np.sort(x)[::-1][k - 1]


def top_p_threshold(xk, top_p):
    """Smallest kept value of the top-p rule over the survivor values ``xk``.

    Returns (theta_p, margin): margin is the distance of the boundary masses
    from top_p (the kept side below it, the dropped side at or above it).
    """
    xk = np.asarray(xk, dtype=np.float32)
    desc = np.sort(xk)[::-1]
    m = np.float64(desc[0])
    e = np.exp(desc.astype(np.float64) - m)
    Z = np.sum(e)
    p = e / Z
    csum = np.concatenate([[0.0], np.cumsum(p)])
    # mass of values strictly greater than desc[j]: the prefix up to the
    # first occurrence of desc[j] in the descending order
    first = np.searchsorted(-desc.astype(np.float64), -desc.astype(np.float64), side="left")
    mass_gt = csum[first]
    kept = mass_gt < np.float64(np.float32(top_p))
    theta_p = desc[kept].min()
    tp = np.float64(np.float32(top_p))
    margin = tp - mass_gt[kept].max()
    if np.any(~kept):
        margin = min(margin, mass_gt[~kept].min() - tp)
    return theta_p, margin


def gumbel_scores(x, ids, request_id, position, seed):
    """double(x_i) - log(-log(u_i)) for the given token ids, float64."""
    u = token_uniforms(ids, request_id, position, seed)
    g = -np.log(-np.log(u))
    return np.asarray(x, dtype=np.float32).astype(np.float64) + g


def sample_row(l, temperature, top_k, top_p, request_id, position, seed, n_logprobs):
    """Sample one row of raw logits ``l`` (float32, length V) by the rules above."""
    l = np.asarray(l, dtype=np.float32)
    V = l.size
    flags = validate(l, temperature, top_k, top_p)
    if flags:
        return RowResult(token=-1, token_logprob=float("nan"),
                         topn_ids=np.full(n_logprobs, -1, np.int64),
                         topn_logprob=np.full(n_logprobs, np.nan), flags=flags)
    lp = log_softmax(l)
    tn = top_n(l, n_logprobs)
    res = RowResult(token=-1, token_logprob=0.0, topn_ids=tn.astype(np.int64),
                    topn_logprob=lp[tn], flags=0)
    finite = np.isfinite(l)
    if np.float32(temperature) == 0:
        token = int(np.argmax(l))            # first maximum = lowest id
        res.token, res.token_logprob = token, float(lp[token])
        return res
    x = scale(l, temperature)
    keep = finite.copy()
    if 0 < top_k < V:
        res.theta_k = top_k_threshold(x, top_k)
        keep &= x >= res.theta_k
    if np.float32(top_p) < 1:
        res.theta_p, res.cut_margin = top_p_threshold(x[keep], top_p)
        res.cut_tie = bool(res.cut_margin < CUT_TIE_ABS)
        keep &= x >= res.theta_p
    ids = np.nonzero(keep)[0]
    s = gumbel_scores(x[ids], ids, request_id, position, seed)
    j = int(np.argmax(s))                    # first maximum = lowest id
    token = int(ids[j])
    if s.size > 1:
        top2 = np.sort(s)[-2:]
        gap = (top2[1] - top2[0]) / max(abs(top2[0]), abs(top2[1]), 1e-300)
        res.score_gap = float(gap)
        res.near_tie = bool(gap <= NEAR_TIE_REL)
    res.kept = keep
    res.token, res.token_logprob = token, float(lp[token])
    return res


@dataclass
class ProcessedResult:
    kept: np.ndarray          # bool mask over V of the set the draw is over
    logprob: np.ndarray       # float64 over V: log q_i on the kept set, -inf elsewhere
    topn_ids: np.ndarray      # n ids, -1 past the kept set
    topn_logprob: np.ndarray  # n values, -inf past the kept set
    flags: int


def processed_logprobs(l, temperature, top_k, top_p, n):
    """Log-probabilities of the distribution the token is drawn from (the
    "processed" logprobs, after temperature, top-k and top-p).

    Readings (the pages only name logprobs; these restate what the draw above
    samples from): for a sampling row the kept set K is the draw's (the same
    top-k and top-p rules), q_i = exp(x_i - m) / sum_{j in K} exp(x_j - m) with
    m = max_K x, in float64, and log q_i = -inf outside K; a greedy row draws
    its argmax with certainty, so its kept set is that one token with log q
    = 0.  The top-n lists the n largest log q (the n largest x of K), lower id
    first on equal x, then (-1, -inf) once K is exhausted.  A flagged row gets
    NaN values and ids -1, as for the raw logprobs.
    """
    l = np.asarray(l, dtype=np.float32)
    V = l.size
    flags = validate(l, temperature, top_k, top_p)
    if flags:
        return ProcessedResult(np.zeros(V, bool), np.full(V, np.nan), np.full(n, -1, np.int64),
                               np.full(n, np.nan), flags)
    lp = np.full(V, -np.inf)
    keep = np.zeros(V, bool)
    if np.float32(temperature) == 0:
        token = int(np.argmax(l))            # first maximum = lowest id
        keep[token] = True
        lp[token] = 0.0
        x = l
    else:
        x = scale(l, temperature)
        keep = np.isfinite(l).copy()
        if 0 < top_k < V:
            keep &= x >= top_k_threshold(x, top_k)
        if np.float32(top_p) < 1:
            theta_p, _ = top_p_threshold(x[keep], top_p)
            keep &= x >= theta_p
        xk = x[keep].astype(np.float64)
        m = xk.max()
        lp[keep] = (xk - m) - np.log(np.sum(np.exp(xk - m)))
    ids = np.nonzero(keep)[0]
    order = ids[np.lexsort((ids, -x[ids].astype(np.float64)))]
    take = order[:n]
    topn_ids = np.full(n, -1, np.int64)
    topn_lp = np.full(n, -np.inf)
    topn_ids[:take.size] = take
    topn_lp[:take.size] = lp[take]
    return ProcessedResult(keep, lp, topn_ids, topn_lp, 0)


def sample_rows(logits, params, seed, n_logprobs, rows=None):
    """Apply ``sample_row`` to each selected row of a (R, V) float32 array.

    ``params`` is a sequence of (temperature, top_k, top_p, request_id,
    position) tuples, one per row.  Returns a list of RowResult.
    """
    logits = np.asarray(logits, dtype=np.float32)
    rows = range(logits.shape[0]) if rows is None else rows
    out = []
    for r in rows:
        T, k, p, req, pos = params[r]
        out.append(sample_row(logits[r], T, k, p, req, pos, seed, n_logprobs))
    return out
