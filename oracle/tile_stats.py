"""Tile statistics of vocab-sliced logits: per block of 128 ids, the maxima of
its four 32-id quarters, the sum of exp over the block and its smallest finite
logit.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix ("Qwen4Exp batch-sharded sampling: inside vLLM PR #61018",
orcarouter.ai blog, section "batch-sharded sampling in one paragraph"): each
rank computes its own slice of the vocabulary projection, and the sampler then
needs, per row, the softmax statistics and the top candidates of the whole
vocabulary (top-k, top-p, logprobs through ``max_logprobs``).  Producing those
statistics tile by tile, where the projection writes the logits, so that the
sampler reads only what can matter, is this build's reading; the block size,
the record and its layout below are choices of the library, stated here so the
tests can check them:

* slice s of row r holds ids s * V_s + j, j < V_s; block b of the slice holds
  j in [128 b, min(128 b + 128, V_s)) and its quarter q the j in
  [128 b + 32 q, 128 b + 32 q + 32) of the block;
* the record of (row r, slice s, block b) is 8 numbers, stored at record
  index r * (S * B) + s * B + b with B = ceil(V_s / 128):
  [0..3] qmax_q, the largest logit of quarter q (-inf for a quarter with no
         id or only -inf; a quarter holding a NaN has an unspecified qmax);
  [4]    bsum = sum over the block's ids of exp(l_j - c), c the block's
         largest logit when that is finite, else 0 (so a block of -inf sums
         to 0; a NaN makes bsum NaN and +inf makes it +inf);
  [5]    bmin, the smallest finite logit of the block (+inf if none);
  [6]    amin, the smallest |l| over the block's logits that are not NaN
         and not 0 (+inf if none; an infinite logit counts as +inf);
  [7]    0.
Everything is float64 here; the library stores float32 (the maxima and minima
exactly, bsum rounded).
"""
import numpy as np

BLOCK = 128
QUARTER = 32
RECORD = 8


def blocks_per_slice(V_s):
    """B = ceil(V_s / 128) blocks per slice."""
    return -(-int(V_s) // BLOCK)


def block_record(vals):
    """The 8-number record of one block given its logits (at most 128, in id order)."""
    vals = np.asarray(vals, np.float64)
    assert 1 <= vals.size <= BLOCK
    rec = np.zeros(RECORD)
    for q in range(4):
        part = vals[q * QUARTER:(q + 1) * QUARTER]
        part = part[~np.isnan(part)]
        rec[q] = part.max() if part.size else -np.inf
    finite = vals[np.isfinite(vals)]
    top = vals[~np.isnan(vals)].max() if (~np.isnan(vals)).any() else -np.inf
    c = top if np.isfinite(top) else 0.0
    with np.errstate(invalid="ignore", over="ignore"):
        rec[4] = np.sum(np.exp(vals - c))
    rec[5] = finite.min() if finite.size else np.inf
    mag = np.abs(vals[~np.isnan(vals) & (vals != 0.0)])
    rec[6] = mag.min() if mag.size else np.inf
    return rec


def tile_stats(slices):
    """Records of every (row, slice, block): array [R, S * B, 8] (float64).

    slices: S arrays [R, V_s] (the row's vocab slices, in order)."""
    slices = [np.asarray(s, np.float64) for s in slices]
    R, V_s = slices[0].shape
    S = len(slices)
    B = blocks_per_slice(V_s)
    out = np.zeros((R, S * B, RECORD))
    for r in range(R):
        for s in range(S):
            for b in range(B):
                out[r, s * B + b] = block_record(slices[s][r, b * BLOCK:min((b + 1) * BLOCK, V_s)])
    return out


def row_logsumexp(records):
    """log sum_j exp(l_j) of a row from its records [S * B, 8]: the merge of
    the blocks' sums (blocks whose c is 0 because they hold no finite value
    add their bsum as is)."""
    rec = np.asarray(records, np.float64)
    top = rec[:, :4].max(axis=1)
    c = np.where(np.isfinite(top), top, 0.0)
    M = c[np.isfinite(top)].max() if np.isfinite(top).any() else 0.0
    return M + np.log(np.sum(rec[:, 4] * np.exp(c - M)))
