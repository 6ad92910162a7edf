"""Vocab-slice projection oracle: each slice's logits with no gather.

Test infrastructure only (see ``oracle/__init__.py``).

Definition ("Qwen4Exp batch-sharded sampling: inside vLLM PR #61018",
orcarouter.ai blog, sections "batch-sharded sampling in one paragraph" and
"why three lines were the whole job"): a rank computes only its own slice of
the vocabulary projection and never gathers the full vocabulary, i.e. for
slice s with weight rows W_s (V_s x H, nn.Linear out x in):

    logits_s[r, j] = sum_h hidden[r, h] * W_s[j, h].

Inputs are the bfloat16 values the kernel consumes, passed here as float32 or
float64 arrays holding exactly those values; the sum is taken in float64 by
a library matrix product (no blocking or reordering of our own).
"""
import numpy as np


def logits_local(hidden, w_slices):
    """Return the list of float64 logits slices [R, V_s], one per weight slice."""
    h = np.asarray(hidden, dtype=np.float64)
    return [h @ np.asarray(w, dtype=np.float64).T for w in w_slices]


def logits_local_entries(hidden, w_slice, rows, cols):
    """logits_s[rows[i], cols[j]] for a row subset x column subset, float64."""
    h = np.asarray(hidden, dtype=np.float64)[np.asarray(rows)]
    w = np.asarray(w_slice, dtype=np.float64)[np.asarray(cols)]
    return h @ w.T
