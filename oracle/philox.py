"""Philox4x32-10 counter-based generator, restated from its published description.

Source: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel Random
Numbers: As Easy as 1, 2, 3", SC'11.  Section 3.2 defines the Philox S-box
(two 32x32 -> 64-bit multiplies whose high halves are xored with the other
counter words and the round key, with a word permutation) and the Weyl key
schedule; Table 2 gives the Philox-4x32 multipliers.  The key increments are
the golden-ratio and sqrt(3)-1 Weyl constants the paper names for 32-bit words.

Test infrastructure only (see ``oracle/__init__.py``).
"""
import numpy as np

# Table 2 (Philox-4x32 round multipliers) and the 32-bit Weyl constants.
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9  # golden ratio, (sqrt(5) - 1) / 2 * 2**32
PHILOX_W1 = 0xBB67AE85  # sqrt(3) - 1, * 2**32
ROUNDS = 10

_MASK32 = np.uint64(0xFFFFFFFF)


def _mulhilo(a, b):
    """32x32 -> 64-bit product of uint32 arrays, returned as (hi, lo) uint32."""
    prod = a.astype(np.uint64) * np.uint64(b)
    return (prod >> np.uint64(32)).astype(np.uint32), (prod & _MASK32).astype(np.uint32)


def philox4x32(ctr, key, rounds=ROUNDS):
    """Apply Philox4x32-``rounds`` to counters ``ctr`` under ``key``.

    ctr: array-like of shape (..., 4) of uint32 words (c0, c1, c2, c3).
    key: array-like of shape (..., 2) of uint32 words (k0, k1), broadcastable.
    Returns a uint32 array of shape (..., 4).

    One round maps (c0, c1, c2, c3) under key (k0, k1) to
        (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0));
    the key is bumped by the Weyl constants between rounds.
    """
    ctr = np.asarray(ctr, dtype=np.uint32)
    key = np.asarray(key, dtype=np.uint32)
    c0, c1, c2, c3 = (ctr[..., i].copy() for i in range(4))
    k0 = np.broadcast_to(key[..., 0], c0.shape).astype(np.uint64)
    k1 = np.broadcast_to(key[..., 1], c0.shape).astype(np.uint64)
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        hi0, lo0 = _mulhilo(c0, PHILOX_M0)
        hi1, lo1 = _mulhilo(c2, PHILOX_M1)
        k0_32 = k0.astype(np.uint32)
        k1_32 = k1.astype(np.uint32)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0_32, lo1, hi0 ^ c3 ^ k1_32, lo0
    return np.stack([c0, c1, c2, c3], axis=-1)


def token_uniforms(token_ids, request_id, position, seed):
    """Uniform u in (0, 1) for global token ids of one row, as float64.

    Reading (the pages give no RNG; the keying is the one the draw is specified
    with): key = (seed mod 2**32, seed >> 32); counter =
    (floor(i / 4), position, request_id, 0); the word with index i mod 4 is
    taken, and u = ((word >> 9) + 0.5) * 2**-23: a 23-bit integer plus one half
    has 24 significant bits, so u is exact in float32 (as is 1 - u) and lies
    strictly inside (0, 1), in [2**-24, 1 - 2**-24].  ``token_ids``, ``request_id`` and
    ``position`` broadcast against each other.
    """
    ids, req, pos = np.broadcast_arrays(np.asarray(token_ids, dtype=np.int64),
                                        np.asarray(request_id, dtype=np.int64),
                                        np.asarray(position, dtype=np.int64))
    seed = int(seed)
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint32)
    ctr = np.zeros(ids.shape + (4,), dtype=np.uint32)
    ctr[..., 0] = (ids // 4).astype(np.uint32)
    ctr[..., 1] = (pos & 0xFFFFFFFF).astype(np.uint32)
    ctr[..., 2] = (req & 0xFFFFFFFF).astype(np.uint32)
    words = philox4x32(ctr, key)
    w = np.take_along_axis(words, (ids % 4)[..., None], axis=-1)[..., 0]
    return ((w >> np.uint32(9)).astype(np.float64) + 0.5) * 2.0 ** -23
