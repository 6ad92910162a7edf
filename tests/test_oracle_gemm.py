"""Pins for the projection oracle: exact integer products, a transposition
check, slice independence and a brute-force triple loop."""
import numpy as np

from oracle.gemm import logits_local, logits_local_entries


def test_integer_inputs_are_exact():
    rng = np.random.default_rng(0)
    h = rng.integers(-4, 5, (7, 96))
    w = [rng.integers(-4, 5, (40, 96)) for _ in range(3)]
    got = logits_local(h.astype(np.float32), [x.astype(np.float32) for x in w])
    for g, ws in zip(got, w):
        assert np.array_equal(g, (h @ ws.T).astype(np.float64))


def test_identity_hidden_returns_weight_transpose():
    H = 32
    rng = np.random.default_rng(1)
    w = rng.normal(size=(10, H)).astype(np.float32)
    out = logits_local(np.eye(H, dtype=np.float32), [w])[0]
    assert out.shape == (H, 10)
    assert np.array_equal(out, w.T.astype(np.float64))


def test_slices_are_column_blocks_of_the_full_projection():
    rng = np.random.default_rng(2)
    h = rng.normal(size=(5, 24))
    W = rng.normal(size=(36, 24))
    full = logits_local(h, [W])[0]
    parts = logits_local(h, [W[0:12], W[12:24], W[24:36]])
    assert np.allclose(np.concatenate(parts, axis=1), full, rtol=0, atol=1e-12)


def test_brute_force_triple_loop_and_entries():
    rng = np.random.default_rng(3)
    h = rng.normal(size=(3, 5))
    w = rng.normal(size=(4, 5))
    out = logits_local(h, [w])[0]
    for r in range(3):
        for j in range(4):
            acc = 0.0
            for k in range(5):
                acc += float(h[r, k]) * float(w[j, k])
            assert abs(out[r, j] - acc) < 1e-12
    sub = logits_local_entries(h, w, [2, 0], [3, 1])
    assert np.allclose(sub, out[np.ix_([2, 0], [3, 1])], rtol=0, atol=0)
