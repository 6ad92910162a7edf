"""Pins for the oracle's Philox4x32-10 and its uniform mapping (CPU only)."""
import numpy as np

from oracle.philox import philox4x32, token_uniforms

# Known-answer vectors published with the Random123 library by the authors of
# "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11): philox4x32, 10 rounds,
# (counter words, key words) -> output words.
KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF), (0xFFFFFFFF, 0xFFFFFFFF),
     (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


def test_known_answer_vectors():
    for ctr, key, expect in KAT:
        got = philox4x32(np.array(ctr, np.uint32), np.array(key, np.uint32))
        assert [int(v) for v in got] == list(expect)


def test_known_answer_vectors_batched():
    ctr = np.array([k[0] for k in KAT], np.uint32)
    key = np.array([k[1] for k in KAT], np.uint32)
    got = philox4x32(ctr, key)
    assert got.tolist() == [list(k[2]) for k in KAT]


def test_uniform_mapping_word_selection():
    # token i uses word i mod 4 of the block floor(i / 4): check against the
    # raw generator output for a hand-built counter
    seed = (0x12345678 << 32) | 0x9ABCDEF0
    words = philox4x32(np.array([5, 77, 3, 0], np.uint32),
                       np.array([0x9ABCDEF0, 0x12345678], np.uint32))
    u = token_uniforms(np.arange(20, 24), 3, 77, seed)
    expect = ((words >> 9).astype(np.float64) + 0.5) * 2.0 ** -23
    assert np.array_equal(u, expect)


def test_uniforms_open_interval_and_float32_exact():
    u = token_uniforms(np.arange(0, 1 << 16), 11, 5, 1234)
    assert np.all(u > 0) and np.all(u < 1)
    assert np.array_equal(u.astype(np.float32).astype(np.float64), u)
    one_minus = 1.0 - u
    assert np.array_equal(one_minus.astype(np.float32).astype(np.float64), one_minus)
    # extremes of the mapping are exact float32 values strictly inside (0, 1)
    lo, hi = (0 + 0.5) * 2.0 ** -23, (2 ** 23 - 1 + 0.5) * 2.0 ** -23
    assert lo == 2.0 ** -24 and hi == 1 - 2.0 ** -24
    assert float(np.float32(hi)) == hi and float(np.float32(lo)) == lo


def test_uniforms_roughly_uniform():
    u = token_uniforms(np.arange(1 << 18), 0, 0, 7)
    hist, _ = np.histogram(u, bins=16, range=(0, 1))
    expect = u.size / 16
    assert np.all(np.abs(hist - expect) < 6 * np.sqrt(expect))
