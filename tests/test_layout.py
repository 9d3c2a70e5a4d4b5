"""The test-side packer (tests/layout.py) against the layout statement in include/tq.h:
every word bit carries exactly one code bit, pack/unpack round-trips, and the
sign-magnitude relabelling is a bijection that keeps the codebook's symmetry."""
import numpy as np
import pytest

import layout


@pytest.mark.parametrize("P", [1, 2, 3, 4, 5])
def test_positions_are_a_bijection(P):
    seen = set()
    for e in range(32):
        for b in range(P):
            w, pos = layout._pos(P, e, b)
            assert 0 <= w < P and 0 <= pos < 32
            seen.add((w, pos))
    assert len(seen) == 32 * P


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_sign_magnitude_roundtrip(k):
    K = 1 << k
    idx = np.arange(K)
    code = layout._to_sign_magnitude(idx, k)
    assert sorted(code.tolist()) == list(range(K))
    assert (layout._from_sign_magnitude(code, k) == idx).all()
    if k > 1:
        # mirrored indices (c[K-1-i] = -c[i]) share the magnitude and differ in the flag
        m = (1 << (k - 1)) - 1
        assert ((code & m) == (code[::-1] & m)).all()
        assert ((code >> (k - 1)) != (code[::-1] >> (k - 1))).all()


@pytest.mark.parametrize("d,k,prod", [(128, 3, True), (128, 4, False), (64, 2, True), (64, 3, False),
                                      (64, 1, True), (64, 2, False), (200, 3, True), (96, 4, True),
                                      (40, 1, False)])
def test_pack_unpack_roundtrip(d, k, prod):
    rng = np.random.default_rng(d * 10 + k)
    n = 7
    idx = rng.integers(0, 1 << k, size=(n, d))
    signs = rng.integers(0, 2, size=(n, d)).astype(np.uint8) if prod else None
    codes = layout.pack(idx, signs, d, k)
    assert codes.shape == (n, layout.geometry(d, k, prod)[2])
    i2, s2, pad = layout.unpack(codes, d, k, prod)
    assert (i2 == idx).all()
    if prod:
        assert (s2 == signs).all()
    assert not pad.any()


def test_p4_word_reading():
    """P = 4: the low three code bits of slice s are nibbles of word s, the top bits of the
    first four coordinates are the byte msbs of that word."""
    d, k = 32, 3
    idx = np.array([[(3 * e) % 8 for e in range(32)]])
    signs = np.array([[e % 3 == 0 for e in range(32)]], dtype=np.uint8)
    w = layout.pack(idx, signs, d, k).view("<u4")[0]
    code = layout._to_sign_magnitude(idx[0], k) | (signs[0].astype(np.int64) << k)
    for s in range(4):
        for j in range(8):
            assert (int(w[s]) >> (4 * j)) & 7 == code[8 * s + j] & 7
        for i in range(4):
            assert (int(w[s]) >> (8 * i + 7)) & 1 == code[8 * s + i] >> 3
            assert (int(w[s]) >> (8 * i + 3)) & 1 == code[8 * s + 4 + i] >> 3
