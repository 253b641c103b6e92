import numpy as np

import oracle
from conftest import read_golden


def test_pack_golden_words():
    for bits, codes, words in read_golden("pack_words.txt"):
        bits = int(bits)
        c = np.array([[int(x) for x in codes.split()]])
        expect = [int(w, 16) for w in words.split()]
        got = oracle.pack_codes(c, bits)
        assert got.dtype == np.uint32
        assert got[0].tolist() == expect
        assert np.array_equal(oracle.unpack_codes(got, bits, c.shape[1]), c)


def test_pack_roundtrip_random():
    g = np.random.default_rng(0)
    for bits in (2, 3, 4, 5, 8):
        c = g.integers(0, 1 << bits, size=(3, 64))
        assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(c, bits), bits, 64), c)
