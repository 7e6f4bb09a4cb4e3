"""The P-code packing of the INT4 softmax, checked on the host: four keys of a
word are rounded into [2^23, 2^24) against four different magic constants
whose bit patterns K0..K3 satisfy K0 + K1 2^8 + K2 2^16 + K3 2^24 = 0 mod 2^32,
so the integer sum t0 + t1 2^8 + t2 2^16 + t3 2^24 of the rounded values' bits
is the word of the four codes.  Keys past N give NaN bits; they form a suffix
of the word and must leave the bytes of the valid keys intact.  The constants
are read from the kernel source."""
import itertools
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "int4_quantized_flashattention_b200", "csrc", "ra_attn_int4.cu")


def _magics():
    s = open(SRC).read()
    lo = re.search(r"kMagLo = make_float2\(([0-9.]+)f, ([0-9.]+)f\)", s)
    hi = re.search(r"kMagHi = make_float2\(([0-9.]+)f, (kMagicF|[0-9.]+f?)\)", s)
    magic = float(re.search(r"kMagicF = ([0-9.]+)f;", s).group(1))
    m3 = magic if hi.group(2) == "kMagicF" else float(hi.group(2).rstrip("f"))
    return [np.float32(float(lo.group(1))), np.float32(float(lo.group(2))), np.float32(float(hi.group(1))),
            np.float32(m3)]


def _bits(x):
    return int(np.array(x, np.float32).view(np.uint32))


def _pack(t):
    lo = (_bits(t[1]) * 256 + _bits(t[0])) & 0xFFFFFFFF
    hi = (_bits(t[3]) * 256 + _bits(t[2])) & 0xFFFFFFFF
    return (hi * 65536 + lo) & 0xFFFFFFFF


def test_magic_constants_cancel():
    M = _magics()
    K = [_bits(m) for m in M]
    assert all(2 ** 23 <= float(m) < 2 ** 24 and (k & 0xFF) == 0 for m, k in zip(M, K))
    assert (K[0] + (K[1] << 8) + (K[2] << 16) + (K[3] << 24)) % 2 ** 32 == 0


def test_every_code_word_packs_exactly():
    M = _magics()
    codes = range(16)
    for c in itertools.product(codes, repeat=4):
        # t = fl(M + c): exact for integer c in [0, 15] in this binade
        t = [np.float32(M[i] + np.float32(c[i])) for i in range(4)]
        assert _pack(t) == c[0] | c[1] << 8 | c[2] << 16 | c[3] << 24


def test_rounding_is_rint_in_every_lane():
    """fl(L e + M) - M = rint(L e) (ties to even) for e in [0, 1], L = 15 and 7."""
    M = _magics()
    rng = np.random.default_rng(0)
    e = np.concatenate([rng.random(20000), (np.arange(31) + 0.5) / 15, (np.arange(15) + 0.5) / 7, [0.0, 1.0]])
    e = e.astype(np.float32)
    for L in (np.float32(15), np.float32(7)):
        want = np.rint(L.astype(np.float64) * e.astype(np.float64))
        for m in M:
            # float32 multiply-add with one rounding: exact product in float64, then round
            got = (L.astype(np.float64) * e.astype(np.float64) + np.float64(m)).astype(np.float32)
            assert np.array_equal(got.astype(np.float64) - np.float64(m), want)


def test_nan_suffix_keeps_valid_bytes():
    M = _magics()
    nan_bits = np.array([0x7FFFFFFF], np.uint32).view(np.float32)[0]
    rng = np.random.default_rng(1)
    for _ in range(2000):
        c = rng.integers(0, 16, 4)
        for nvalid in range(1, 4):
            t = [np.float32(M[i] + np.float32(c[i])) if i < nvalid else nan_bits for i in range(4)]
            w = _pack(t)
            mask = (1 << (8 * nvalid)) - 1
            assert w & mask == sum(int(c[i]) << (8 * i) for i in range(nvalid))
