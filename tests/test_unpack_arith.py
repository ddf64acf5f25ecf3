"""CPU check of the float arithmetic the decode kernel uses to turn V codes
into exact offsets (code - qmax) * eps without converting integers: a code
placed in mantissa bits [p, p + width) of 1.0 reads as 1 + code * 2^(p - 23),
and subtracting 1 + qmax * 2^(p - 23) in float32 leaves (code - qmax) *
2^(p - 23) exactly, for every code, at every placement the kernel uses
(4-bit at p = 0, 4, 8, 12; 8-bit at p = 0, 8).  The kernel's own results are
checked against the oracle by the GPU tests; this pins the identity its
unpacking rests on, so a placement that reached the exponent field or an
offset that rounded would fail here first."""

import numpy as np
import pytest


def mant_or(x: np.ndarray, mask: int) -> np.ndarray:
    return ((x.astype(np.uint32) & np.uint32(mask)) | np.uint32(0x3F800000)).view(np.float32)


@pytest.mark.parametrize("bits,positions", [(4, (0, 4, 8, 12)), (8, (0, 8))])
def test_offsets_are_exact(bits, positions):
    qmax = 7 if bits == 4 else 127
    width = bits
    codes = np.arange(0, 2 * qmax + 1, dtype=np.uint32)
    for p in positions:
        assert p + width <= 23                       # below the exponent field
        f = mant_or(codes << np.uint32(p), ((1 << width) - 1) << p)
        corr = np.float32(1.0 + qmax * 2.0 ** (p - 23))
        assert float(corr) == 1.0 + qmax * 2.0 ** (p - 23)          # the constant itself is exact
        got = (f - corr).astype(np.float64)                         # one float32 subtraction
        want = (codes.astype(np.float64) - qmax) * 2.0 ** (p - 23)
        np.testing.assert_array_equal(got, want)
        assert got[qmax] == 0.0                                      # the zero code gives exactly 0


def test_word_split_keeps_channel_order():
    """A 32-bit code word and the word shifted right by 16 give the eight
    nibbles (or four bytes) of the word in channel order at the placements
    above."""
    rng = np.random.default_rng(0)
    nib = rng.integers(0, 15, size=8).astype(np.uint32)
    w = np.uint32(0)
    for k in range(8):
        w |= nib[k] << np.uint32(4 * k)
    got = []
    for h in range(2):
        x = np.array([w >> np.uint32(16 * h)], np.uint32)
        for p in (0, 4, 8, 12):
            f = mant_or(x, 0xF << p)[0]
            got.append(round((float(f) - 1.0) / 2.0 ** (p - 23)))
    assert got == [int(n) for n in nib]
    byts = rng.integers(0, 255, size=4).astype(np.uint32)
    w = np.uint32(byts[0] | (byts[1] << 8) | (byts[2] << 16) | (byts[3] << 24))
    got = []
    for h in range(2):
        x = np.array([w >> np.uint32(16 * h)], np.uint32)
        for p in (0, 8):
            f = mant_or(x, 0xFF << p)[0]
            got.append(round((float(f) - 1.0) / 2.0 ** (p - 23)))
    assert got == [int(b) for b in byts]
