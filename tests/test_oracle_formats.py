"""Pins of the oracle's number formats against the format definitions and library routines.

e4m3 here is the OCP 8-bit floating point E4M3 format (the "FP8 E4M3" that the chip-design
page, section on numeric formats, names): sign, 4 exponent bits with bias 7, 3 mantissa bits,
subnormals below 2^-6, no infinities, one NaN pattern per sign (S.1111.111), max finite 448.
"""
import math

import numpy as np
import pytest
import torch


def _code_table_values():
    """Independent table: every positive finite e4m3 value from the format's bit layout."""
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        vals.append(v)
    return np.array(vals)


def _ref_encode_nonneg(x: np.ndarray) -> np.ndarray:
    """Nearest table value, ties to the even code, saturating above 448 (brute force)."""
    vals = _code_table_values()
    x = np.minimum(x.astype(np.float64), 448.0)
    hi = np.searchsorted(vals, x, side="left").clip(0, 126)
    lo = (hi - 1).clip(0, 126)
    dlo = np.abs(x - vals[lo])
    dhi = np.abs(vals[hi] - x)
    pick = np.where(dlo < dhi, lo, hi)
    tie = dlo == dhi
    pick = np.where(tie & (lo % 2 == 0), lo, pick)
    pick = np.where(tie & (hi % 2 == 0), hi, pick)
    return pick.astype(np.uint8)


def test_e4m3_decode_known_values(orc):
    # values fixed by the format definition
    known = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x39: 1.125, 0x40: 2.0, 0x7E: 448.0, 0x7D: 416.0, 0x78: 256.0, 0xB8: -1.0,
             0xFE: -448.0, 0x80: -0.0}
    for code, v in known.items():
        assert orc.e4m3_decode(code) == v, hex(code)
    assert math.isnan(orc.e4m3_decode(0x7F)) and math.isnan(orc.e4m3_decode(0xFF))


def test_e4m3_roundtrip_all_finite_codes(orc):
    codes = [c for c in range(256) if c & 0x7F != 0x7F]
    vals = np.array([orc.e4m3_decode(c) for c in codes], np.float32)
    assert list(orc.e4m3_encode(vals)) == codes


def test_e4m3_midpoints_ties_to_even(orc):
    vals = _code_table_values()
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (vals[:-1] + vals[1:]) / 2)  # exact in fp32
    got = orc.e4m3_encode(mids)
    lo = np.arange(126)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want.astype(np.uint8))
    # one fp32 ulp either side of each midpoint goes to the nearer neighbour
    above = np.nextafter(mids, np.float32(np.inf))
    below = np.nextafter(mids, np.float32(0))
    assert np.array_equal(orc.e4m3_encode(above), (lo + 1).astype(np.uint8))
    assert np.array_equal(orc.e4m3_encode(below), lo.astype(np.uint8))


def test_e4m3_saturation_and_sign(orc):
    x = np.array([448.0, 460.0, 464.0, 465.0, 1e6, np.inf, 3.4e38], np.float32)
    assert list(orc.e4m3_encode(x)) == [0x7E] * len(x)
    assert list(orc.e4m3_encode(-x)) == [0xFE] * len(x)
    assert orc.e4m3_encode(np.float32(np.nan))[0] & 0x7F == 0x7F
    # tiny magnitudes: below a quarter of the smallest subnormal -> signed zero
    assert list(orc.e4m3_encode(np.array([1e-9, -1e-9], np.float32))) == [0x00, 0x80]
    # exactly half the smallest subnormal ties to even -> zero; just above -> 2^-9
    assert orc.e4m3_encode(np.float32(2.0 ** -10))[0] == 0
    assert orc.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1)))[0] == 1


def test_e4m3_sweep_against_table(orc):
    """A strided sweep over every fp32 bit pattern in [0, 480] against the brute-force table."""
    top = np.array([480.0], np.float32).view(np.uint32)[0]
    bits = np.arange(0, int(top), 37, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    got = orc.e4m3_encode(x)
    assert np.array_equal(got, _ref_encode_nonneg(x))
    got_neg = orc.e4m3_encode(-x)
    assert np.array_equal(got_neg, _ref_encode_nonneg(x) | 0x80)


def test_e4m3_matches_torch_conversion_in_range(orc):
    """torch's float8_e4m3fn cast rounds to nearest even; it agrees wherever |x| <= 448."""
    g = torch.Generator().manual_seed(5)
    x = torch.randn(200_000, generator=g) * torch.exp2(torch.randint(-14, 9, (200_000,), generator=g).float())
    x = x.clamp(-448, 448)
    want = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.e4m3_encode(x.numpy())
    # torch keeps the sign of a zero result; so does the oracle
    assert np.array_equal(got, want)


def test_bf16_rounding(orc):
    # values exact in fp32: one rounding either way, compare with torch's fp32 -> bf16 cast
    g = torch.Generator().manual_seed(6)
    x = torch.randn(50_000, generator=g, dtype=torch.float32) * 10.0
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.double_to_bf16(float(v)) for v in x.numpy()], np.uint16)
    assert np.array_equal(got, want)
    # a double just above a bf16 midpoint must round up; a detour through fp32 would land
    # exactly on the midpoint and round to even (down) instead
    assert orc.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert orc.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80      # exact midpoint -> even
    assert orc.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82  # midpoint, odd below -> up
    assert orc.double_to_bf16(-2.5) == 0xC020
    assert orc.double_to_bf16(1e39) == 0x7F80
    assert orc.double_to_bf16(0.0) == 0x0000 and orc.double_to_bf16(-0.0) == 0x8000
