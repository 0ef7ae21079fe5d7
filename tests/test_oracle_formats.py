"""Pins of the oracle's number formats against hand-derived values and exact arithmetic."""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats as F
from tests.conftest import read_golden


def test_e2m1_table_matches_definition():
    rows = read_golden("e2m1_codes.txt")
    assert len(rows) == 16
    for code, val in rows:
        c = int(code, 16)
        got = float(F.e2m1_value(np.array([c]))[0])
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code


def test_ue4m3_table_matches_definition():
    for code, val in read_golden("ue4m3_codes.txt"):
        assert float(F.ue4m3_value(np.array([int(code, 16)]))[0]) == float(val), code
    assert np.isnan(F.ue4m3_value(np.array([0x7F]))[0])


def test_round_trips():
    codes = np.arange(16, dtype=np.uint8)
    vals = F.e2m1_value(codes).astype(np.float32)
    assert np.array_equal(F.e2m1_encode(vals), codes)
    sc = np.arange(127, dtype=np.uint8)
    assert np.array_equal(F.ue4m3_encode(F.ue4m3_value(sc).astype(np.float32)), sc)


def test_rounding_cases():
    for kind, x, want in read_golden("rounding_cases.txt"):
        arr = np.array([float(x)], dtype=np.float32)
        got = F.e2m1_encode(arr)[0] if kind == "e2m1" else F.ue4m3_encode(arr)[0]
        assert int(got) == int(want, 16), (kind, x, hex(int(got)))


def test_e2m1_encode_is_nearest():
    """Brute force: the encoded value is a nearest table entry for many random inputs."""
    rng = np.random.default_rng(0)
    t = (rng.standard_normal(20000) * 3).astype(np.float32)
    enc = F.e2m1_value(F.e2m1_encode(t))
    mags = np.concatenate([F.E2M1_MAG, -F.E2M1_MAG])
    best = np.abs(t.astype(np.float64)[:, None] - mags[None, :]).min(axis=1)
    clipped = np.clip(t.astype(np.float64), -6, 6)
    assert np.all(np.abs(enc - clipped) <= best + 1e-12)


def _bf16_exact(x: float) -> int:
    """BF16 bits of float32 x by exact rational rounding (half to even)."""
    bits = struct.unpack("<I", struct.pack("<f", x))[0]
    sign = bits >> 31
    fr = abs(Fraction(x))
    if fr == 0:
        return sign << 15
    e = math.floor(math.log2(fr))
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    e = max(e, -126)
    step = Fraction(2) ** (e - 7)
    q = fr / step
    n = math.floor(q)
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    y = float(n * step)
    yb = struct.unpack("<I", struct.pack("<f", y))[0]
    return (yb >> 16) | (sign << 15)


def test_bf16_rounding_exact_rational():
    rng = np.random.default_rng(1)
    xs = np.concatenate([
        (rng.standard_normal(3000) * 10).astype(np.float32),
        (rng.standard_normal(500) * 1e-39).astype(np.float32),     # subnormals
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -(1 + 2 ** -8)],
                 dtype=np.float32),
    ])
    got = F.f32_to_bf16_rne(xs)
    for x, g in zip(xs.tolist(), got.tolist()):
        assert g == _bf16_exact(float(np.float32(x))), x


def test_bf16_midpoints_hand():
    xs = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 2 ** -130], dtype=np.float32)
    assert F.f32_to_bf16_rne(xs).tolist() == [0x3F80, 0x3F82, 0x0008]
