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
        enc = {"e2m1": F.e2m1_encode, "ue4m3": F.ue4m3_encode, "e4m3": F.e4m3_encode}[kind]
        got = enc(arr)[0]
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


def test_e4m3_sign_symmetry_and_nan():
    mags = np.arange(127)
    pos = F.e4m3_value(mags)
    neg = F.e4m3_value(mags | 0x80)
    assert np.array_equal(neg, -pos)
    assert np.array_equal(pos, F.ue4m3_value(mags))
    assert np.isnan(F.e4m3_value(np.array([0x7F, 0xFF]))).all()
    assert math.copysign(1.0, float(F.e4m3_value(np.array([0x80]))[0])) == -1.0


def test_e4m3_round_trip_every_finite_code():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    vals = F.e4m3_value(codes).astype(np.float32)
    assert np.array_equal(F.e4m3_encode(vals), codes)


def test_e4m3_encode_is_nearest():
    """Brute force over random float32 inputs: the decoded code is a nearest finite E4M3
    value (or +-448 beyond it), with the input's sign."""
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(4000) * 10.0, rng.standard_normal(2000) * 0.01,
                        rng.uniform(-600, 600, 1000)]).astype(np.float32)
    finite = np.unique(np.abs(F.e4m3_value(np.arange(127))))
    got = F.e4m3_value(F.e4m3_encode(x))
    for xi, gi in zip(x.astype(np.float64), got):
        m = min(abs(xi), 448.0)
        best = np.min(np.abs(finite - m))
        assert abs(abs(gi) - m) == best, (xi, gi)
        assert math.copysign(1.0, gi) == math.copysign(1.0, xi)
