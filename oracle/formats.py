"""Number formats used by the oracle, written from their public definitions.

TEST INFRASTRUCTURE: only tests, the smoke check and the bench's CPU-baseline leg use this.

  * BF16: 1 sign, 8 exponent, 7 fraction bits (the upper half of an IEEE binary32).
  * FP16: IEEE binary16.
  * E2M1 (the element type of NVFP4): 1 sign, 2 exponent, 1 mantissa bit, bias 1, no
    inf/NaN; magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; bit 3 is the sign.
  * UE4M3 (the NVFP4 block-scale type, an E4M3 with the sign bit unused): 4 exponent bits,
    bias 7, 3 mantissa bits; subnormals m * 2^-9; largest finite 448 (0x7E); 0x7F is NaN.
  * E4M3 (the FP8 element type of the reduced-precision projected-key cache): bit 7 is the
    sign, bits 6..0 a UE4M3 magnitude; 0x7F and 0xFF are NaN.

"Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention" (Full text)
names NVFP4 storage; the element/scale layout above is the public NVFP4 format.

Encoders are "nearest representable value, ties to the even code, saturate to the largest
finite value" (round-to-nearest-even, satfinite), done by table lookup so that they can be
checked by eye against the tables.
"""
from __future__ import annotations

import numpy as np

# ---- BF16 / FP16 -----------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (nearest, ties to even); returns BF16 bit patterns.

    Written as scaling to an 8-significant-bit integer, rounding half to even, and scaling
    back; exact in float64 for every finite float32 input.
    """
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    _, e = np.frexp(x64)                       # x = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                    # below 2^-126 the BF16 spacing is 2^-133
    step = np.ldexp(1.0, e - 8)                # spacing of 8-significant-bit values at x
    y = np.round(x64 / step) * step            # np.round is half-to-even
    y32 = y.astype(np.float32)                 # exact: y has at most 8 significant bits
    return (y32.view(np.uint32) >> np.uint32(16)).astype(np.uint16) | (
        (np.signbit(x64).astype(np.uint16) << np.uint16(15)))


# ---- E2M1 -------------------------------------------------------------------------------------

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_value(code: np.ndarray) -> np.ndarray:
    """Decode 4-bit E2M1 codes (0..15) to float64."""
    c = np.asarray(code).astype(np.int64)
    mag = E2M1_MAG[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def _nearest_even(table: np.ndarray, mag: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of an ascending table; ties go to the even index."""
    mid = (table[:-1] + table[1:]) / 2.0
    idx = np.searchsorted(mid, mag, side="left")           # count of midpoints < mag
    at_mid = (idx < len(mid)) & (mid[np.minimum(idx, len(mid) - 1)] == mag)
    odd = (idx & 1) == 1
    return np.where(at_mid & odd, idx + 1, idx)


def e2m1_encode(t: np.ndarray) -> np.ndarray:
    """float32 -> E2M1 code, round to nearest even, saturating at +-6; sign bit copied."""
    t64 = np.asarray(t, dtype=np.float32).astype(np.float64)
    mag = np.abs(t64)
    code = _nearest_even(E2M1_MAG, mag)
    code = np.where(mag >= 6.0, 7, code)
    return (code | np.where(np.signbit(t64), 8, 0)).astype(np.uint8)


# ---- UE4M3 ------------------------------------------------------------------------------------

def ue4m3_value(code: np.ndarray) -> np.ndarray:
    """Decode unsigned E4M3 scale codes (0..126) to float64; 127 decodes to NaN."""
    c = np.asarray(code).astype(np.int64)
    e = c >> 3
    m = c & 7
    v = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    return np.where(c == 0x7F, np.nan, v)


UE4M3_VALUES = ue4m3_value(np.arange(127))                  # codes 0..126, ascending


def ue4m3_encode(sf: np.ndarray) -> np.ndarray:
    """Non-negative float32 -> UE4M3 code, nearest even, saturating at 448 (code 0x7E)."""
    s64 = np.asarray(sf, dtype=np.float32).astype(np.float64)
    code = _nearest_even(UE4M3_VALUES, s64)
    return np.where(s64 >= 448.0, 126, code).astype(np.uint8)


# ---- E4M3 (signed FP8) ------------------------------------------------------------------------

def e4m3_value(code: np.ndarray) -> np.ndarray:
    """Decode signed E4M3 codes (0..255) to float64 (0x7F / 0xFF decode to NaN)."""
    c = np.asarray(code).astype(np.int64)
    mag = ue4m3_value(c & 0x7F)
    return np.where((c & 0x80) != 0, -mag, mag)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 code: magnitude to the nearest UE4M3 value (ties to the even code,
    saturating at 448), sign bit copied (so -0.0 and negative values that round to zero
    keep it)."""
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    mag = ue4m3_encode(np.abs(x64)).astype(np.int64)
    return (mag | np.where(np.signbit(x64), 0x80, 0)).astype(np.uint8)
