"""Exact decoding of the stored number formats (oracle; test infrastructure only).

BF16: the upper 16 bits of an IEEE-754 binary32 value.
FP8 e4m3 (OCP 8-bit floating point, "E4M3"): 1 sign bit, 4 exponent bits with bias 7,
3 mantissa bits; exponent field 0 encodes subnormals m/8 * 2**-6; there are no
infinities; S.1111.111 is NaN; the largest finite magnitude is S.1111.110 = 448.
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_value(code: int) -> float:
    """Value of one e4m3 code, straight from the definition."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_to_f64(codes: np.ndarray, scale: np.ndarray | None = None) -> np.ndarray:
    """FP8 e4m3 codes (uint8, [..., D]) -> float64, times the per-row scale ([...]) if given."""
    v = E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]
    if scale is not None:
        v = v * np.asarray(scale, dtype=np.float64)[..., None]
    return v


def decode_rows(data: np.ndarray, scale: np.ndarray | None) -> np.ndarray:
    """Rows of a cache as float64: BF16 bits when ``scale`` is None, else e4m3 codes x scale."""
    if scale is None:
        return bf16_to_f64(data)
    return e4m3_to_f64(data, scale)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value to each float64 x, ties to the even mantissa, magnitudes beyond 448
    saturated to 448 (round-to-nearest-even with saturation to the largest finite value).

    The e4m3 grid from the definition above: in the binade [2**e, 2**(e+1)), e >= -6, the
    values are spaced 2**(e-3); below 2**-6 the subnormals are spaced 2**-9.  Returns values,
    not codes.  NaN stays NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, E = np.frexp(np.where(a > 0, a, 1.0))          # a = f * 2**E with f in [0.5, 1)
    e = np.maximum(E - 1, -6)                          # floor(log2 a), at least the smallest normal binade
    quantum = np.ldexp(1.0, e - 3)
    v = np.minimum(np.rint(a / quantum) * quantum, 448.0)   # np.rint: half to even
    v = np.where(a > 0, v, 0.0)
    return np.where(np.isnan(x), np.nan, np.copysign(v, x))
