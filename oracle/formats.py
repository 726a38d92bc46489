"""Exact conversion of stored-precision values to fp64 (test infrastructure only).

bf16: the upper 16 bits of an IEEE-754 binary32; widening is exact.
e4m3 (OCP 8-bit floating point, "fn" variant): 1 sign bit, 4 exponent bits with
bias 7, 3 mantissa bits; exponent field 0 encodes subnormals m/8 * 2^-6; the two
codes with all exponent and mantissa bits set (0x7F, 0xFF) are NaN; no infinities.
The largest finite magnitude is 1.75 * 2^8 = 448, the smallest subnormal 2^-9.
The FP8 expert weights follow the per-tensor FP8 MoE path of the SageMaker MoE
kernels page (second item); the format itself is the OCP definition above.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(u16) -> np.ndarray:
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


def _e4m3_table() -> np.ndarray:
    tab = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        exp = (code >> 3) & 0xF
        man = code & 0x7
        if exp == 0xF and man == 0x7:
            tab[code] = np.nan
        elif exp == 0:
            tab[code] = sign * (man / 8.0) * 2.0 ** (1 - 7)
        else:
            tab[code] = sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)
    return tab


E4M3_TABLE = _e4m3_table()


def e4m3_bits_to_f64(u8) -> np.ndarray:
    return E4M3_TABLE[np.asarray(u8, dtype=np.uint8)]


def to_f64(raw: np.ndarray, dtype: str) -> np.ndarray:
    """raw storage (uint16 for bf16, uint8 for e4m3, float32 for f32) -> fp64."""
    if dtype == "bf16":
        return bf16_bits_to_f64(raw)
    if dtype == "e4m3":
        return e4m3_bits_to_f64(raw)
    if dtype == "f32":
        return np.asarray(raw, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)
