"""Number formats of the NVFP4 weights and activations (CPU oracle, test infrastructure).

The model cards fix the formats ("Compression details" table of the
Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card): values are NVFP4 (E2M1), with one
FP8-E4M3 block scale per 32 dense K elements and an FP32 per-tensor global
scale.  Packed NVFP4 stores two adjacent K elements per byte ("Sparse storage
layout (paired48_sparse, pair-bitmask v1)" on the same card).  The pages do not
say which nibble holds the lower-K element; this oracle reads it as the low
nibble, the same convention the card states for the mask ("the low nibble is
the lower-K chunk").

Everything here is written from the format definitions, in float64/int64,
element by element where that is clearer than speed.  This module is test
infrastructure: only tests, the smoke check and the CPU-baseline leg of the
benchmark use it.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------- E2M1 -------
# E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN.
#   e == 0: subnormal, value = m * 0.5
#   e  > 0: value = 2**(e-1) * (1 + m/2)


def e2m1_magnitude(code: int) -> float:
    """Magnitude of the 3 low bits of an E2M1 code, from the format definition."""
    e, m = (code >> 1) & 3, code & 1
    if e == 0:
        return 0.5 * m
    return float(2.0 ** (e - 1) * (1.0 + m / 2.0))


E2M1_MAG = np.array([e2m1_magnitude(c) for c in range(8)], dtype=np.float64)


def e2m1_decode(codes) -> np.ndarray:
    """float64 values of 4-bit E2M1 codes (bit 3 = sign)."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    v = E2M1_MAG[c & 7]
    return np.where(c & 8, -v, v)


def e2m1_quantize(v) -> np.ndarray:
    """Round float32 values to E2M1 codes: nearest value, ties to the even code,
    magnitudes above 6 saturate to 6, the sign bit follows the input's sign
    (so -0.0 and small negatives give code 0x8)."""
    v = np.asarray(v, dtype=np.float32)
    if np.isnan(v).any():
        raise ValueError("NaN input to e2m1_quantize")
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[..., None] - E2M1_MAG)              # distance to each magnitude
    best = d.min(axis=-1, keepdims=True)
    cand = d == best                                  # one or two candidates
    even = cand & ((np.arange(8) & 1) == 0)
    pick = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    pick = np.where(a > 6.0, 7, pick)
    sign = np.signbit(v).astype(np.int64) << 3
    return (pick.astype(np.int64) | sign).astype(np.uint8)


# ---------------------------------------------------------------- E4M3 -------
# FP8 E4M3 ("fn" flavour): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
# no infinities, 0x7F/0xFF are NaN, largest finite 448.
#   e == 0: subnormal, value = m * 2**-9
#   e  > 0: value = 2**(e-7) * (1 + m/8)


def e4m3_value(byte: int) -> float:
    s, e, m = (byte >> 7) & 1, (byte >> 3) & 0xF, byte & 7
    if e == 15 and m == 7:
        return float("nan")
    v = m * 2.0 ** -9 if e == 0 else 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return -v if s else v


E4M3_VAL = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)
_E4M3_POS = E4M3_VAL[:127]   # codes 0x00..0x7E: the nonnegative finite values, increasing


def e4m3_decode(b) -> np.ndarray:
    return E4M3_VAL[np.asarray(b).astype(np.int64) & 0xFF]


def e4m3_quantize(x) -> np.ndarray:
    """Round float32 values to E4M3 codes: nearest, ties to the even code,
    finite values above 448 in magnitude saturate to 448 (satfinite)."""
    x = np.asarray(x, dtype=np.float32)
    if np.isnan(x).any():
        raise ValueError("NaN input to e4m3_quantize")
    a = np.abs(x.astype(np.float64))
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 126)  # first value >= a
    lo = np.clip(hi - 1, 0, 126)
    dlo, dhi = a - _E4M3_POS[lo], _E4M3_POS[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= 448.0, 126, pick)
    pick = np.where(a == _E4M3_POS[hi], hi, pick)
    sign = np.signbit(x).astype(np.int64) << 7
    return (pick.astype(np.int64) | sign).astype(np.uint8)


# ---------------------------------------------------------------- bf16 -------

def f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float32)


def bf16_round(x) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even), returned as float32."""
    x = np.asarray(x, dtype=np.float32)
    shape = x.shape
    x = np.ascontiguousarray(x).reshape(-1)
    if np.isnan(x).any():
        raise ValueError("NaN input to bf16_round")
    u = x.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (r.astype(np.uint32) << 16).view(np.float32).reshape(shape)


def bf16_bits(x) -> np.ndarray:
    """uint16 bit patterns of float32 values already on the bf16 grid."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32)
    return (b << 16).view(np.float32)
