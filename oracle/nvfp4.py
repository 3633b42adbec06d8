"""NVFP4 quantisation with per-32 E4M3 block scales (CPU oracle, test infrastructure).

Weights and activations share one rule ("Compression details" table of the
Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card: NVFP4 values, one FP8-E4M3 scale
per 32 dense K elements, FP32 per-tensor global scale; activations use dynamic
per-32 group scales).  The pages give the format but not the arithmetic, so
this oracle fixes it as follows (every operation IEEE binary32, round to
nearest even; the same reading is stated in the library header):

  for each row and each group of 32 consecutive K elements, with global g:
    amax = max |x_i|
    s    = amax / (6 * g)               6*g rounded to fp32 first; s = 0 if 6*g == 0
    sc   = E4M3(s)                      nearest, ties to even, saturating at 448
    sdq  = value(sc) * g
    if sdq == 0: every code is 0x0
    else:        inv = 1 / sdq ;  code_i = E2M1(x_i * inv)

The weight global is g = amax(|W|) / (6 * 448) over the (pruned) tensor, the
multiplier convention: dequantised value = E2M1 * E4M3 * g.
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_quantize, e4m3_decode, e4m3_quantize, f32

GROUP = 32          # dense K elements per block scale
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def global_scale(amax) -> np.float32:
    """FP32 per-tensor global: amax / (6 * 448)."""
    return np.float32(f32(amax) / np.float32(E2M1_MAX * E4M3_MAX))


def quantize_groups(x, g):
    """Quantise float32 rows ``x [rows, K]`` with per-row global ``g`` (scalar or [rows]).

    Returns (codes uint8 [rows, K] one 4-bit code per element,
             scales uint8 [rows, K/32] E4M3 codes).
    """
    x = f32(x)
    rows, K = x.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 32")
    g = np.broadcast_to(f32(g).reshape(-1, 1), (rows, 1)).astype(np.float32)
    xg = x.reshape(rows, K // GROUP, GROUP)
    amax = np.abs(xg).max(axis=-1)                                   # exact in fp32
    six_g = f32(np.float32(E2M1_MAX) * g)                            # [rows, 1]
    with np.errstate(divide="ignore", invalid="ignore"):
        s = np.where(six_g == 0, np.float32(0), f32(amax / six_g))
    sc = e4m3_quantize(s)
    sdq = f32(f32(e4m3_decode(sc)) * g)                              # [rows, K/32]
    with np.errstate(divide="ignore"):
        inv = np.where(sdq == 0, np.float32(0), f32(np.float32(1.0) / np.where(sdq == 0, 1, sdq)))
    v = f32(xg * inv[..., None])
    codes = e2m1_quantize(v)
    codes = np.where((sdq == 0)[..., None], np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(rows, K), sc.astype(np.uint8)


def pack_codes(codes) -> np.ndarray:
    """Two 4-bit codes per byte, the lower-K element in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_codes(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
