"""Pins of the oracle's number formats (CPU only).

E2M1 and E4M3 are the NVFP4 value and block-scale formats of the "Compression
details" table of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card; bf16 is the
layer's input/output type.  The pins are hand-worked values (tests/golden) and
library casts of torch (float8_e4m3fn, bfloat16), not the oracle's own code.
"""
import fractions

import numpy as np
import pytest
import torch

from oracle import formats as F


def test_e2m1_values_match_golden(golden):
    g = golden("e2m1.json")
    want = np.array(g["values"], dtype=np.float64)
    got = F.e2m1_decode(np.arange(16))
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_e2m1_rounding_golden(golden):
    for v, code in golden("e2m1.json")["round_nearest_even_cases"]:
        assert int(F.e2m1_quantize(np.float32(v))) == code, v


def test_e2m1_rounding_is_nearest_with_even_ties():
    rng = np.random.default_rng(7)
    ties = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    v = np.concatenate([rng.uniform(-8, 8, 200000).astype(np.float32), ties, -ties])
    c = F.e2m1_quantize(v)
    q = F.e2m1_decode(c)
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    a = np.minimum(np.abs(v.astype(np.float64)), 6.0)
    dist = np.abs(a[:, None] - mags[None, :]).min(axis=1)
    assert np.allclose(np.abs(np.abs(q) - a), dist, atol=0)          # a nearest value
    tie = np.isclose(np.abs(a[:, None] - mags[None, :]), dist[:, None], atol=0).sum(axis=1) == 2
    assert ((c[tie] & 1) == 0).all()                                   # ties to even code
    assert ((c >> 3) == np.signbit(v)).all()                           # sign follows input


def test_e4m3_decode_matches_torch():
    b = torch.arange(256, dtype=torch.uint8)
    t = b.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    o = F.e4m3_decode(np.arange(256))
    nan = np.isnan(t)
    assert np.array_equal(nan, np.isnan(o))
    assert np.array_equal(t[~nan], o[~nan])
    assert F.e4m3_value(0x7E) == 448.0 and F.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_rounding_matches_torch_in_range():
    vals = F.e4m3_decode(np.arange(127))
    mids = (vals[1:] + vals[:-1]) / 2
    rng = np.random.default_rng(1)
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        rng.uniform(0, 448, 100000), rng.uniform(0, 2 ** -5, 50000)]).astype(np.float32)
    x = x[x <= 448]
    x = np.concatenate([x, -x])
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_quantize(x), t)


def test_e4m3_saturates():
    assert int(F.e4m3_quantize(np.float32(1000.0))) == 0x7E
    assert int(F.e4m3_quantize(np.float32(465.0))) == 0x7E
    assert int(F.e4m3_quantize(np.float32(-1e30))) == 0xFE
    assert int(F.e4m3_quantize(np.float32(2.0 ** -10))) == 0        # tie at half the smallest subnormal
    assert int(F.e4m3_quantize(np.float32(2.0 ** -10 * 1.0001))) == 1


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000),
                        [129.5, 128.5, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 0.0, 3e38]]).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(F.bf16_round(x), t)


def test_bf16_round_exact_fraction_cases():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert F.bf16_round(np.float32(1 + 2 ** -8)) == np.float32(1.0)
    assert F.bf16_round(np.float32(1 + 3 * 2 ** -8)) == np.float32(1 + 2 ** -6)
    assert fractions.Fraction(float(F.bf16_round(np.float32(129.5)))) == 130
