"""Pins of the oracle's exact grouped GEMM, SwiGLU and expert MLP (CPU only).

The GEMM is the quantised sparse product of the "Compression details" table of
the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card (NVFP4 weights and activations,
E4M3 per-32 scales, FP32 globals).  Pins: brute force with exact rationals on
tiny inputs, and special cases that reduce to a plain float64 matmul.
"""
from fractions import Fraction

import numpy as np
import torch

import workloads as W
from oracle import formats as F
from oracle import gemm as G
from oracle import nvfp4 as N
from oracle import routing as R
from oracle import storage as S


def _fr(x):
    return Fraction(float(x))


def _random_linear(rng, out, K, n_seg=1):
    w = F.bf16_round((rng.standard_normal((out, K)) * 0.02).astype(np.float32))
    return S.quantize_weight(w, n_seg)


def test_grouped_gemm_matches_exact_rationals():
    rng = np.random.default_rng(21)
    E, M, K = 3, 6, 64
    linears = [_random_linear(rng, M, K) for _ in range(E)]
    counts = [2, 0, 3]
    off = np.concatenate([[0], np.cumsum(counts)])
    S_ = int(off[-1])
    x = (rng.standard_normal((S_, K)) * 2).astype(np.float32)
    g_act = np.float32([0.004, 0.01, 0.0021])
    e_of = R.slot_expert(off)
    a_codes, a_sf = N.quantize_groups(x, g_act[e_of])
    y, bound = G.grouped_gemm_exact([G.weight_int(l) for l in linears], [l["g"][0] for l in linears],
                                    G.dequant_int(a_codes, a_sf), g_act, off)
    for s in range(S_):
        e = e_of[s]
        st = linears[e]
        wcodes = N.unpack_codes(S.decode(st["packed"], st["mask"]))
        for m in range(M):
            acc, ab = Fraction(0), Fraction(0)
            for k in range(K):
                wv = _fr(F.e2m1_decode(wcodes[m, k])) * _fr(F.e4m3_decode(st["scale"][m, k // 32]))
                av = _fr(F.e2m1_decode(a_codes[s, k])) * _fr(F.e4m3_decode(a_sf[s, k // 32]))
                acc += wv * av
                ab += abs(wv * av)
            glob = _fr(np.float32(g_act[e])) * _fr(np.float32(st["g"][0]))
            want = acc * glob
            assert abs(Fraction(y[s, m]) - want) <= abs(want) * Fraction(1, 2 ** 50)
            assert abs(Fraction(bound[s, m]) - ab * glob) <= ab * glob * Fraction(1, 2 ** 50)


def test_unit_scales_reduce_to_float64_matmul():
    rng = np.random.default_rng(8)
    M, K, S_ = 16, 128, 9
    nib = rng.choice([3, 5, 6, 9, 10, 12], size=(M, K // 8))
    mask = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    packed = rng.integers(0, 256, (M, K // 4)).astype(np.uint8)
    ones = np.full((M, K // 32), 0x38, np.uint8)                  # E4M3 1.0
    st = dict(packed=packed, mask=mask, scale=ones, g=np.float32([1.0]))
    a_codes = rng.integers(0, 16, (S_, K)).astype(np.uint8)
    a_sf = np.full((S_, K // 32), 0x38, np.uint8)
    y, _ = G.grouped_gemm_exact([G.weight_int(st)], [np.float32(1)], G.dequant_int(a_codes, a_sf),
                                np.float32([1.0]), np.array([0, S_]))
    Wd = torch.from_numpy(F.e2m1_decode(N.unpack_codes(S.decode(packed, mask))))
    A = torch.from_numpy(F.e2m1_decode(a_codes))
    assert torch.equal(torch.from_numpy(y), A @ Wd.T)


def test_first_half_mask_is_dense_matmul_on_first_pairs():
    rng = np.random.default_rng(9)
    M, K, S_ = 8, 64, 5
    mask = np.full((M, K // 16), 0x33, np.uint8)                  # keep bytes 0,1 of every chunk
    packed = rng.integers(0, 256, (M, K // 4)).astype(np.uint8)
    scale = rng.integers(0x30, 0x48, (M, K // 32)).astype(np.uint8)
    st = dict(packed=packed, mask=mask, scale=scale, g=np.float32([0.5]))
    a_codes = rng.integers(0, 16, (S_, K)).astype(np.uint8)
    a_sf = rng.integers(0x30, 0x48, (S_, K // 32)).astype(np.uint8)
    y, _ = G.grouped_gemm_exact([G.weight_int(st)], [np.float32(0.5)], G.dequant_int(a_codes, a_sf),
                                np.float32([0.25]), np.array([0, S_]))
    # kept weights: elements 0..3 of each 8-element chunk are the 4 codes of packed bytes 2c, 2c+1
    wk = F.e2m1_decode(N.unpack_codes(packed)).reshape(M, K // 8, 4)
    ws = np.repeat(F.e4m3_decode(scale), 32, axis=1).reshape(M, K // 8, 8)[..., :4]
    a = (F.e2m1_decode(a_codes) * np.repeat(F.e4m3_decode(a_sf), 32, axis=1)).reshape(S_, K // 8, 8)[..., :4]
    want = torch.from_numpy(a.reshape(S_, -1)) @ torch.from_numpy((wk * ws).reshape(M, -1)).T * 0.125
    assert torch.allclose(torch.from_numpy(y), want, rtol=1e-14, atol=0)


def test_silu_and_swiglu_gate_first():
    x = np.linspace(-30, 30, 601)
    assert np.allclose(G.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(), rtol=1e-14, atol=1e-300)
    gu = np.array([[0.0, 2.0, 5.0, -1.0], [40.0, -40.0, 1.0, 1.0]])   # I = 2: gate cols 0,1 ; up cols 2,3
    h = G.swiglu(gu)
    assert h[0, 0] == 0.0                                      # silu(0) = 0
    assert np.isclose(h[0, 1], 2.0 / (1 + np.exp(-2.0)) * -1.0)
    assert np.isclose(h[1, 0], 40.0, rtol=1e-15)               # silu(40) ~ 40, up = 1
    assert abs(h[1, 1]) < 1e-15


def test_moe_forward_composition_tiny_exact():
    """A small layer, the expert MLP recomputed with exact rationals per slot."""
    cfg = W.LayerConfig("pin", 31, 3, 2, 64, 32, (5,), "uniform", True)
    rng = np.random.default_rng(31)
    gu = [S.quantize_weight(F.bf16_round((rng.standard_normal((64, 64)) * 0.02).astype(np.float32)), 2)
          for _ in range(3)]
    dn = [S.quantize_weight(F.bf16_round((rng.standard_normal((64, 32)) * 0.02).astype(np.float32)), 1)
          for _ in range(3)]
    x = torch.randn(5, 64, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    ids, w = W.route(torch.randn(5, 3, generator=torch.Generator().manual_seed(4)), cfg.k)
    g_in_gu = np.float32([W.activation_global_scale_input(x)] * 3)
    g_in_dn = np.float32([0.003, 0.002, 0.004])
    res = G.moe_forward(x.float().numpy(), ids.numpy(), w.numpy(), gu, dn, g_in_gu, g_in_dn, 3)

    def exact_linear(st, scale, g0, codes, sf, gact):
        wc = N.unpack_codes(S.decode(st["packed"], st["mask"]))
        rows, K = wc.shape
        out = []
        for m in range(rows):
            acc = Fraction(0)
            for k in range(K):
                acc += (_fr(F.e2m1_decode(wc[m, k])) * _fr(F.e4m3_decode(scale[m, k // 32]))
                        * _fr(F.e2m1_decode(codes[k])) * _fr(F.e4m3_decode(sf[k // 32])))
            out.append(float(acc * _fr(g0) * _fr(gact)))
        return np.array(out)

    perm = res["perm"]
    e_of = R.slot_expert(perm["expert_offsets"])
    xs = x.float().numpy()
    for s in range(len(perm["slot_token"])):
        e, t = e_of[s], perm["slot_token"][s]
        c, sf = N.quantize_groups(xs[t][None], g_in_gu[e])
        st = gu[e]
        scale = st["scale"].copy()
        scale[32:] = S.fold_up_scales(scale[32:], st["g"][0], st["g"][1])
        acc = exact_linear(st, scale, st["g"][0], c[0], sf[0], g_in_gu[e])
        assert np.allclose(acc, res["acc_gu"][s], rtol=1e-15, atol=0)
        h = torch.nn.functional.silu(torch.from_numpy(acc[:32])).numpy() * acc[32:]
        assert np.allclose(h, res["h"][s], rtol=1e-14, atol=1e-300)
        hc, hsf = N.quantize_groups(h.astype(np.float32)[None], g_in_dn[e])
        y = exact_linear(dn[e], dn[e]["scale"], dn[e]["g"][0], hc[0], hsf[0], g_in_dn[e])
        assert np.allclose(y, res["y"][s], rtol=1e-15, atol=0)
    ts = perm["token_slot"]
    want = sum(w.numpy()[:, j:j + 1].astype(np.float64) * res["y"][ts[:, j]] for j in range(cfg.k))
    assert np.allclose(res["out"], want, rtol=1e-15, atol=0)


def _split_storage(seed=7, I=64, K=256):
    w = torch.randn((2 * I, K), generator=torch.Generator().manual_seed(seed)) * 0.02
    return S.quantize_weight(w.to(torch.bfloat16).float().numpy(), 2)


def _routed_acts(seed=8, T=24, K=256, E=1):
    x = torch.randn((T, K), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    off = np.array([0, T], np.int64)
    g_in = np.array([np.float32(x.float().abs().max()) / np.float32(2688)], np.float32)
    c, s = G.quant_act(x.float().numpy(), np.arange(T), off, g_in)
    return G.dequant_int(c, s), g_in, off


def test_unfolded_gate_up_equals_float64_matmul_of_decoded_halves():
    """Each half with its own global ("exact per-half alpha"): the exact int64 path
    against a float64 matmul of the decoded values times scales times globals."""
    st = _split_storage()
    A, g_in, off = _routed_acts()
    acc, _ = G.gate_up_exact([st], A, g_in, off, fold=False)
    codes = N.unpack_codes(S.decode(st["packed"], st["mask"]))
    Wd = F.e2m1_decode(codes) * np.repeat(F.e4m3_decode(st["scale"]), 32, axis=1)
    g = np.asarray(st["g"], np.float64)
    I = Wd.shape[0] // 2
    Wd[:I] *= g[0]
    Wd[I:] *= g[1]
    ref = (torch.from_numpy(A.astype(np.float64) * 2.0 ** -10) @ torch.from_numpy(Wd).T).numpy() * np.float64(g_in[0])
    assert np.allclose(acc, ref, rtol=1e-12, atol=1e-300)


def test_fold_is_exact_for_a_power_of_two_ratio():
    """With g_up = g_gate / 2 and every up scale representable at half its value, the
    pages' fold loses nothing: the folded and the per-half paths agree exactly."""
    st = dict(_split_storage())
    g0 = np.float32(st["g"][0])
    st["g"] = np.array([g0, g0 * np.float32(0.5)], np.float32)
    sc = np.array(st["scale"], np.uint8, copy=True)
    I = sc.shape[0] // 2
    vals = F.e4m3_decode(sc[I:])
    ok = (vals >= 2.0 ** -5) & (vals <= 448)          # halving stays a normal E4M3 value
    sc[I:] = np.where(ok, sc[I:], np.uint8(0x38))      # elsewhere 1.0
    st["scale"] = sc
    assert (F.e4m3_decode(S.fold_up_scales(sc[I:], st["g"][0], st["g"][1])) == F.e4m3_decode(sc[I:]) / 2).all()
    A, g_in, off = _routed_acts(seed=9)
    a, _ = G.gate_up_exact([st], A, g_in, off, fold=True)
    b, _ = G.gate_up_exact([st], A, g_in, off, fold=False)
    assert np.array_equal(a, b)


def test_int_matmul_exact_equals_int64_product():
    """The float64 route of the exact GEMM equals the int64 product (its definition),
    including operands at the largest quantised magnitude (12 * 448 * 512) and the
    deepest K of the layer shapes, where every term has the same sign."""
    rng = np.random.default_rng(31)
    top = 12 * 448 * 512
    for n, m, K in ((7, 5, 64), (33, 17, 7168), (3, 4, 4096)):
        a = rng.integers(-top, top + 1, (n, K), dtype=np.int64)
        w = rng.integers(-top, top + 1, (m, K), dtype=np.int64)
        assert np.array_equal(G.int_matmul_exact(a, w), a @ w.T)
    a = np.full((2, 7168), top, np.int64)
    w = np.full((3, 7168), -top, np.int64)
    w[1] = top
    assert np.array_equal(G.int_matmul_exact(a, w), a @ w.T)
    assert G.int_matmul_exact(np.zeros((0, 8), np.int64), np.ones((2, 8), np.int64)).shape == (0, 2)
