"""Exact grouped expert GEMMs, SwiGLU and the MoE layer (CPU oracle).

Test infrastructure only.  What the method computes is a quantised sparse
GEMM with a plain definition, so this oracle writes that definition out:

  y[s, m] = g_act[e] * g_w[e] * sum_k  W(m, k) * A(s, k)
  W(m, k) = E2M1(w_mk) * E4M3(sw_m,k/32)          (pruned elements are 0)
  A(s, k) = E2M1(a_sk) * E4M3(sa_s,k/32)

for every slot s routed to expert e ("Compression details" table of the
Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card: NVFP4 weights and activations,
E4M3 scale per 32 dense K, FP32 per-tensor globals; the grouped GEMM is the
kernel line of the same card).

The inner sum is exact: E2M1 values are integers in units of 1/2 and E4M3
values integers in units of 2**-9, so every product W*A is an integer in units
of 2**-20 below 2**44 in magnitude, and sums over K <= 7168 fit in int64.  The
FP32 globals are applied in float64 afterwards.

The expert MLP is SwiGLU over the fused gate_up weight (gate rows first):
h = silu(gate) * up with silu(x) = x / (1 + exp(-x)), then NVFP4 requantisation
of h with the per-expert down input global, then the down GEMM ("gate_proj,
up_proj, down_proj" are the compressed linears; the kernels carry the
activation, MoESQ repository README).
"""
from __future__ import annotations

import numpy as np

from .formats import E2M1_MAG, bf16_round, e4m3_decode, f32
from .nvfp4 import quantize_groups, unpack_codes
from .routing import permute, unpermute
from .storage import decode

_E2M1_HALVES = np.array([int(round(2 * v)) for v in E2M1_MAG], dtype=np.int64)   # 0..12


def e2m1_int(codes) -> np.ndarray:
    """E2M1 codes -> integer values in units of 1/2 (range -12..12)."""
    c = np.asarray(codes).astype(np.int64)
    v = _E2M1_HALVES[c & 7]
    return np.where(c & 8, -v, v)


def e4m3_int(b) -> np.ndarray:
    """Finite nonnegative E4M3 codes -> integer values in units of 2**-9."""
    v = e4m3_decode(b) * 512.0
    if np.isnan(v).any() or (v < 0).any():
        raise ValueError("block scale must be a finite nonnegative E4M3 value")
    vi = np.rint(v).astype(np.int64)
    assert np.array_equal(vi.astype(np.float64), v)
    return vi


def dequant_int(codes, scales) -> np.ndarray:
    """Per-element codes [rows, K] and E4M3 block scales [rows, K/32] -> int64 in units of 2**-10."""
    c = e2m1_int(codes)
    s = np.repeat(e4m3_int(scales), 32, axis=1)
    return c * s


def weight_int(storage) -> np.ndarray:
    """Pair-bitmask storage of one expert linear -> int64 W in units of 2**-10, [out, K]."""
    dense = decode(storage["packed"], storage["mask"])
    return dequant_int(unpack_codes(dense), storage["scale"])


def int_matmul_exact(a, w) -> np.ndarray:
    """a @ w.T for int64 a [n, K] and w [m, K], exactly, by float64 matrix products.

    The quantised operands are integers below 2**22 in magnitude (units of 2**-10:
    at most 12 halves times 448 * 512).  Writing a = hi * 2**11 + lo with
    0 <= lo < 2**11 makes both |hi| and |lo| at most 2**11, so every product with
    w is an integer below 2**33 and every partial sum over K < 2**19 terms an
    integer below 2**52: float64 represents all of them, and the float64 products
    are exact whatever order the library sums in.  The operand ranges are
    checked; outside them the plain int64 product is used.
    """
    a = np.asarray(a, dtype=np.int64)
    w = np.asarray(w, dtype=np.int64)
    K = a.shape[1]
    if a.size == 0 or w.size == 0:
        return np.zeros((a.shape[0], w.shape[0]), dtype=np.int64)
    wmax = int(np.abs(w).max())
    if int(np.abs(a).max()) >= 2 ** 22 or wmax * (2 ** 11) * K >= 2 ** 52:
        return a @ w.T
    hi = a >> 11
    lo = a - (hi << 11)
    wf = w.astype(np.float64).T
    r_hi = hi.astype(np.float64) @ wf
    r_lo = lo.astype(np.float64) @ wf
    return (r_hi.astype(np.int64) << 11) + r_lo.astype(np.int64)


def grouped_gemm_exact(W_int, g_w, A_int, g_act, expert_offsets):
    """Exact grouped GEMM.

    W_int: list over experts of int64 [M, K] (units 2**-10); g_w: [E] float32
    weight globals; A_int: int64 [S, K] routed activations (units 2**-10);
    g_act: [E] float32 activation globals; expert_offsets: [E+1].
    Returns (y float64 [S, M], absbound float64 [S, M]) where absbound is
    sum_k |W A| with the same globals applied (the per-element error scale).
    """
    off = np.asarray(expert_offsets, dtype=np.int64)
    S, K = A_int.shape
    M = W_int[0].shape[0] if len(W_int) else 0
    y = np.zeros((S, M), dtype=np.float64)
    bound = np.zeros((S, M), dtype=np.float64)
    for e in range(off.size - 1):
        s0, s1 = off[e], off[e + 1]
        if s1 == s0:
            continue
        a = A_int[s0:s1]
        w = W_int[e]
        acc = int_matmul_exact(a, w)                    # exact
        aab = int_matmul_exact(np.abs(a), np.abs(w))
        scale = float(np.float64(g_act[e]) * np.float64(g_w[e])) * 2.0 ** -20
        y[s0:s1] = acc.astype(np.float64) * scale
        bound[s0:s1] = aab.astype(np.float64) * abs(scale)
    return y, bound


def gate_up_exact(storage_per_expert, A_int, g_act, expert_offsets, fold=True):
    """The fused gate_up GEMM over the routed activations, exact.

    ``storage_per_expert``: list of storage dicts (packed, mask, scale, g) of the
    fused [2I, K] weight, gate rows first.  With one global, or with two and
    ``fold`` (the pages' load-time fold, "Compression details"/"Known limitations"
    of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card: the up/gate ratio of the
    globals goes into the up block scales and the gate global serves both halves),
    one pass with g[0].  With two globals and not ``fold``: the gate rows with g[0]
    and the up rows with g[1], each with its own unfolded scales.
    Returns (acc float64 [S, 2I], absbound float64 [S, 2I]).
    """
    from .storage import fold_up_scales

    gs = [np.asarray(st["g"], dtype=np.float32).reshape(-1) for st in storage_per_expert]
    split = any(g.size == 2 for g in gs)
    if not split or fold:
        W, gw = [], []
        for st, g in zip(storage_per_expert, gs):
            scale = np.array(st["scale"], dtype=np.uint8, copy=True)
            if g.size == 2:
                I = scale.shape[0] // 2
                scale[I:] = fold_up_scales(scale[I:], g[0], g[1])
            W.append(dequant_int(unpack_codes(decode(st["packed"], st["mask"])), scale))
            gw.append(g[0])
        return grouped_gemm_exact(W, gw, A_int, g_act, expert_offsets)
    Wfull = [weight_int(st) for st in storage_per_expert]
    I = Wfull[0].shape[0] // 2
    yg, bg = grouped_gemm_exact([w[:I] for w in Wfull], [g[0] for g in gs], A_int, g_act, expert_offsets)
    yu, bu = grouped_gemm_exact([w[I:] for w in Wfull], [g[1] for g in gs], A_int, g_act, expert_offsets)
    return np.concatenate([yg, yu], axis=1), np.concatenate([bg, bu], axis=1)


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def swiglu(gate_up) -> np.ndarray:
    """h = silu(gate) * up for a fused [S, 2I] accumulator (gate columns first)."""
    gu = np.asarray(gate_up, dtype=np.float64)
    I = gu.shape[1] // 2
    return silu(gu[:, :I]) * gu[:, I:]


def quant_act(x_bf16, slot_token, expert_offsets, g_in):
    """NVFP4 quantisation of the routed activations, one row per slot.

    Row s is x[slot_token[s]] quantised with the input global of its expert.
    Returns (codes uint8 [S, K], scales uint8 [S, K/32]).
    """
    x = f32(x_bf16)
    st = np.asarray(slot_token, dtype=np.int64)
    off = np.asarray(expert_offsets, dtype=np.int64)
    e_of_slot = np.repeat(np.arange(off.size - 1), np.diff(off))
    g = f32(np.asarray(g_in, dtype=np.float32)[e_of_slot])
    return quantize_groups(x[st], g)


def moe_forward(x_bf16, topk_ids, topk_w, gate_up, down, g_in_gu, g_in_down, E, fold=True):
    """The routed-expert MLP of one MoE layer, every step exact or float64.

    gate_up / down: lists over experts of storage dicts (packed, mask, scale, g);
    gate_up as in gate_up_exact (folded, the default, or each half with its own
    global).  Returns dict with the intermediate results and ``out`` (float64,
    before the final bf16 rounding) and ``out_bf16``.
    """
    perm = permute(topk_ids, E)
    off = perm["expert_offsets"]
    a_codes, a_sf = quant_act(x_bf16, perm["slot_token"], off, g_in_gu)
    A = dequant_int(a_codes, a_sf)

    acc_gu, bound_gu = gate_up_exact(gate_up, A, g_in_gu, off, fold=fold)
    h = swiglu(acc_gu)

    e_of_slot = np.repeat(np.arange(E), np.diff(off))
    h_codes, h_sf = quantize_groups(f32(h), f32(np.asarray(g_in_down, np.float32)[e_of_slot]))
    Hq = dequant_int(h_codes, h_sf)
    Wd = [weight_int(st) for st in down]
    gd = [np.asarray(st["g"], dtype=np.float32).reshape(-1)[0] for st in down]
    y, bound_d = grouped_gemm_exact(Wd, gd, Hq, g_in_down, off)

    ts = perm["token_slot"]
    w = np.asarray(topk_w, dtype=np.float64)
    out = np.zeros((ts.shape[0], y.shape[1]), dtype=np.float64)
    for j in range(ts.shape[1]):
        out += w[:, j:j + 1] * y[ts[:, j]]
    return dict(perm=perm, a_codes=a_codes, a_sf=a_sf, acc_gu=acc_gu, bound_gu=bound_gu,
                h=h, h_codes=h_codes, h_sf=h_sf, y=y, bound_d=bound_d, out=out,
                out_bf16=bf16_round(f32(out)),
                y_bf16_combined=unpermute(bf16_round(f32(y)), ts, topk_w))
