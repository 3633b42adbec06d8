"""Helpers shared by the GPU parity tests: build device layers from oracle
storage, convert padded kernel layouts back to per-slot rows for comparison,
and bound the effect of legitimate rounding-boundary flips in requantised
activations.  Only comparison logic lives here; every expected value comes from
the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import formats as F
from oracle import gemm as G
from oracle import nvfp4 as N
from oracle import routing as R
from oracle import storage as S

KIND_DOWN, KIND_GATE_UP, KIND_GATE_UP_SPLIT, KIND_GATE_UP_EXACT = 0, 1, 2, 3


def cuda(a, dtype=None):
    t = torch.as_tensor(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def storage_to_device(storages):
    """List of oracle storage dicts (one per expert) -> stacked device tensors."""
    st = dict(packed=cuda(np.stack([s["packed"] for s in storages])),
              mask=cuda(np.stack([s["mask"] for s in storages])),
              scale=cuda(np.stack([s["scale"] for s in storages])),
              g_w=cuda(np.stack([np.asarray(s["g"], np.float32).reshape(-1) for s in storages])))
    E, out, K4 = st["packed"].shape
    st.update(E=E, out=out, K=K4 * 4)
    return st


def kernel_rows_to_slots(codes_pad, sf_blocks, expert_offsets, pad_offsets, K):
    """Padded operand (codes [P, K/2], 512-byte scale blocks) -> per-slot linear
    (codes [S, K/2], scales [S, K/32]) using the documented block layout."""
    off = np.asarray(expert_offsets, np.int64)
    rows = R.padded_row_of_slot(off, pad_offsets)
    codes = np.asarray(codes_pad)[rows]
    sfb = np.asarray(sf_blocks).reshape(-1, K // 128, 512)
    Sn = rows.size
    sf = np.empty((Sn, K // 32), np.uint8)
    r = rows % 128
    for g in range(K // 32):
        off_in = (r % 32) * 16 + (r // 32) * 4 + (g % 4)
        sf[:, g] = sfb[rows // 128, g // 4, off_in]
    return codes, sf


def oracle_layer(cfg, T, experts_storage_gu, experts_storage_dn, x_bf16, ids, w, g_in_gu, g_in_dn):
    return G.moe_forward(x_bf16, ids, w, experts_storage_gu, experts_storage_dn, g_in_gu, g_in_dn,
                         cfg.E)


def calibrate_g_in_down(acc_gu, expert_offsets, E):
    """Static down-input globals from an exact gate_up pass: amax(h_e) / (6*448)
    per expert (median of the nonempty experts for empty ones)."""
    h = G.swiglu(acc_gu)
    off = np.asarray(expert_offsets)
    g = np.zeros(E, np.float32)
    for e in range(E):
        if off[e + 1] > off[e]:
            g[e] = np.float32(np.float32(np.abs(h[off[e]:off[e + 1]]).max()) / np.float32(2688))
    nz = g[g > 0]
    g[g == 0] = np.median(nz) if nz.size else np.float32(1e-3)
    return g


# ------------------------------------------------------ requant ambiguity ---

def e2m1_bracket(v_lo, v_hi):
    """Codes of the two ends of an interval of pre-rounding values."""
    return N.e2m1_quantize(np.float32(v_lo)), N.e2m1_quantize(np.float32(v_hi))


def requant_analysis(h_exact, err_h, g_next):
    """For exact activations h [rows, I] with absolute error bounds err_h on the
    kernel's float32 values, return which codes/scales the NVFP4 rule fixes
    uniquely and, for the rest, the largest possible change of the dequantised
    value.  g_next: [rows] float32 globals.

    Returns dict(codes, sc (oracle's), code_fixed bool [rows,I], sc_fixed bool
    [rows, I/32], max_dev float64 [rows, I] bound on |deq_gpu - deq_oracle|).
    """
    h = np.asarray(h_exact, np.float64)
    rows, I = h.shape
    codes, sc = N.quantize_groups(h.astype(np.float32), np.asarray(g_next, np.float32))
    g = np.asarray(g_next, np.float64).reshape(-1, 1)
    hg = h.reshape(rows, I // 32, 32)
    eg = np.asarray(err_h, np.float64).reshape(rows, I // 32, 32) + np.abs(hg) * 2.0 ** -22
    amax = np.abs(hg).max(-1)
    emax = eg.max(-1)
    six_g = (6.0 * g).astype(np.float32).astype(np.float64)
    s_lo = np.maximum(amax - emax, 0) / six_g
    s_hi = (amax + emax) / six_g
    sc_lo = F.e4m3_quantize(s_lo.astype(np.float32) * np.float32(1 - 2 ** -22))
    sc_hi = F.e4m3_quantize((s_hi * (1 + 2 ** -22)).astype(np.float32))
    sc_fixed = (sc_lo == sc_hi)
    max_dev = np.zeros_like(hg)
    code_fixed = np.ones_like(hg, dtype=bool)
    deq_ref = F.e2m1_decode(codes).reshape(rows, I // 32, 32) * (F.e4m3_decode(sc) * g)[..., None]
    for cand in {0, 1}:
        sc_c = np.where(cand == 0, sc_lo, sc_hi)
        sdq = (F.e4m3_decode(sc_c) * g).astype(np.float32).astype(np.float64)
        with np.errstate(divide="ignore"):
            inv = np.where(sdq == 0, 0.0, (np.float32(1) / sdq.astype(np.float32)).astype(np.float64))
        v_lo = (hg - eg) * inv[..., None]
        v_hi = (hg + eg) * inv[..., None]
        c_lo = F.e2m1_decode(N.e2m1_quantize(np.float32(v_lo * (1 - 2 ** -22))))
        c_hi = F.e2m1_decode(N.e2m1_quantize(np.float32(v_hi * (1 + 2 ** -22))))
        d_lo = np.abs(c_lo * sdq[..., None] - deq_ref)
        d_hi = np.abs(c_hi * sdq[..., None] - deq_ref)
        max_dev = np.maximum(max_dev, np.maximum(d_lo, d_hi))
        code_fixed &= (c_lo == c_hi)
    code_fixed &= sc_fixed[..., None]
    return dict(codes=codes, sc=sc, code_fixed=code_fixed.reshape(rows, I), sc_fixed=sc_fixed,
                max_dev=max_dev.reshape(rows, I))


def swiglu_error_bound(acc_gu, bound_gu, rel=1e-5):
    """Bound on |h_gpu - h_exact| from the gate_up accumulator tolerance."""
    a = np.asarray(acc_gu, np.float64)
    b = np.asarray(bound_gu, np.float64)
    I = a.shape[1] // 2
    gte, up = a[:, :I], a[:, I:]
    eg = rel * b[:, :I] + np.abs(gte) * 2.0 ** -22
    eu = rel * b[:, I:] + np.abs(up) * 2.0 ** -22
    sg = G.silu(gte)
    # |silu'| <= 1.1 everywhere; plus the float32 evaluation of silu and the product
    return 1.1 * (np.abs(up) + eu) * eg + np.abs(sg) * eu + 1e-5 * np.abs(sg * up) + 1e-30


def forward_error_limit(ref, down_storages, g_in_dn, topk_w, tol=1e-5):
    """Per-element bound on |out_gpu - out_exact| of the whole expert MLP.

    ref: the oracle's G.moe_forward result.  The bound adds, per slot, the down GEMM
    tolerance, the largest effect of a legitimate requantisation flip of h (propagated
    through |W_down|), the bf16 rounding of y, then combines with |w| in j order and
    adds the final bf16 rounding.
    """
    off = ref["perm"]["expert_offsets"]
    e_of = R.slot_expert(off)
    an = requant_analysis(ref["h"], swiglu_error_bound(ref["acc_gu"], ref["bound_gu"], tol),
                          np.asarray(g_in_dn, np.float32)[e_of])
    flip = np.zeros_like(ref["y"])
    for e, st in enumerate(down_storages):
        if off[e + 1] > off[e]:
            wabs = np.abs(G.weight_int(st)).astype(np.float64) * 2.0 ** -10 * np.float64(st["g"][0])
            flip[off[e]:off[e + 1]] = an["max_dev"][off[e]:off[e + 1]] @ wabs.T
    y_lim = tol * ref["bound_d"] + flip + bf16_ulp(ref["y"]) + bf16_ulp(ref["y"] + flip)
    ts = ref["perm"]["token_slot"]
    w = np.asarray(topk_w)
    lim = sum(np.abs(w[:, j:j + 1]).astype(np.float64) * y_lim[ts[:, j]] for j in range(ts.shape[1]))
    return lim + bf16_ulp(np.abs(ref["out"]) + lim) + 1e-30


def bf16_ulp(v):
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)
