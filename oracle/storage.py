"""Paired-4:8 pruning, pair-bitmask storage and the tensor-core layouts (CPU oracle).

Test infrastructure only.  Sources, by page:

* "Compression details" table, Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card:
  paired 4:8 sparsity along K -- in every 8 consecutive elements (4 pairs)
  exactly 2 pairs are kept.
* "Sparse storage layout (paired48_sparse, pair-bitmask v1)", same card:
  one pair is one packed-NVFP4 byte, so every 4-byte chunk keeps exactly 2
  bytes.  ``weight_sparse_packed`` uint8 [out, K/4] holds the 2 kept bytes of
  every 4 in K order; ``weight_sparse_mask`` uint8 [out, K/16] holds 4 bits per
  chunk (exactly 2 set, bit i means byte i is kept, the low nibble is the
  lower-K chunk); ``weight_scale`` E4M3 [out, K/32]; the conversion to and from
  dense NVFP4 is lossless.
* MoESQ repository README, "Usage" (Output bullet): ``--no-sparse-storage``
  writes dense packed NVFP4 with the pruned elements zeroed; a tool converts
  losslessly between the two.
* Qwen3.8-Flash-Next-P48NVFP4-MoESQ and Qwen3-30B-A3B-P48NVFP4-MoESQ model
  cards: gate and up carry separate global scales and their ratio is folded
  into the block scales at load time (upstream would apply the gate scale to
  both).

Readings where the pages are silent (each listed in the design notes):
* pruning score of a pair (a, b) is a*a + b*b in fp32 on the bf16 values; the
  2 highest-scoring pairs of each 8-element chunk are kept, ties to the lower
  pair index (the synthetic recipe: "keep the 2 highest-L2 pairs of every 4");
* a kept byte may quantise to 0x00, so "2 nonzero bytes" reads as "2 kept
  bytes"; encoding without a mask marks the nonzero bytes and fills up to 2
  with the lowest-index zero bytes (more than 2 nonzero bytes is an error);
* the gate/up fold keeps the gate global and multiplies each up block scale
  by g_up / g_gate, re-rounded to E4M3 (nearest even, saturating).
"""
from __future__ import annotations

import numpy as np

from .formats import e4m3_decode, e4m3_quantize, f32
from .nvfp4 import global_scale, pack_codes, quantize_groups


class SparsityError(ValueError):
    """A chunk violates paired-4:8 structure (bad mask nibble or >2 nonzero bytes)."""


# ----------------------------------------------------------------- pruning ---

def prune_paired48(w) -> np.ndarray:
    """Keep-mask per pair for bf16 weights ``w [rows, K]`` (given as float32 values).

    Returns bool [rows, K/2]: True where the pair (elements 2p, 2p+1) is kept.
    """
    w = f32(w)
    rows, K = w.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    a, b = w[:, 0::2], w[:, 1::2]
    score = f32(f32(a * a) + f32(b * b)).reshape(rows, K // 8, 4)
    # rank pairs by descending score; stable sort keeps the lower index first on ties
    order = np.argsort(-score, axis=-1, kind="stable")
    keep = np.zeros_like(score, dtype=bool)
    np.put_along_axis(keep, order[..., :2], True, axis=-1)
    return keep.reshape(rows, K // 2)


def keep_to_mask(keep) -> np.ndarray:
    """Pair keep-flags [rows, K/2] -> weight_sparse_mask bytes [rows, K/16]."""
    keep = np.asarray(keep, dtype=np.uint8)
    rows, npair = keep.shape
    kc = keep.reshape(rows, npair // 4, 4)
    nib = kc[..., 0] | (kc[..., 1] << 1) | (kc[..., 2] << 2) | (kc[..., 3] << 3)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def mask_nibbles(mask) -> np.ndarray:
    """weight_sparse_mask bytes [rows, K/16] -> one nibble per chunk [rows, K/8]."""
    m = np.asarray(mask, dtype=np.uint8)
    out = np.empty(m.shape[:-1] + (m.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = m & 0xF
    out[..., 1::2] = m >> 4
    return out


_POPC4 = np.array([bin(i).count("1") for i in range(16)], dtype=np.int64)


# ------------------------------------------------------------ weight export ---

def quantize_weight(w_bf16, n_seg: int = 1):
    """Prune and quantise one expert linear to pair-bitmask storage.

    ``w_bf16`` float32 values of a bf16 [out, K] weight; ``n_seg`` equal row
    segments each get their own FP32 global (2 = fused gate_up with separate
    gate and up globals).  Returns dict(packed [out,K/4], mask [out,K/16],
    scale [out,K/32] E4M3 codes, g [n_seg] float32, dense [out,K/2] packed
    NVFP4 with pruned bytes zero).
    """
    w = f32(w_bf16)
    out, K = w.shape
    if out % n_seg:
        raise ValueError("rows not divisible into segments")
    keep = prune_paired48(w)
    pruned = np.where(np.repeat(keep, 2, axis=1), w, np.float32(0))
    seg = out // n_seg
    g = np.array([global_scale(np.abs(pruned[i * seg:(i + 1) * seg]).max()) for i in range(n_seg)],
                 dtype=np.float32)
    g_row = np.repeat(g, seg)
    codes, scale = quantize_groups(pruned, g_row)
    dense = pack_codes(codes)
    mask = keep_to_mask(keep)
    packed, mask2 = encode(dense, mask)
    assert np.array_equal(mask, mask2)
    return dict(packed=packed, mask=mask, scale=scale, g=g, dense=dense)


# ----------------------------------------------------------- encode/decode ---

def _kept_positions(nib):
    """Ascending byte positions (pos0 < pos1) of the 2 set bits of each nibble."""
    nib = np.asarray(nib, dtype=np.int64)
    if (_POPC4[nib] != 2).any():
        raise SparsityError("mask nibble without exactly 2 bits set")
    lowest = np.array([(n & -n).bit_length() - 1 if n else 0 for n in range(16)])
    highest = np.array([n.bit_length() - 1 if n else 0 for n in range(16)])
    return lowest[nib], highest[nib]


def decode(packed, mask) -> np.ndarray:
    """pair-bitmask -> dense packed NVFP4 bytes [rows, K/2] (pruned bytes 0).

    Chunk c (dense bytes 4c..4c+3) takes packed bytes 2c and 2c+1, placed at
    the positions of the two set mask bits in ascending order.
    """
    packed = np.asarray(packed, dtype=np.uint8)
    nib = mask_nibbles(mask)
    rows, nchunk = nib.shape
    if packed.shape != (rows, 2 * nchunk):
        raise ValueError("packed/mask shape mismatch")
    p0, p1 = _kept_positions(nib)
    pk = packed.reshape(rows, nchunk, 2)
    dense = np.zeros((rows, nchunk, 4), dtype=np.uint8)
    np.put_along_axis(dense, p0[..., None], pk[..., 0:1], axis=-1)
    np.put_along_axis(dense, p1[..., None], pk[..., 1:2], axis=-1)
    return dense.reshape(rows, nchunk * 4)


def encode(dense, mask_hint=None):
    """dense packed NVFP4 [rows, K/2] -> (packed [rows, K/4], mask [rows, K/16]).

    With ``mask_hint`` the kept bytes are the hinted ones (the bytes outside the
    hint must be zero).  Without it the nonzero bytes are kept and the chunk is
    filled up to 2 with its lowest-index zero bytes.
    """
    dense = np.asarray(dense, dtype=np.uint8)
    rows, nb = dense.shape
    if nb % 8:
        raise ValueError("K/2 must be a multiple of 8")
    d = dense.reshape(rows, nb // 4, 4)
    bit = (1 << np.arange(4)).astype(np.int64)
    if mask_hint is not None:
        nib = mask_nibbles(mask_hint).astype(np.int64)
        if nib.shape != d.shape[:2]:
            raise ValueError("mask_hint shape mismatch")
    else:
        nz = d != 0
        cnt = nz.sum(axis=-1)
        if (cnt > 2).any():
            raise SparsityError("chunk with more than 2 nonzero bytes")
        zero_rank = np.cumsum(~nz, axis=-1)                 # 1-based rank among zero bytes
        fill = (~nz) & (zero_rank <= (2 - cnt)[..., None])
        nib = ((nz | fill) * bit).sum(axis=-1)
    p0, p1 = _kept_positions(nib)
    kept = ((nib[..., None] & bit) != 0)
    if ((d != 0) & ~kept).any():
        raise SparsityError("nonzero byte outside the kept pair positions")
    b0 = np.take_along_axis(d, p0[..., None], axis=-1)[..., 0]
    b1 = np.take_along_axis(d, p1[..., None], axis=-1)[..., 0]
    packed = np.stack([b0, b1], axis=-1).reshape(rows, nb // 2).astype(np.uint8)
    nib = nib.astype(np.uint8)
    mask = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return packed, mask


# ------------------------------------------------------------- gate/up fold ---

def fold_up_scales(scale_up, g_gate, g_up) -> np.ndarray:
    """Up block scales with the ratio g_up / g_gate folded in (E4M3 re-rounded)."""
    ratio = np.float32(f32(g_up) / f32(g_gate))
    return e4m3_quantize(f32(f32(e4m3_decode(scale_up)) * ratio))


# ----------------------------------------------- tensor-core operand layouts ---
# The sparse block-scaled FP4 MMA of sm_100a (tcgen05.mma.sp ... mxf4nvf4) reads
#   * sparse metadata: per 8-element chunk (4 pairs) two 2-bit pair indices
#     i0 < i1, nibble = i0 | i1 << 2; two chunks per byte, lower-K chunk in the
#     low nibble; 128 rows x 16 bytes (256 dense K) per block, row r at 16*r;
#   * block scales: per 128 rows and 4 scales (128 dense K) a 512-byte block,
#     row r scale j at (r % 32) * 16 + (r // 32) * 4 + j.
# The library lays out whole operands as
#   meta[e][tile][kb256][128][16]   sfw[e][tile][kb128][512]   sfa[pb][kb128][512]
# where "tile" is a 128-row block of the weight in tile row order.  For down,
# tile t holds rows 128t..128t+127 with neighbouring rows 8 apart inside each
# 16-row group (tile row 16g + 8p + j is row 128t + 16g + 2j + p), so that one TMEM
# load gives a thread both outputs of a bf16 pair.  For fused gate_up, tile t holds the gate and the up rows of the same
# 64 outputs 64t..64t+63, interleaved so that the SwiGLU epilogue finds a gate
# value and its up value, for two adjacent outputs, in one thread: tile row
# r = 32q + 16h + 8s + j (q < 4, h, s < 2, j < 8) is output f = 64t + 16q + 2j + h
# of the gate rows (s = 0) or of the up rows (s = 1, source row I + f).  This row
# order is the library's own layout choice; the pages fix none.

def meta_nibble_from_mask_nibble(n: int) -> int:
    pos = [i for i in range(4) if (n >> i) & 1]
    if len(pos) != 2:
        raise SparsityError("mask nibble without exactly 2 bits set")
    return pos[0] | (pos[1] << 2)


def tile_rows(out: int, gate_up: bool) -> np.ndarray:
    """Source weight row of each tile row, concatenated over tiles."""
    if out % 128:
        raise ValueError("out must be a multiple of 128")
    if not gate_up:
        r = np.arange(out)
        return (r // 16) * 16 + 2 * (r % 8) + (r // 8) % 2
    I = out // 2
    rows = []
    for t in range(out // 128):
        for r in range(128):
            q, h, s, j = r // 32, (r // 16) % 2, (r // 8) % 2, r % 8
            rows.append(s * I + 64 * t + 16 * q + 2 * j + h)
    return np.array(rows)


def repack_meta(mask, gate_up: bool) -> np.ndarray:
    """One expert's weight_sparse_mask [out, K/16] -> metadata blocks (flat uint8)."""
    nib = mask_nibbles(mask)
    out, nchunk = nib.shape
    K = nchunk * 8
    if K % 128:
        raise ValueError("K must be a multiple of 128")
    lut = np.array([meta_nibble_from_mask_nibble(n) if _POPC4[n] == 2 else 0xFF
                    for n in range(16)], dtype=np.int64)
    meta = lut[nib]
    if (meta == 0xFF).any():
        raise SparsityError("mask nibble without exactly 2 bits set")
    meta = meta[tile_rows(out, gate_up)]                    # rows in tile order
    nkb = (K + 255) // 256
    pad = np.zeros((out, nkb * 32), dtype=np.int64)
    pad[:, :nchunk] = meta
    byte = pad[:, 0::2] | (pad[:, 1::2] << 4)               # [out, nkb*16]
    res = byte.reshape(out // 128, 128, nkb, 16).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(res).astype(np.uint8).reshape(-1)


def sf_block_offset(r: int, j: int) -> int:
    return (r % 32) * 16 + (r // 32) * 4 + j


def repack_weight_scales(scale, gate_up: bool) -> np.ndarray:
    """One expert's block scales [out, K/32] (already folded) -> SF blocks (flat uint8)."""
    scale = np.asarray(scale, dtype=np.uint8)
    out, ng = scale.shape
    K = ng * 32
    if K % 128:
        raise ValueError("K must be a multiple of 128")
    sc = scale[tile_rows(out, gate_up)].reshape(out // 128, 128, K // 128, 4)
    res = np.zeros((out // 128, K // 128, 512), dtype=np.uint8)
    r = np.arange(128)
    for j in range(4):
        off = (r % 32) * 16 + (r // 32) * 4 + j
        res[:, :, off] = sc[:, :, :, j].transpose(0, 2, 1)
    return res.reshape(-1)


def repack_linear(storage_per_expert, kind: str, fold: bool = True):
    """Load-time repack of one linear over all experts.

    ``storage_per_expert``: list of dicts (packed, mask, scale, g) per expert.
    kind: "gate_up" (fused, g has 1 or 2 entries) or "down".
    Returns dict(meta, sf, alpha) where alpha[e] is the FP32 weight global the
    kernel applies (the gate global for gate_up).  With two gate_up globals and
    ``fold`` False, the up scales are left as stored and alpha holds both
    globals per expert, [E, 2] flattened (gate, up).
    """
    gate_up = kind == "gate_up"
    metas, sfs, alpha = [], [], []
    for st in storage_per_expert:
        scale = np.array(st["scale"], dtype=np.uint8, copy=True)
        g = np.asarray(st["g"], dtype=np.float32).reshape(-1)
        if gate_up and g.size == 2 and fold:
            I = scale.shape[0] // 2
            scale[I:] = fold_up_scales(scale[I:], g[0], g[1])
        metas.append(repack_meta(st["mask"], gate_up))
        sfs.append(repack_weight_scales(scale, gate_up))
        if gate_up and g.size == 2 and not fold:
            alpha.extend([g[0], g[1]])
        else:
            alpha.append(g[0])
    return dict(meta=np.concatenate(metas), sf=np.concatenate(sfs),
                alpha=np.array(alpha, dtype=np.float32))


def storage_bytes_per_dense_element() -> tuple:
    """(sparse, dense) bytes per dense weight element of the two storage forms."""
    sparse = 1 / 4 + 1 / 16 + 1 / 32     # kept bytes + mask + E4M3 scale
    dense = 1 / 2 + 1 / 32               # packed NVFP4 + E4M3 scale
    return sparse, dense
