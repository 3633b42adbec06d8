"""Routing permutation and weighted combine of the MoE layer (CPU oracle).

Test infrastructure only.  The pages' kernel is a grouped GEMM over the tokens
the router sends to each expert ("Kernel: paired-4:8 sparse NVFP4 grouped
GEMM", header list of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card); the
router itself stays BF16 ("Left in BF16" row of its "Compression details"
table).  The pages fix neither the slot order nor the combine arithmetic, so:

* slots are ordered by (expert, token, j) -- a stable sort of the flattened
  top-k ids by expert; ``expert_offsets`` is the exclusive scan of the counts;
* each expert's group is also given a 128-row aligned place in the padded
  activation buffers the GEMM reads (``pad_offsets``);
* the combine accumulates out[t] = sum_j w[t, j] * y[slot(t, j)] in float32 in
  j order, one product and one sum rounding per term (no fused multiply-add),
  then rounds to bf16 (nearest even).
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_round, f32

PAD_ROWS = 128


class RoutingError(ValueError):
    pass


def permute(topk_ids, E: int):
    """Group routed (token, j) pairs by expert.

    Returns dict(expert_offsets [E+1], pad_offsets [E+1], slot_token [S],
    token_slot [T, k]) as int64 arrays.
    """
    ids = np.asarray(topk_ids).astype(np.int64)
    T, k = ids.shape
    if ((ids < 0) | (ids >= E)).any():
        raise RoutingError("expert id out of range")
    flat = ids.reshape(-1)
    order = np.argsort(flat, kind="stable")              # slot -> flat index
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    padded = -(-counts // PAD_ROWS) * PAD_ROWS
    pad_offsets = np.concatenate([[0], np.cumsum(padded)])
    slot_token = order // k
    token_slot = np.empty(T * k, dtype=np.int64)
    token_slot[order] = np.arange(T * k)
    return dict(expert_offsets=offsets, pad_offsets=pad_offsets,
                slot_token=slot_token, token_slot=token_slot.reshape(T, k))


def slot_expert(expert_offsets) -> np.ndarray:
    off = np.asarray(expert_offsets, dtype=np.int64)
    return np.repeat(np.arange(off.size - 1), np.diff(off))


def padded_row_of_slot(expert_offsets, pad_offsets) -> np.ndarray:
    off = np.asarray(expert_offsets, dtype=np.int64)
    pad = np.asarray(pad_offsets, dtype=np.int64)
    e = slot_expert(off)
    s = np.arange(off[-1])
    return pad[e] + (s - off[e])


def unpermute(y, token_slot, topk_w) -> np.ndarray:
    """Weighted combine, float32 in j order, then bf16.  Returns float32 values on the bf16 grid."""
    y = f32(y)
    ts = np.asarray(token_slot, dtype=np.int64)
    w = f32(topk_w)
    T, k = ts.shape
    acc = np.zeros((T, y.shape[1]), dtype=np.float32)
    for j in range(k):
        prod = f32(w[:, j:j + 1] * y[ts[:, j]])
        acc = f32(acc + prod)
    return bf16_round(acc)
