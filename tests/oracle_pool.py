"""Oracle weight export in a pool of spawned CPU processes (test infrastructure).

The full-size parity tests need the pair-bitmask storage of dozens of expert linears
as the oracle computes it from the seeded bf16 weights; that export takes seconds per
expert in numpy, so the tests spread it over the host's cores.  Workers import only
numpy and the oracle (no CUDA), and the pool is started with `spawn`, never `fork`, so
it is safe after the parent has used the GPU.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

KEEP = ("packed", "mask", "scale", "g")


def _export(task):
    """(key, bf16 bits of gate_up [2I, H], bf16 bits of down [H, I], n_seg) -> storages."""
    from oracle import storage as S
    key, gu_bits, dn_bits, n_seg = task
    gu = S.quantize_weight((gu_bits.astype(np.uint32) << 16).view(np.float32), n_seg)
    dn = S.quantize_weight((dn_bits.astype(np.uint32) << 16).view(np.float32), 1)
    return key, {k: gu[k] for k in KEEP}, {k: dn[k] for k in KEEP}


def export_experts(tasks, workers=None):
    """Run the oracle's export for every (key, gu_bits, dn_bits, n_seg) task; returns
    {key: (gate_up storage, down storage)}."""
    if not tasks:
        return {}
    n = min(len(tasks), workers or max(1, min(16, (os.cpu_count() or 2) - 1)))
    if n == 1:
        return {k: (g, d) for k, g, d in map(_export, tasks)}
    with mp.get_context("spawn").Pool(n) as pool:
        return {k: (g, d) for k, g, d in pool.imap_unordered(_export, tasks)}
