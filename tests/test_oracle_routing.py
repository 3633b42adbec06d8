"""Pins of the oracle's routing permutation and weighted combine (CPU only).

The grouped GEMM runs over the tokens the router sends to each expert (kernel
line of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card); the slot order and
the combine arithmetic are this library's readings (see include/moesq.h).
"""
import numpy as np
import pytest

from oracle import formats as F
from oracle import routing as R


def test_permute_brute_force_order():
    rng = np.random.default_rng(0)
    T, k, E = 37, 3, 7
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    p = R.permute(ids, E)
    # brute force: walk experts, then tokens, then j
    slots = [(t, j) for e in range(E) for t in range(T) for j in range(k) if ids[t, j] == e]
    assert [t for t, _ in slots] == p["slot_token"].tolist()
    for s, (t, j) in enumerate(slots):
        assert p["token_slot"][t, j] == s
    counts = [sum(1 for t in range(T) for j in range(k) if ids[t, j] == e) for e in range(E)]
    assert p["expert_offsets"].tolist() == [sum(counts[:e]) for e in range(E + 1)]
    pads = [-(-c // 128) * 128 for c in counts]
    assert p["pad_offsets"].tolist() == [sum(pads[:e]) for e in range(E + 1)]


def test_permute_invariants_and_errors():
    rng = np.random.default_rng(1)
    T, k, E = 500, 8, 64
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    p = R.permute(ids, E)
    off = p["expert_offsets"]
    assert (np.diff(off) >= 0).all() and off[-1] == T * k
    assert sorted(p["token_slot"].ravel().tolist()) == list(range(T * k))     # bijection
    e_of = R.slot_expert(off)
    assert (ids.ravel()[np.argsort(p["token_slot"].ravel())] == e_of).all()
    with pytest.raises(R.RoutingError):
        R.permute(np.array([[0, 64]]), E)
    with pytest.raises(R.RoutingError):
        R.permute(np.array([[-1, 0]]), E)


def test_padded_rows_are_128_aligned_per_expert():
    ids = np.array([[0, 2], [2, 0], [2, 1]])
    p = R.permute(ids, 4)
    rows = R.padded_row_of_slot(p["expert_offsets"], p["pad_offsets"])
    assert rows.tolist() == [0, 1, 128, 256, 257, 258]


def test_combine_golden(golden):
    g = golden("combine.json")
    out = R.unpermute(np.array(g["y"], np.float32), np.array(g["token_slot"]), np.array(g["topk_w"], np.float32))
    assert out.tolist() == g["out"]


def test_combine_single_expert_unit_weight_is_identity():
    rng = np.random.default_rng(2)
    y = F.bf16_round(rng.standard_normal((10, 16)).astype(np.float32))
    out = R.unpermute(y, np.arange(10)[:, None], np.ones((10, 1), np.float32))
    assert np.array_equal(out, y)
