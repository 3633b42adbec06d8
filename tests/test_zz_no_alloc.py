"""moesq_permute_noalloc: the routing permutation for callers that cannot allocate.

Some callers may not allocate device memory while they route a batch: a serving
engine that reserves all device memory up front, or a plugin that is handed only
its bound input and output buffers.  For them the library offers a variant of
moesq_permute whose scratch is a fixed array in device memory instead of a
caller-provided workspace.  These checks call both entry points through the C
ABI and require identical integer outputs, on two calls in a row with different
sizes (so stale scratch from the first call must not leak into the second).
The allocation-free entry point has its own chain of kernels (per-chunk counts, a
scan, a scatter), so its outputs are also compared with the oracle's permutation
(oracle/routing.py) directly: small batches (where moesq_permute takes its one-block
path), zero tokens, slot counts that are not a multiple of the 1024-slot chunk, more
than 512 experts, calls of different expert counts back to back, and an invalid
expert id, which must raise MOESQ_DFLAG_BAD_EXPERT and be routed to expert 0 as the
header states.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
import workloads as W
from oracle import routing as R
from sparse_nvfp4_moe_b200 import _lib

pytestmark = pytest.mark.gpu


def _outputs(T, k, E):
    i32 = dict(dtype=torch.int32, device="cuda")
    return (torch.full((E + 1,), -1, **i32), torch.full((E + 1,), -1, **i32),
            torch.full((max(T * k, 1),), -1, **i32), torch.full((max(T * k, 1),), -1, **i32))


def _with_workspace(ids, T, k, E):
    eo, po, st, ts = _outputs(T, k, E)
    n = M.permute_workspace_size(T, k, E)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moesq_permute(ids, T, k, E, eo, po, st, ts, ws, n, status)
    return eo, po, st, ts, status


def _without_workspace(ids, T, k, E):
    eo, po, st, ts = _outputs(T, k, E)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moesq_permute_noalloc(ids, T, k, E, eo, po, st, ts, status)
    return eo, po, st, ts, status


def test_noalloc_permute_matches_workspace_permute_on_consecutive_calls():
    cases = [("qwen3_30b_a3b", 4096), ("qwen3_5_397b_a17b", 256), ("kimi_k2", 1024)]
    for name, T in cases:
        cfg = W.CONFIGS[name]
        ids, _ = W.routing(cfg, T, device="cuda")
        ref = _with_workspace(ids, T, cfg.k, cfg.E)
        got = _without_workspace(ids, T, cfg.k, cfg.E)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b), name
        assert int(got[-1].item()) == 0


def test_noalloc_permute_rejects_requests_beyond_its_scratch():
    E, k = 4096, 1
    T = 1024 * (_lib.PERMUTE_NOALLOC_MAX_COUNTS // E + 1)     # one chunk too many
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(M.MoesqError) as err:
        M.moesq_permute_noalloc(dummy, T, k, E, dummy, dummy, dummy, dummy)
    assert err.value.status == 8
    assert "scratch" in M.status_string(8)


def _check_against_oracle(ids_np, E, got, bad=False):
    """got = (expert_offsets, pad_offsets, slot_token, token_slot, status) of one call."""
    T, k = ids_np.shape
    ref = R.permute(np.where((ids_np < 0) | (ids_np >= E), 0, ids_np), E)
    eo, po, st, ts, status = (t.cpu().numpy() for t in got)
    assert np.array_equal(eo, ref["expert_offsets"])
    assert np.array_equal(po, ref["pad_offsets"])
    assert np.array_equal(st[:T * k], ref["slot_token"])
    assert np.array_equal(ts[:T * k].reshape(T, k), ref["token_slot"])
    assert int(status[0]) == (2 if bad else 0)


NOALLOC_CASES = [
    # (E, k, T, seed): one-block sizes, a ragged last chunk, E > 512, the largest E x chunks
    (8, 2, 5, 1), (16, 4, 256, 2), (128, 8, 127, 3), (512, 10, 1000, 4), (1024, 8, 2049, 5),
    (4096, 1, 3000, 6), (1024, 4, 65535, 7), (64, 8, 32768 - 3, 8),
]


@pytest.mark.parametrize("E,k,T,seed", NOALLOC_CASES)
def test_noalloc_permute_matches_oracle(E, k, T, seed):
    assert -(-T * k // 1024) * E <= _lib.PERMUTE_NOALLOC_MAX_COUNTS
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    got = _without_workspace(torch.from_numpy(ids).cuda(), T, k, E)
    _check_against_oracle(ids, E, got)


def test_noalloc_permute_back_to_back_different_expert_counts():
    """Two calls in a row with different E and sizes on one stream, then the first again:
    no call may read the previous call's scratch."""
    rng = np.random.default_rng(11)
    shapes = [(2048, 2, 1536), (32, 8, 700), (2048, 2, 1536)]
    runs = []
    for E, k, T in shapes:
        ids = rng.integers(0, E, (T, k)).astype(np.int32)
        runs.append((ids, E, _without_workspace(torch.from_numpy(ids).cuda(), T, k, E)))
    for ids, E, got in runs:
        _check_against_oracle(ids, E, got)


def test_noalloc_permute_zero_tokens():
    E = 16
    eo, po, st, ts, status = _without_workspace(torch.zeros(16, dtype=torch.int32, device="cuda"), 0, 4, E)
    assert np.array_equal(eo.cpu().numpy(), np.zeros(E + 1, np.int32))
    assert np.array_equal(po.cpu().numpy(), np.zeros(E + 1, np.int32))
    assert int(status.item()) == 0


@pytest.mark.parametrize("T,k,E", [(3, 2, 4), (700, 4, 64)])
def test_noalloc_permute_flags_bad_expert(T, k, E):
    rng = np.random.default_rng(13)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    ids[T // 2, k - 1] = E + 5
    ids[0, 0] = -1
    got = _without_workspace(torch.from_numpy(ids).cuda(), T, k, E)
    _check_against_oracle(ids, E, got, bad=True)
