"""moesq_permute_noalloc: the routing permutation for callers that cannot allocate.

Some callers may not allocate device memory while they route a batch: a serving
engine that reserves all device memory up front, or a plugin that is handed only
its bound input and output buffers.  For them the library offers a variant of
moesq_permute whose scratch is a fixed array in device memory instead of a
caller-provided workspace.  These checks call both entry points through the C
ABI and require identical integer outputs, on two calls in a row with different
sizes (so stale scratch from the first call must not leak into the second).
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
import workloads as W
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
