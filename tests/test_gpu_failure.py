"""Failure detection on the GPU without a fault: every pipeline wait of the library
is bounded, and one that runs out reports it through the status word and returns.

The self-test kernel waits, with each of the library's three bounded waits, on an
mbarrier phase that nothing completes (no trap, no bad address, no endless loop).
After the limit each wait gives up and flags MOESQ_DFLAG_TIMEOUT; the context stays
usable, which the test shows by running a library call afterwards and checking it.
"""
import time

import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
from oracle import routing as R

pytestmark = pytest.mark.gpu

DFLAG_TIMEOUT = 0x4


def test_bounded_waits_give_up_and_flag_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gave_up = torch.zeros(3, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    M.moesq_selftest_wait_timeout(status, 2_000_000, gave_up)      # 2 ms per wait
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert gave_up.tolist() == [1, 1, 1]
    assert int(status.item()) & DFLAG_TIMEOUT
    assert dt < 5.0                                                   # bounded, not hung

    # the context is intact: a permutation right after is still bit-exact
    rng = np.random.default_rng(0)
    T, k, E = 300, 4, 16
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    ref = R.permute(ids, E)
    eo = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    po = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    st = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ts = torch.empty(T * k, dtype=torch.int32, device="cuda")
    n = M.permute_workspace_size(T, k, E)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    s2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moesq_permute(torch.from_numpy(ids).cuda(), T, k, E, eo, po, st, ts, ws, n, s2)
    assert int(s2.item()) == 0
    assert np.array_equal(eo.cpu().numpy(), ref["expert_offsets"])
    assert np.array_equal(st.cpu().numpy(), ref["slot_token"])
