"""GPU parity of the whole expert path on degenerate routings.

The generated routings of the other cases spread slots over many experts.  These
cases pin the schedule's corners instead:

- every token routed to one expert, the other experts empty (including the first
  and the last);
- every token routed to the same two experts, in either order within a token;
- one token;
- expert groups sized around the tile edges (1, 16/17, 31-33, 64/65, 127-129,
  255-257 rows), empty groups between them, and a token order that does not
  follow the groups;
- zero tokens.

Each layer runs through the library's forward (permute, activation quantisation,
gate_up with fused SwiGLU + NVFP4 requant, down, combine) and is held to the same
bound as the generated cases: 1e-5 * sum|a w| per GEMM output, the requantisation
flips that bound allows, and one bf16 ulp per rounding.
"""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
import workloads as W
from oracle import routing as R
from tests.parity_util import cuda
from tests.test_gpu_gemm import Layer
from tests.test_gpu_gemm import test_moe_forward_end_to_end as forward_check

pytestmark = pytest.mark.gpu


def _weights(T, k, seed):
    w = np.random.default_rng(seed).random((T, k)).astype(np.float32) + np.float32(0.05)
    return w / w.sum(axis=1, keepdims=True)


def one_expert(T, E, e, seed):
    return np.full((T, 1), e, np.int64), _weights(T, 1, seed)


def two_experts(T, e0, e1, seed):
    ids = np.empty((T, 2), np.int64)
    ids[0::2] = (e0, e1)
    ids[1::2] = (e1, e0)
    return ids, _weights(T, 2, seed)


def sized_groups(sizes, seed):
    """k = 1 routing in which expert e receives exactly sizes[e] tokens, tokens shuffled."""
    ids = np.repeat(np.arange(len(sizes), dtype=np.int64), sizes)
    np.random.default_rng(seed).shuffle(ids)
    return ids.reshape(-1, 1), _weights(ids.size, 1, seed + 1)


GROUPS = (0, 1, 16, 17, 31, 32, 33, 0, 64, 65, 127, 128, 129, 255, 256, 257, 0)

CASES = {
    # H = 512: one full 512-deep gate_up stage; I = 384: a ragged 384-deep down stage
    "one_expert_takes_all": (W.LayerConfig("one", 51, 8, 1, 512, 384, (300,), "uniform", True), 300,
                             one_expert(300, 8, 5, 1)),
    "first_expert_takes_all": (W.LayerConfig("first", 52, 6, 1, 256, 256, (129,), "uniform", False), 129,
                               one_expert(129, 6, 0, 2)),
    "two_experts_take_all": (W.LayerConfig("two", 53, 8, 2, 512, 256, (200,), "uniform", True), 200,
                             two_experts(200, 7, 2, 3)),
    "single_token": (W.LayerConfig("single", 54, 16, 4, 1024, 512, (1,), "uniform", True), 1,
                     (np.array([[15, 0, 7, 3]], np.int64), _weights(1, 4, 4))),
    "tile_edge_groups": (W.LayerConfig("edges", 55, len(GROUPS), 1, 512, 384, (sum(GROUPS),), "uniform", True),
                         sum(GROUPS), sized_groups(GROUPS, 5)),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def edge_layer(request):
    cfg, T, routing = CASES[request.param]
    L = Layer(cfg, T, routing=routing)
    counts = np.diff(L.perm["expert_offsets"])
    if request.param == "tile_edge_groups":
        assert tuple(counts) == GROUPS
    return L


def test_edge_routing_forward_within_tolerance(edge_layer):
    forward_check(edge_layer)


def test_edge_routing_permutation_bit_exact(edge_layer):
    L = edge_layer
    eo, po, st, ts = L.device_routing()
    assert np.array_equal(eo.cpu().numpy(), L.perm["expert_offsets"])
    assert np.array_equal(po.cpu().numpy(), L.perm["pad_offsets"])
    assert np.array_equal(st.cpu().numpy(), L.perm["slot_token"])
    assert np.array_equal(ts.cpu().numpy().reshape(L.T, L.cfg.k), L.perm["token_slot"])
    # the padded row layout gives every nonempty group whole 128-row tiles
    pad = np.diff(L.perm["pad_offsets"])
    cnt = np.diff(L.perm["expert_offsets"])
    assert (pad % 128 == 0).all() and (pad >= cnt).all() and (pad - cnt < 128).all()
    assert np.array_equal(R.slot_expert(L.perm["expert_offsets"]), np.repeat(np.arange(L.cfg.E), cnt))


def test_zero_tokens_is_a_no_op():
    cfg, T, routing = CASES["two_experts_take_all"]
    L = Layer(cfg, T, routing=routing)
    moe = M.MoELayer(cfg.k, L.dgu, L.ddn, cuda(L.g_in_gu), cuda(L.g_in_dn))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.empty((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((0, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((0, cfg.k), dtype=torch.float32, device="cuda")
    out = moe.forward(x, ids, w, d_status=status)
    torch.cuda.synchronize()
    assert out.shape == (0, cfg.H)
    assert int(status.item()) == 0
