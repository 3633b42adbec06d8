"""GPU parity: permutation, activation quantisation and the weighted combine are
bit-exact against the oracle (grouped GEMM over routed tokens, kernel line of the
Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card; "dynamic per-32 group scales" of
its "Compression details" table)."""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
import workloads as W
from oracle import formats as F
from oracle import gemm as G
from oracle import routing as R
from tests.parity_util import cuda, kernel_rows_to_slots

pytestmark = pytest.mark.gpu


def gpu_permute(ids, E):
    T, k = ids.shape
    d_ids = cuda(ids.astype(np.int32))
    eo = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    po = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    st = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    ts = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    n = M.permute_workspace_size(T, k, E)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moesq_permute(d_ids, T, k, E, eo, po, st, ts, ws, n, status)
    return eo, po, st, ts, status


@pytest.mark.parametrize("cfg_name,T", [("tiny", 64), ("qwen3_30b_a3b", 1), ("qwen3_30b_a3b", 4096),
                                        ("qwen3_5_397b_a17b", 256), ("kimi_k2", 16384),
                                        ("qwen3_235b_a22b", 65536)])
def test_permute_bit_exact(cfg_name, T):
    cfg = W.CONFIGS[cfg_name]
    ids, _ = W.routing(cfg, T)
    ids = ids.numpy()
    ref = R.permute(ids, cfg.E)
    eo, po, st, ts, status = gpu_permute(ids, cfg.E)
    assert np.array_equal(eo.cpu().numpy(), ref["expert_offsets"])
    assert np.array_equal(po.cpu().numpy(), ref["pad_offsets"])
    assert np.array_equal(st.cpu().numpy()[:T * cfg.k], ref["slot_token"])
    assert np.array_equal(ts.cpu().numpy()[:T * cfg.k].reshape(T, cfg.k), ref["token_slot"])
    assert int(status.item()) == 0


@pytest.mark.parametrize("T,k,E,dist", [
    (128, 8, 128, "uniform"),    # one block at its largest batch (1024 slots)
    (128, 8, 512, "uniform"),    # one block, largest table (above the 48 KB default shared memory)
    (129, 8, 512, "uniform"),    # just past one chunk: three passes, largest table
    (200, 4, 1024, "uniform"),   # one block, more experts than the table holds: warps take turns
    (600, 4, 1024, "uniform"),   # three passes, warps take turns
    (512, 8, 128, "uniform"),    # three passes, table
    (1024, 8, 384, "uniform"),   # three passes, table above 48 KB
    (3000, 8, 16, "skew"),       # most slots on one expert: long runs inside every warp
    (100, 8, 16, "skew"),        # the same in one block
    (1, 1, 1, "uniform"),
    (5000, 2, 2, "uniform"),
])
def test_permute_bit_exact_sizes(T, k, E, dist):
    """Stable expert-major order against the oracle's counting sort at the sizes where
    the kernel changes form (one block or three passes; table or turns)."""
    rng = np.random.default_rng(T * 1000 + k * 10 + E)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    if dist == "skew":
        ids[rng.random((T, k)) < 0.9] = 3
    ref = R.permute(ids, E)
    eo, po, st, ts, status = gpu_permute(ids, E)
    assert np.array_equal(eo.cpu().numpy(), ref["expert_offsets"])
    assert np.array_equal(po.cpu().numpy(), ref["pad_offsets"])
    assert np.array_equal(st.cpu().numpy()[:T * k], ref["slot_token"])
    assert np.array_equal(ts.cpu().numpy()[:T * k].reshape(T, k), ref["token_slot"])
    assert int(status.item()) == 0


def test_permute_flags_bad_expert():
    ids = np.array([[0, 1], [2, 9]], np.int32)
    *_, status = gpu_permute(ids, 4)
    assert int(status.item()) & 2


@pytest.mark.parametrize("cfg_name,T,layout", [("tiny", 64, 0), ("tiny", 64, 1), ("qwen3_30b_a3b", 64, 1),
                                               ("qwen3_30b_a3b", 512, 0), ("kimi_k2", 32, 1)])
def test_quant_act_bit_exact(cfg_name, T, layout):
    cfg = W.CONFIGS[cfg_name]
    x = W.layer_input_bf16(cfg, T)
    ids, _ = W.routing(cfg, T)
    ref = R.permute(ids.numpy(), cfg.E)
    rng = np.random.default_rng(T)
    g_in = (np.float32(W.activation_global_scale_input(x)) *
            rng.uniform(0.5, 2.0, cfg.E)).astype(np.float32)            # per-expert path
    want_c, want_s = G.quant_act(x.float().numpy(), ref["slot_token"], ref["expert_offsets"], g_in)
    want_packed = (want_c[:, 0::2] | (want_c[:, 1::2] << 4)).astype(np.uint8)
    eo, po, st, ts, _ = gpu_permute(ids.numpy(), cfg.E)
    Sn = T * cfg.k
    K = cfg.H
    if layout == 0:
        codes = torch.empty((Sn, K // 2), dtype=torch.uint8, device="cuda")
        sf = torch.empty((Sn, K // 32), dtype=torch.uint8, device="cuda")
    else:
        P = M.padded_rows(Sn, cfg.E)
        codes = torch.empty((P, K // 2), dtype=torch.uint8, device="cuda")
        sf = torch.empty((P // 128) * (K // 128) * 512, dtype=torch.uint8, device="cuda")
    M.moesq_quant_act(x.cuda().view(torch.uint16), K, st, eo, po, cfg.E, cuda(g_in), Sn, layout, codes, sf)
    if layout == 0:
        got_c, got_s = codes.cpu().numpy(), sf.cpu().numpy()
    else:
        got_c, got_s = kernel_rows_to_slots(codes.cpu().numpy(), sf.cpu().numpy(), ref["expert_offsets"],
                                            ref["pad_offsets"], K)
    assert np.array_equal(got_s, want_s)
    assert np.array_equal(got_c, want_packed)


def test_quant_act_golden_groups(golden):
    """The hand-worked NVFP4 groups, through the GPU kernel (bf16-exact inputs only)."""
    for grp in golden("nvfp4_groups.json")["groups"]:
        x = np.array(grp["x"], np.float32)
        if not np.array_equal(F.bf16_round(x), x):
            continue
        xx = np.zeros((1, 128), np.float32)
        xx[0, :32] = x
        codes = torch.empty((1, 64), dtype=torch.uint8, device="cuda")
        sf = torch.empty((1, 4), dtype=torch.uint8, device="cuda")
        M.moesq_quant_act(cuda(xx, torch.bfloat16).view(torch.uint16), 128, None, None, None, 1,
                          cuda(np.float32([grp["g"]])), 1, 0, codes, sf)
        c = codes.cpu().numpy()[0, :16]
        got = np.stack([c & 0xF, c >> 4], axis=1).reshape(-1)
        assert int(sf.cpu().numpy()[0, 0]) == grp["scale"], grp["name"]
        assert got.tolist() == grp["codes"], grp["name"]


@pytest.mark.parametrize("T,k,H", [(1, 1, 8), (64, 2, 256), (1000, 8, 2048), (7, 10, 4096)])
def test_unpermute_bit_exact(T, k, H):
    rng = np.random.default_rng(T + k)
    Sn = T * k
    y = F.bf16_round((rng.standard_normal((Sn, H)) * 3).astype(np.float32))
    ts = rng.permutation(Sn).reshape(T, k).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    w /= w.sum(1, keepdims=True)
    want = R.unpermute(y, ts, w)
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    M.moesq_unpermute(cuda(y, torch.bfloat16).view(torch.uint16), cuda(ts), cuda(w), T, k, H,
                      out.view(torch.uint16))
    assert np.array_equal(out.float().cpu().numpy(), want)


def test_combine_golden_on_gpu(golden):
    g = golden("combine.json")
    y = np.zeros((5, 8), np.float32)
    y[:, :2] = np.array(g["y"], np.float32)
    out = torch.empty((2, 8), dtype=torch.bfloat16, device="cuda")
    M.moesq_unpermute(cuda(y, torch.bfloat16).view(torch.uint16), cuda(np.array(g["token_slot"], np.int32)),
                      cuda(np.array(g["topk_w"], np.float32)), 2, 3, 8, out.view(torch.uint16))
    assert out.float().cpu().numpy()[:, :2].tolist() == g["out"]


ROUTED_CASES = [("tiny", 64, False), ("qwen3_30b_a3b", 512, False), ("qwen3_5_397b_a17b", 16, False),
                ("kimi_k2", 32, False)]
# batches whose codes reach 64 MiB: the scales are written as rows and rearranged into the
# tensor-core blocks by a second kernel (Zipf routing: empty experts, ragged padding)
ROUTED_ROWS_CASES = [("qwen3_30b_a3b", 8192, True), ("qwen3_5_397b_a17b", 4096, True)]


@pytest.mark.parametrize("cfg_name,T,rows", ROUTED_CASES + ROUTED_ROWS_CASES)
@pytest.mark.parametrize("shared_global", [False, True])
def test_quant_act_routed_bit_exact(cfg_name, T, rows, shared_global):
    """Token-major quantisation (x read once per token) equals the per-slot oracle rule,
    with a global per expert and with one global shared by all experts (the kernel then
    reuses a group's codes across the token's slots)."""
    assert (T * W.CONFIGS[cfg_name].k * W.CONFIGS[cfg_name].H // 2 >= 64 << 20) == rows
    cfg = W.CONFIGS[cfg_name]
    x = W.layer_input_bf16(cfg, T)
    ids, _ = W.routing(cfg, T)
    ref = R.permute(ids.numpy(), cfg.E)
    rng = np.random.default_rng(T + 1)
    g_in = (np.float32(W.activation_global_scale_input(x)) * rng.uniform(0.5, 2.0, cfg.E)).astype(np.float32)
    if shared_global:
        g_in[:] = g_in[0]
    want_c, want_s = G.quant_act(x.float().numpy(), ref["slot_token"], ref["expert_offsets"], g_in)
    want_packed = (want_c[:, 0::2] | (want_c[:, 1::2] << 4)).astype(np.uint8)
    eo, po, st, ts, _ = gpu_permute(ids.numpy(), cfg.E)
    Sn, K = T * cfg.k, cfg.H
    P = M.padded_rows(Sn, cfg.E)
    codes = torch.empty((P, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((P // 128) * (K // 128) * 512, dtype=torch.uint8, device="cuda")
    M.moesq_quant_act_routed(x.cuda().view(torch.uint16), T, K, ids.cuda(), ts, cfg.k, eo, po, cfg.E,
                             cuda(g_in), codes, sf)
    got_c, got_s = kernel_rows_to_slots(codes.cpu().numpy(), sf.cpu().numpy(), ref["expert_offsets"],
                                        ref["pad_offsets"], K)
    assert np.array_equal(got_s, want_s)
    assert np.array_equal(got_c, want_packed)
