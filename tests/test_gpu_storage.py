"""GPU parity: storage codecs, weight export and load-time repack are bit-exact
against the oracle ("Sparse storage layout (paired48_sparse, pair-bitmask v1)",
Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card; gate/up fold of the Qwen3-30B-A3B
and Qwen3.8-Flash-Next cards)."""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
import workloads as W
from oracle import storage as S
from tests.parity_util import cuda

pytestmark = pytest.mark.gpu


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("rows,K", [(1, 64), (37, 128), (256, 2048), (130, 7168)])
def test_decode_encode_bit_exact(rows, K):
    rng = np.random.default_rng(rows * 7 + K)
    nib = rng.choice([3, 5, 6, 9, 10, 12], size=(rows, K // 8))
    mask = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    packed = rng.integers(0, 256, (rows, K // 4)).astype(np.uint8)
    packed[rng.random(packed.shape) < 0.1] = 0
    want = S.decode(packed, mask)
    st = _status()
    d_dense = torch.empty((rows, K // 2), dtype=torch.uint8, device="cuda")
    M.moesq_decode(cuda(packed), cuda(mask), d_dense, rows, K, st)
    assert np.array_equal(d_dense.cpu().numpy(), want)
    # encode with the mask as hint: exact inverse
    p2 = torch.empty((rows, K // 4), dtype=torch.uint8, device="cuda")
    m2 = torch.empty((rows, K // 16), dtype=torch.uint8, device="cuda")
    M.moesq_encode(d_dense, cuda(mask), p2, m2, rows, K, st)
    assert np.array_equal(p2.cpu().numpy(), packed) and np.array_equal(m2.cpu().numpy(), mask)
    # encode without a hint: the oracle's canonical fill rule
    wp, wm = S.encode(want)
    M.moesq_encode(d_dense, None, p2, m2, rows, K, st)
    assert np.array_equal(p2.cpu().numpy(), wp) and np.array_equal(m2.cpu().numpy(), wm)
    assert int(st.item()) == 0


def test_bad_sparsity_is_flagged_not_trapped():
    K = 64
    mask = np.full((2, K // 16), 0x33, np.uint8)
    mask[1, 2] = 0x37                                   # a nibble with 3 bits set
    packed = np.arange(2 * K // 4, dtype=np.uint8).reshape(2, K // 4)
    st = _status()
    out = torch.empty((2, K // 2), dtype=torch.uint8, device="cuda")
    M.moesq_decode(cuda(packed), cuda(mask), out, 2, K, st)
    assert int(st.item()) & 1
    dense = np.zeros((1, K // 2), np.uint8)
    dense[0, :3] = [1, 2, 3]                            # 3 nonzero bytes in one chunk
    st2 = _status()
    p = torch.empty((1, K // 4), dtype=torch.uint8, device="cuda")
    m = torch.empty((1, K // 16), dtype=torch.uint8, device="cuda")
    M.moesq_encode(cuda(dense), None, p, m, 1, K, st2)
    assert int(st2.item()) & 1


@pytest.mark.parametrize("cfg_name,which,n_seg,experts", [
    ("tiny", "gate_up", 1, [0, 1, 7]), ("tiny", "down", 1, [2, 3]),
    ("qwen3_30b_a3b", "gate_up", 2, [0, 77]), ("qwen3_30b_a3b", "down", 1, [5]),
    ("kimi_k2", "down", 1, [383]),
])
def test_quant_weight_bit_exact(cfg_name, which, n_seg, experts):
    cfg = W.CONFIGS[cfg_name]
    w = W.all_expert_weights_bf16(cfg, which, experts=experts)
    st = M.quantize_expert_weights(w.cuda(), n_seg)
    for i, e in enumerate(experts):
        ref = S.quantize_weight(w[i].float().numpy(), n_seg)
        assert np.array_equal(st["mask"][i].cpu().numpy(), ref["mask"]), e
        assert np.array_equal(st["scale"][i].cpu().numpy(), ref["scale"]), e
        assert np.array_equal(st["packed"][i].cpu().numpy(), ref["packed"]), e
        assert np.array_equal(st["g_w"][i].cpu().numpy(), ref["g"]), e


@pytest.mark.parametrize("kind,out,K", [(0, 128, 256), (0, 256, 384), (1, 256, 256), (2, 512, 384),
                                        (2, 1536, 2048), (3, 512, 384)])
def test_repack_bit_exact(kind, out, K):
    rng = np.random.default_rng(out + K + kind)
    E = 3
    sts = []
    for e in range(E):
        wv = (rng.standard_normal((out, K)) * 0.02).astype(np.float32)
        sts.append(S.quantize_weight(S.f32(torch.from_numpy(wv).to(torch.bfloat16).float().numpy()),
                                     2 if kind >= 2 else 1))
    # kind 3: both gate_up globals kept (alpha [E, 2]), up scales not folded
    ref = S.repack_linear(sts, "down" if kind == 0 else "gate_up", fold=kind != 3)
    dev = dict(mask=cuda(np.stack([s["mask"] for s in sts])), scale=cuda(np.stack([s["scale"] for s in sts])),
               g_w=cuda(np.stack([s["g"] for s in sts])))
    mb, sb = M.repack_sizes(out, K)
    meta = torch.empty(E * mb, dtype=torch.uint8, device="cuda")
    sf = torch.empty(E * sb, dtype=torch.uint8, device="cuda")
    alpha = torch.empty(2 * E if kind == 3 else E, dtype=torch.float32, device="cuda")
    st = _status()
    M.moesq_repack_meta(dev["mask"], dev["scale"], dev["g_w"], E, out, K, kind, meta, sf, alpha, st)
    assert np.array_equal(meta.cpu().numpy(), ref["meta"])
    assert np.array_equal(sf.cpu().numpy(), ref["sf"])
    assert np.array_equal(alpha.cpu().numpy(), ref["alpha"])
    assert int(st.item()) == 0


@pytest.mark.slow
def test_kimi_storage_round_trip_all_experts_sampled_rows():
    """Kimi-K2-shaped storage: all 384 down linears exported on the GPU, decoded and
    re-encoded bit-exactly; a sample of experts checked against the oracle."""
    cfg = W.CONFIGS["kimi_k2"]
    E = cfg.E
    chunk = 48
    rng = np.random.default_rng(5)
    sample = set(rng.choice(E, 3, replace=False).tolist())
    st_dev = _status()
    for e0 in range(0, E, chunk):
        ids = list(range(e0, min(E, e0 + chunk)))
        w = W.all_expert_weights_bf16(cfg, "down", device="cuda", experts=ids)
        st = M.quantize_expert_weights(w, 1)
        n, out, K = len(ids), cfg.H, cfg.I
        dense = torch.empty((n * out, K // 2), dtype=torch.uint8, device="cuda")
        M.moesq_decode(st["packed"], st["mask"], dense, n * out, K, st_dev)
        p2 = torch.empty_like(st["packed"])
        m2 = torch.empty_like(st["mask"])
        M.moesq_encode(dense, st["mask"], p2, m2, n * out, K, st_dev)
        assert torch.equal(p2, st["packed"]) and torch.equal(m2, st["mask"])
        for i, e in enumerate(ids):
            if e in sample:
                ref = S.quantize_weight(w[i].float().cpu().numpy(), 1)
                assert np.array_equal(st["packed"][i].cpu().numpy(), ref["packed"])
                assert np.array_equal(st["mask"][i].cpu().numpy(), ref["mask"])
                assert np.array_equal(dense[i * out:(i + 1) * out].cpu().numpy(), ref["dense"])
        del w, st, dense, p2, m2
    assert int(st_dev.item()) == 0
