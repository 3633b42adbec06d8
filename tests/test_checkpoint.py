"""The paired48 sparse-storage checkpoint reader ("Sparse storage layout
(paired48_sparse, pair-bitmask v1)" of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model
card) against files written by the safetensors library itself: a synthetic
two-shard checkpoint of one MoE layer whose expert tensors come from the oracle's
weight quantiser."""
import json
import os

import numpy as np
import pytest
import torch
from safetensors.torch import save_file

import workloads as W
from oracle import storage as S
from sparse_nvfp4_moe_b200 import checkpoint as C

PREFIX = "model.layers.3.mlp"
CFG = W.LayerConfig("ckpt", 61, 3, 2, 256, 128, (32,), "uniform", True)


def _experts():
    gu = W.all_expert_weights_bf16(CFG, "gate_up")
    dn = W.all_expert_weights_bf16(CFG, "down")
    st_gu = [S.quantize_weight(gu[e].float().numpy(), 2) for e in range(CFG.E)]
    st_dn = [S.quantize_weight(dn[e].float().numpy(), 1) for e in range(CFG.E)]
    g_in = np.float32([0.0125, 0.0125, 0.0125])          # same input for gate and up of an expert
    g_in_dn = np.float32([0.003, 0.0041, 0.0027])
    return st_gu, st_dn, g_in, g_in_dn


def _linear_tensors(name, packed, mask, scale, g, g_in, reciprocal):
    gv = np.float32(1) / np.float32(g) if reciprocal else np.float32(g)
    gi = np.float32(1) / np.float32(g_in) if reciprocal else np.float32(g_in)
    return {f"{name}.weight_sparse_packed": torch.from_numpy(np.ascontiguousarray(packed)),
            f"{name}.weight_sparse_mask": torch.from_numpy(np.ascontiguousarray(mask)),
            f"{name}.weight_scale": torch.from_numpy(np.ascontiguousarray(scale)).view(torch.float8_e4m3fn),
            f"{name}.weight_global_scale": torch.tensor(gv),
            f"{name}.input_global_scale": torch.tensor([gi])}


def write_checkpoint(d, reciprocal=True, marker=None, fmt="nvfp4-pack-quantized"):
    """One MoE layer in paired48 storage.  By default the globals are stored the way the
    compressed-tensors NVFP4 format stores them, as reciprocals (6 * 448 / amax)."""
    st_gu, st_dn, g_in, g_in_dn = _experts()
    I = CFG.I
    shards = [{}, {}]
    for e in range(CFG.E):
        sg, sd = st_gu[e], st_dn[e]
        base = f"{PREFIX}.experts.{e}"
        t = {}
        t.update(_linear_tensors(f"{base}.gate_proj", sg["packed"][:I], sg["mask"][:I], sg["scale"][:I],
                                 sg["g"][0], g_in[e], reciprocal))
        t.update(_linear_tensors(f"{base}.up_proj", sg["packed"][I:], sg["mask"][I:], sg["scale"][I:],
                                 sg["g"][1], g_in[e], reciprocal))
        t.update(_linear_tensors(f"{base}.down_proj", sd["packed"], sd["mask"], sd["scale"], sd["g"][0],
                                 g_in_dn[e], reciprocal))
        shards[e % 2].update(t)
    shards[0]["model.embed_tokens.weight"] = torch.zeros(4, 8, dtype=torch.bfloat16)   # unrelated tensor
    wm = {}
    for i, sh in enumerate(shards):
        fn = f"model-{i + 1:05d}-of-00002.safetensors"
        save_file(sh, os.path.join(d, fn), metadata={"format": "pt"})
        wm.update({n: fn for n in sh})
    json.dump({"metadata": {}, "weight_map": wm}, open(os.path.join(d, "model.safetensors.index.json"), "w"))
    qc = {"format": fmt,
          "paired48_sparse": marker if marker is not None else {"layout": "pair-bitmask", "version": 1}}
    json.dump({"quantization_config": qc}, open(os.path.join(d, "config.json"), "w"))
    return st_gu, st_dn, g_in, g_in_dn


def test_read_back_bit_exact(tmp_path):
    """Globals stored as multipliers (the library's own convention) read back bit for bit."""
    st_gu, st_dn, g_in, g_in_dn = write_checkpoint(str(tmp_path), reciprocal=False, fmt="")
    r = C.read_moe_experts(C.Checkpoint(str(tmp_path)), PREFIX, CFG.E)
    gu, dn = r["gate_up"], r["down"]
    assert (gu["E"], gu["out"], gu["K"]) == (CFG.E, 2 * CFG.I, CFG.H)
    assert (dn["E"], dn["out"], dn["K"]) == (CFG.E, CFG.H, CFG.I)
    for e in range(CFG.E):
        for key in ("packed", "mask", "scale"):
            assert np.array_equal(gu[key][e].numpy(), st_gu[e][key])
            assert np.array_equal(dn[key][e].numpy(), st_dn[e][key])
        assert np.array_equal(gu["g_w"][e].numpy(), np.asarray(st_gu[e]["g"], np.float32))
        assert dn["g_w"][e, 0].item() == np.float32(st_dn[e]["g"][0])
    assert np.array_equal(r["g_in_gate_up"].numpy(), g_in)
    assert np.array_equal(r["g_in_down"].numpy(), g_in_dn)


def test_reciprocal_convention(tmp_path):
    st_gu, _, g_in, _ = write_checkpoint(str(tmp_path), reciprocal=True)
    for conv in ("auto", "reciprocal"):
        r = C.read_moe_experts(C.Checkpoint(str(tmp_path)), PREFIX, CFG.E, global_convention=conv)
        for e in range(CFG.E):
            stored = np.float32(1) / np.float32(st_gu[e]["g"][0])
            assert r["gate_up"]["g_w"][e, 0].item() == np.float32(np.float32(1) / stored)
        assert r["g_in_gate_up"][0].item() == np.float32(np.float32(1) / (np.float32(1) / g_in[0]))


def test_compressed_tensors_globals_decode_to_the_weights(tmp_path):
    """A tensor written as compressed-tensors writes it (global = 6 * 448 / amax, the
    reciprocal) decodes, under the default reading, to the same weights as the
    multiplier-form storage it came from: E2M1 x E4M3 x multiplier, elementwise."""
    from oracle import formats as F
    from oracle import nvfp4 as N
    st_gu, st_dn, _, _ = write_checkpoint(str(tmp_path), reciprocal=True)
    r = C.read_moe_experts(C.Checkpoint(str(tmp_path)), PREFIX, CFG.E)
    for e in range(CFG.E):
        st = st_dn[e]
        want = F.e2m1_decode(N.unpack_codes(S.decode(st["packed"], st["mask"])))
        want = want * np.repeat(F.e4m3_decode(st["scale"]), 32, axis=1) * np.float64(np.float32(st["g"][0]))
        d = r["down"]
        got = F.e2m1_decode(N.unpack_codes(S.decode(d["packed"][e].numpy(), d["mask"][e].numpy())))
        got = got * np.repeat(F.e4m3_decode(d["scale"][e].numpy()), 32, axis=1) * np.float64(d["g_w"][e, 0].item())
        assert np.allclose(got, want, rtol=2 ** -22, atol=0)
        assert np.abs(want).max() < 1.0                    # weights of N(0, 0.02), not amax**2 / 2688**2 off


def test_a_contradicted_convention_is_refused(tmp_path):
    """Reading reciprocal globals as multipliers (or the reverse) would scale every weight
    by about (2688 / amax)**2: the reader refuses instead of guessing."""
    write_checkpoint(str(tmp_path), reciprocal=True)
    with pytest.raises(C.CheckpointError):
        C.read_moe_experts(C.Checkpoint(str(tmp_path)), PREFIX, CFG.E, global_convention="multiplier")
    d2 = tmp_path / "mult"
    d2.mkdir()
    write_checkpoint(str(d2), reciprocal=False, fmt="")
    with pytest.raises(C.CheckpointError):
        C.read_moe_experts(C.Checkpoint(str(d2)), PREFIX, CFG.E, global_convention="reciprocal")
    r = C.read_moe_experts(C.Checkpoint(str(d2)), PREFIX, CFG.E)          # auto: multipliers
    assert r["down"]["g_w"][0, 0].item() < 1e-3


@pytest.mark.parametrize("marker", [{}, {"layout": "pair-bitmask", "version": 2}, {"layout": "dense", "version": 1}])
def test_marker_is_checked(tmp_path, marker):
    write_checkpoint(str(tmp_path), marker=marker)
    with pytest.raises(C.CheckpointError):
        C.read_moe_experts(C.Checkpoint(str(tmp_path)), PREFIX, CFG.E)


def test_missing_tensor_and_bad_shapes(tmp_path):
    write_checkpoint(str(tmp_path))
    ck = C.Checkpoint(str(tmp_path))
    with pytest.raises(C.CheckpointError):
        C.read_moe_experts(ck, PREFIX, CFG.E + 1)                      # no expert E
    d2 = tmp_path / "bad"
    d2.mkdir()
    name = f"{PREFIX}.experts.0.gate_proj"
    t = _linear_tensors(name, np.zeros((128, 64), np.uint8), np.zeros((128, 8), np.uint8),   # mask K/16 wrong
                        np.zeros((128, 8), np.uint8), 1.0, 1.0, False)
    save_file(t, str(d2 / "model.safetensors"))
    with pytest.raises(C.CheckpointError):
        C.read_linear(C.Checkpoint(str(d2)), name)


def test_container_parser_matches_library(tmp_path):
    """Every dtype the reader maps, against safetensors' own loader."""
    from safetensors.torch import load_file
    t = {"a": torch.arange(12, dtype=torch.int32).reshape(3, 4), "b": torch.randn(5).to(torch.bfloat16),
         "c": torch.randn(2, 3), "d": torch.arange(7, dtype=torch.uint8), "e": torch.tensor(3.5),
         "f": torch.randn(4).to(torch.float8_e4m3fn), "g": torch.arange(3, dtype=torch.int64)}
    p = str(tmp_path / "x.safetensors")
    save_file(t, p, metadata={"k": "v"})
    f = C.SafetensorsFile(p)
    ref = load_file(p)
    assert f.metadata == {"k": "v"}
    for n, v in ref.items():
        got = f.get(n)
        want = v.view(torch.uint8) if v.dtype == torch.float8_e4m3fn else (
            v.view(torch.uint16) if v.dtype == torch.bfloat16 else v)
        assert got.shape == tuple(v.shape)
        assert np.array_equal(got, want.numpy())


@pytest.mark.gpu
def test_loaded_layer_equals_layer_from_storage(tmp_path):
    """A layer loaded from the checkpoint runs bit-identically to one built from the
    same storages directly (the reader adds nothing and loses nothing)."""
    import sparse_nvfp4_moe_b200 as M
    from tests import parity_util as PU
    st_gu, st_dn, g_in, g_in_dn = write_checkpoint(str(tmp_path), reciprocal=False, fmt="")
    T = 96
    x = W.layer_input_bf16(CFG, T).cuda()
    ids, w = W.routing(CFG, T)
    ids, w = ids.to(torch.int32).cuda(), w.cuda()
    for exact in (False, True):
        a = C.load_moe_layer(str(tmp_path), PREFIX, CFG.E, CFG.k, exact=exact)
        kind = M.KIND_GATE_UP_EXACT if exact else M.KIND_GATE_UP_SPLIT
        gu = M.ExpertLinear.from_storage(PU.storage_to_device(st_gu), kind)
        dn = M.ExpertLinear.from_storage(PU.storage_to_device(st_dn), M.KIND_DOWN)
        b = M.MoELayer(CFG.k, gu, dn, PU.cuda(g_in), PU.cuda(g_in_dn))
        assert torch.equal(a.forward(x, ids, w), b.forward(x, ids, w))
