"""Pins of the oracle's quantisation, pruning and pair-bitmask storage (CPU only).

Sources: "Compression details" and "Sparse storage layout (paired48_sparse,
pair-bitmask v1)" of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card; the
memory table of the Qwen3.8-Flash-Next-P48NVFP4-MoESQ card; "Usage" of the
MoESQ repository README; the gate/up global-scale fold of the
Qwen3-30B-A3B-P48NVFP4-MoESQ card.
"""
import itertools

import numpy as np
import pytest

import workloads as W
from oracle import formats as F
from oracle import nvfp4 as N
from oracle import storage as S


# -------------------------------------------------------------- NVFP4 rule --

def test_nvfp4_groups_golden(golden):
    for grp in golden("nvfp4_groups.json")["groups"]:
        x = np.array(grp["x"], dtype=np.float32)[None]
        codes, sc = N.quantize_groups(x, np.float32(grp["g"]))
        assert int(sc[0, 0]) == grp["scale"], grp["name"]
        assert codes[0].tolist() == grp["codes"], grp["name"]


def test_reciprocal_multiply_reading_differs_from_division(golden):
    """The rule multiplies by fp32(1/sdq) (reading R4 of the rounding rule); the golden
    group 'reciprocal_multiply_not_division' is worked by hand so that dividing by sdq
    instead gives other codes.  Recompute its key elements with exact rationals."""
    from fractions import Fraction
    grp = next(g for g in golden("nvfp4_groups.json")["groups"] if g["name"] == "reciprocal_multiply_not_division")
    assert grp["codes"] != grp["codes_if_division"]
    sdq = Fraction(15, 4)                                        # E4M3 0x47 = 2 * 1.875
    assert F.e4m3_decode(np.uint8(grp["scale"])) == float(sdq)
    inv = Fraction(float(np.float32(1) / np.float32(3.75)))
    assert inv == Fraction(8947849, 2 ** 25)                     # 1/3.75 rounded up to fp32
    for xv, c_mul, c_div in zip(grp["x"], grp["codes"], grp["codes_if_division"]):
        q = Fraction(xv) / sdq                                   # exact quotient
        p_ = float(np.float32(float(Fraction(xv) * inv)))        # fp32 product, one rounding
        assert int(F.e2m1_quantize(np.array([p_], np.float32))[0]) == c_mul
        assert int(F.e2m1_quantize(np.array([float(q)], np.float32))[0]) == c_div


def test_nvfp4_dequant_error_bound():
    """Unsaturated groups: every element lands within half an E2M1 step of x."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 3, (64, 1))).astype(np.float32)
    g = np.float32(np.abs(x).max() / 2688.0)
    codes, sc = N.quantize_groups(x, g)
    sdq = F.e4m3_decode(sc).astype(np.float64) * np.float64(g)
    deq = F.e2m1_decode(codes).reshape(64, 8, 32) * sdq[..., None]
    xg = x.reshape(64, 8, 32).astype(np.float64)
    # E2M1 spacing is at most 2 (between 4 and 6); half of it times the scale
    assert (np.abs(deq - xg) <= 1.0 * sdq[..., None] * (1 + 1e-6)).all()
    assert (F.e4m3_decode(sc) <= 448).all()
    # the group maximum maps close to the top code value 6
    top = np.abs(deq).max(axis=-1) / sdq
    assert ((top >= 4) | (np.abs(xg).max(axis=-1) == 0)).all()


def test_nvfp4_zero_global_gives_zero_codes():
    codes, sc = N.quantize_groups(np.ones((1, 32), np.float32), np.float32(0))
    assert (sc == 0).all() and (codes == 0).all()


def test_pack_nibble_order_low_is_lower_k():
    assert N.pack_codes(np.array([[1, 7, 8, 15]], np.uint8)).tolist() == [[0x71, 0xF8]]
    assert N.unpack_codes(np.array([[0x71, 0xF8]], np.uint8)).tolist() == [[1, 7, 8, 15]]


# ----------------------------------------------------------------- pruning --

def test_prune_brute_force_top2_pairs():
    rng = np.random.default_rng(11)
    w = F.bf16_round(rng.standard_normal((16, 64)).astype(np.float32) * 0.02)
    w[0, :8] = np.float32([1, 1, 1, 1, 0, 0, 0, 0])           # tie: lower pairs win
    keep = S.prune_paired48(w)
    for r in range(w.shape[0]):
        for c in range(w.shape[1] // 8):
            sc = [float(np.float32(np.float32(w[r, 8 * c + 2 * p] ** 2) + np.float32(w[r, 8 * c + 2 * p + 1] ** 2)))
                  for p in range(4)]
            # brute force over the 6 ways to keep 2 of 4 pairs: max total score,
            # ties resolved towards lower pair indices (lexicographic)
            best = max(itertools.combinations(range(4), 2),
                       key=lambda pq: (sc[pq[0]] + sc[pq[1]], -pq[0], -pq[1]))
            got = tuple(np.nonzero(keep[r, 4 * c:4 * c + 4])[0])
            assert got == best, (r, c, sc)


def test_quantized_weight_invariants():
    cfg = W.CONFIGS["tiny"]
    w = W.expert_weights_bf16(cfg, 3, "gate_up").float().numpy()
    st = S.quantize_weight(w, n_seg=2)
    out, K = w.shape
    assert st["packed"].shape == (out, K // 4)
    assert st["mask"].shape == (out, K // 16)
    assert st["scale"].shape == (out, K // 32)
    nib = S.mask_nibbles(st["mask"])
    popc = np.vectorize(lambda n: bin(int(n)).count("1"))(nib)
    assert (popc == 2).all()                                    # exactly 2 bits per nibble
    dense = S.decode(st["packed"], st["mask"])
    codes = N.unpack_codes(dense)
    # 16 surviving elements per 32-element scale group (pruned ones are code 0)
    kept = np.repeat(S.prune_paired48(w), 2, axis=1).reshape(out, K // 32, 32)
    assert (kept.sum(axis=-1) == 16).all()
    assert (codes.reshape(out, K // 32, 32)[~kept] == 0).all()
    # per-segment globals
    I = out // 2
    pruned = np.where(np.repeat(S.prune_paired48(w), 2, axis=1), w, 0)
    assert st["g"][0] == np.float32(np.float32(np.abs(pruned[:I]).max()) / np.float32(2688))
    assert st["g"][1] == np.float32(np.float32(np.abs(pruned[I:]).max()) / np.float32(2688))


# ------------------------------------------------------------ pair-bitmask --

def test_pair_bitmask_golden(golden):
    g = golden("pair_bitmask.json")
    dense = np.array([g["dense"]], np.uint8)
    packed, mask = S.encode(dense)
    assert packed[0].tolist() == g["packed"]
    assert mask[0].tolist() == g["mask"]
    assert S.decode(packed, mask)[0].tolist() == g["dense"]
    z = g["kept_zero_byte_case"]
    p2, m2 = S.encode(np.array([z["dense"]], np.uint8))
    assert S.mask_nibbles(m2)[0].tolist() == z["canonical_mask_nibbles"]
    assert p2[0].tolist() == z["canonical_packed"]
    p3, m3 = S.encode(np.array([z["dense"]], np.uint8), np.array([z["hint_mask"]], np.uint8))
    assert p3[0].tolist() == z["hint_packed"] and m3[0].tolist() == z["hint_mask"]
    with pytest.raises(S.SparsityError):
        S.encode(np.array([g["bad_dense_three_nonzero"]], np.uint8))
    with pytest.raises(S.SparsityError):
        S.decode(np.zeros((1, 8), np.uint8), np.array([g["bad_mask_three_bits"]], np.uint8))


def test_round_trip_is_lossless_random_masks():
    rng = np.random.default_rng(2)
    legal = np.array([3, 5, 6, 9, 10, 12])
    rows, K = 64, 512
    nib = rng.choice(legal, size=(rows, K // 8))
    mask = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    packed = rng.integers(0, 256, (rows, K // 4)).astype(np.uint8)
    packed[rng.random(packed.shape) < 0.2] = 0                 # kept bytes that are zero
    dense = S.decode(packed, mask)
    # every chunk has nonzero bytes only at kept positions
    kept = np.zeros((rows, K // 8, 4), bool)
    for i in range(4):
        kept[..., i] = (nib >> i) & 1
    assert (dense.reshape(rows, K // 8, 4)[~kept] == 0).all()
    p2, m2 = S.encode(dense, mask)                                  # sparse -> dense -> sparse
    assert np.array_equal(p2, packed) and np.array_equal(m2, mask)
    p3, m3 = S.encode(dense)                                        # dense -> sparse -> dense
    assert np.array_equal(S.decode(p3, m3), dense)


def test_all_six_legal_nibbles_round_trip():
    for n in (3, 5, 6, 9, 10, 12):
        mask = np.array([[n | (n << 4)] * 2], np.uint8)             # K = 32
        packed = np.arange(1, 9, dtype=np.uint8)[None]
        dense = S.decode(packed, mask)
        pos = [i for i in range(4) if (n >> i) & 1]
        assert dense[0, pos[0]] == 1 and dense[0, pos[1]] == 2
        assert S.encode(dense)[0].tolist() == packed.tolist()


def test_storage_sizes_match_pages(golden):
    g = golden("storage_sizes.json")
    cfg = W.CONFIGS["tiny"]
    w = W.expert_weights_bf16(cfg, 0, "down").float().numpy()
    st = S.quantize_weight(w)
    n = w.size
    sparse_b = (st["packed"].nbytes + st["mask"].nbytes + st["scale"].nbytes) / n
    dense_b = (st["dense"].nbytes + st["scale"].nbytes) / n
    assert (sparse_b, dense_b) == S.storage_bytes_per_dense_element() == (0.34375, 0.53125)
    gib = 2.0 ** 30
    fn = g["flash_next"]
    tol = fn["printed_to"] / 2 + 1e-9
    assert abs(fn["routed_params"] * sparse_b / gib - fn["sparse_GiB"]) <= tol
    assert abs(fn["routed_params"] * dense_b / gib - fn["dense_nvfp4_GiB"]) <= tol
    assert abs(fn["routed_params"] * 2 / gib - fn["bf16_GiB"]) <= tol
    q = g["qwen35_397b"]
    routed = q["layers"] * q["experts"] * 3 * q["hidden"] * q["intermediate"]
    saved = routed * (dense_b - sparse_b) / gib
    assert abs(saved - (q["ckpt_dense_GiB"] - q["ckpt_sparse_GiB"])) <= q["printed_to"] + 1e-9
    assert abs(sparse_b / dense_b - g["expert_bytes_ratio_about"]) < 0.005
    assert st["packed"].nbytes * 8 / n == g["value_bits_about"]


# ---------------------------------------------------------------- fold ------

def test_fold_ratio_one_is_identity_and_power_of_two_is_exact():
    sc = np.arange(0, 0x70, dtype=np.uint8)
    assert np.array_equal(S.fold_up_scales(sc, np.float32(0.01), np.float32(0.01)), sc)
    folded = S.fold_up_scales(sc[8:0x60], np.float32(0.01), np.float32(0.02))
    assert np.array_equal(F.e4m3_decode(folded), 2 * F.e4m3_decode(sc[8:0x60]))


# ------------------------------------------------------- operand layouts ----

def test_sparse_metadata_golden(golden):
    g = golden("sparse_meta.json")
    for nib, meta in g["nibble_to_meta"].items():
        assert S.meta_nibble_from_mask_nibble(int(nib)) == meta
    ex = g["layout_example"]
    nib = np.full((ex["out"], ex["K"] // 8), 3, np.uint8)
    nib[ex["row"], ex["chunk"]] = ex["mask_nibble"]
    mask = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    meta = S.repack_meta(mask, ex["gate_up"])
    byte = int(meta[ex["byte_offset"]])
    got = byte >> 4 if ex["nibble"] == "high" else byte & 0xF
    assert got == ex["meta"]
    assert (byte & 0xF) == 4                                   # neighbour chunk keeps nibble 3 -> 4
    tr = g["gate_up_tile_rows"]
    rows = S.tile_rows(tr["out"], True)
    assert rows[128 * tr["tile"] + tr["tile_row"]] == tr["source_row"]
    assert rows[128 * tr["tile_b"] + tr["tile_row_b"]] == tr["source_row_b"]
    assert rows[128 * tr["tile_c"] + tr["tile_row_c"]] == tr["source_row_c"]
    # each tile holds the gate and up rows of the same 64 outputs, once each
    I = tr["out"] // 2
    for t in range(tr["out"] // 128):
        blk = rows[128 * t:128 * t + 128]
        assert sorted(blk) == list(range(64 * t, 64 * t + 64)) + list(range(I + 64 * t, I + 64 * t + 64))
    sf = g["sf_offset_example"]
    assert S.sf_block_offset(sf["row"], sf["j"]) == sf["offset"]


def test_weight_scale_layout_is_a_permutation():
    rng = np.random.default_rng(4)
    sc = rng.integers(0, 0x7F, (256, 16)).astype(np.uint8)
    blk = S.repack_weight_scales(sc, gate_up=True).reshape(2, 4, 512)
    src = S.tile_rows(256, True)
    for t in range(2):
        for kb in range(4):
            for r in range(128):
                for j in range(4):
                    assert blk[t, kb, (r % 32) * 16 + (r // 32) * 4 + j] == sc[src[128 * t + r], 4 * kb + j]
