"""GPU parity of the grouped GEMMs when every CTA pair runs several work items.

The grouped GEMM is persistent: pair pid of npairs walks the (expert, token tile,
weight-tile pair) items pid, pid + npairs, ... and alternates two TMEM accumulator
buffers, so from its second item on a pair uses the second buffer, the accumulator
phase flips, the expert record it loaded a tile ahead and the (tile, pair) stride
walk.  The other GEMM tests have fewer items than the device has pairs, so here:

* the layers of tests/test_gpu_gemm.py run with the launch capped at 1, 2 and 3 pairs
  (moesq_set_gemm_pair_limit), so one pair runs every item or the stride walk wraps
  over weight-tile pairs with a remainder; every output element is compared with the
  oracle (FP32 and bf16 gate_up, SwiGLU + requant, bf16 down, the dense comparison
  kernel);
* a layer whose item list is many times the device's own pair count (32 experts,
  top-4, H = 512, I = 256, 8192 tokens: 512 items per GEMM) runs at the uncapped
  launch, and the whole layer is compared element by element; on one pair its 512
  items exceed the set-up table of per-item experts (128), so the roles walk them;
* a decode-sized layer (64 experts holding one 128-token tile each) at 8, 16 and all
  pairs, where each pair looks its items' experts up in a table built at set-up rather
  than walking the expert records (the kernel's rule, restated in table_used);
* wide items of the SwiGLU gate_up GEMM (two 128-token tiles of one expert, one MMA
  of N <= 256 per K step, a single 256-column accumulator): forced on layers whose
  experts hold 0, 7, 40, 128, 129, 250, 256, 300, 517 and 700 tokens, so items with a
  full and a ragged second tile (N = 144 .. 256), single-tile items of <= 16, <= 64
  and 128 tokens and empty experts all occur, at 1, 3 and all pairs, with the fold
  and with separate gate and up globals; the many-item layer runs forced to wide
  items as well (256 items per pair: the accumulator columns alternate many times).

Tolerances are those of tests/test_gpu_gemm.py (1e-5 * sum|a w| in FP32, one bf16 ulp
beyond it; requantised codes bit-exact where the NVFP4 rule fixes them).  The grouped
GEMM is the kernel line of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card.
"""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
import workloads as W
from tests import test_gpu_dense as TD
from tests import test_gpu_gemm as TG

pytestmark = pytest.mark.gpu

LIMITS = (1, 2, 3)
CAPPED = ("tiny", "ragged_multi_tile", "sparse_routing", "mid_ktail", "deep_k", "exact_per_half_alpha")
MANY = W.LayerConfig("many_items", 46, 32, 4, 512, 256, (8192,), "uniform", True)
# decode-sized: 64 experts of one tile each, so a pair's walk would jump over many experts
# an item and the set-up table of per-item experts is used instead (at every launch size
# below; see table_used)
DECODE = W.LayerConfig("decode_items", 49, 64, 2, 512, 256, (256,), "uniform", True)
# tokens per expert of the wide-item layers (top-1 routing, built directly)
WIDE_COUNTS = (0, 7, 40, 128, 129, 250, 256, 300, 517, 700)
WIDE = {
    "fold": (W.LayerConfig("wide_fold", 47, 10, 1, 1024, 384, (2327,), "uniform", True), {}),
    "exact": (W.LayerConfig("wide_exact", 48, 10, 1, 512, 256, (2327,), "uniform", True), dict(exact=True)),
}


def items(layer, out_rows):
    """Work items of one grouped GEMM: token tiles of 128 times weight-tile pairs."""
    counts = np.diff(layer.perm["expert_offsets"])
    mt = out_rows // 128
    return int(((counts + 127) // 128).sum()) * ((mt + 1) // 2)


class TilesPerItem:
    def __init__(self, n):
        self.n = n

    def __enter__(self):
        M.moesq_set_gemm_tiles_per_item(self.n)
        return self

    def __exit__(self, *a):
        M.moesq_set_gemm_tiles_per_item(0)


class PairLimit:
    def __init__(self, n):
        self.n = n

    def __enter__(self):
        M.moesq_set_gemm_pair_limit(self.n)
        return self

    def __exit__(self, *a):
        M.moesq_set_gemm_pair_limit(0)


@pytest.fixture(scope="module", params=CAPPED)
def capped_layer(request):
    cfg, T, *opt = TG.CASES[request.param]
    return TG.Layer(cfg, T, **(opt[0] if opt else {}))


@pytest.mark.parametrize("limit", LIMITS)
def test_capped_pairs_gate_up_f32(capped_layer, limit):
    with PairLimit(limit):
        assert M.moesq_gemm_launch_pairs(0, M.EPI_F32) == limit
        TG.test_gate_up_f32_within_tolerance(capped_layer)


@pytest.mark.parametrize("limit", LIMITS)
def test_capped_pairs_gate_up_bf16(capped_layer, limit):
    with PairLimit(limit):
        TG.test_gate_up_bf16_within_tolerance(capped_layer)


@pytest.mark.parametrize("limit", LIMITS)
def test_capped_pairs_swiglu_requant(capped_layer, limit):
    with PairLimit(limit):
        TG.test_swiglu_requant_epilogue(capped_layer)


@pytest.mark.parametrize("limit", LIMITS)
def test_capped_pairs_down_bf16(capped_layer, limit):
    with PairLimit(limit):
        TG.test_down_bf16_within_tolerance(capped_layer)


@pytest.mark.parametrize("limit", (1, 3))
def test_capped_pairs_forward(capped_layer, limit):
    with PairLimit(limit):
        TG.test_moe_forward_end_to_end(capped_layer)


@pytest.fixture(scope="module")
def dense_layer():
    cfg, T, *opt = TG.CASES["ragged_multi_tile"]
    L = TG.Layer(cfg, T, **(opt[0] if opt else {}))
    L.dense_gu = TD.DenseLinear(L.gu, L.dgu)
    L.dense_dn = TD.DenseLinear(L.dn, L.ddn)
    return L


@pytest.mark.parametrize("limit", (1, 3))
def test_capped_pairs_dense_comparison(dense_layer, limit):
    """The dense comparison kernel on one and on three pairs, against the same oracle."""
    with PairLimit(limit):
        assert M.moesq_gemm_launch_pairs(1, M.EPI_F32) == limit
        TD.test_dense_gate_up_f32_within_tolerance(dense_layer)
        TD.test_dense_swiglu_requant_epilogue(dense_layer)
        TD.test_dense_down_bf16_within_tolerance(dense_layer)


@pytest.fixture(scope="module")
def many_layer():
    M.moesq_set_gemm_pair_limit(0)
    L = TG.Layer(MANY, 8192)
    pairs = max(M.moesq_gemm_launch_pairs(0, e) for e in (M.EPI_F32, M.EPI_BF16, M.EPI_SWIGLU_NVFP4))
    n_gu, n_dn = items(L, 2 * MANY.I), items(L, MANY.H)
    # every pair of the uncapped launch runs at least two items of each GEMM
    assert n_gu >= 2 * pairs and n_dn >= 2 * pairs, (n_gu, n_dn, pairs)
    return L


def test_many_items_gate_up_f32(many_layer):
    TG.test_gate_up_f32_within_tolerance(many_layer)


def test_many_items_gate_up_bf16(many_layer):
    TG.test_gate_up_bf16_within_tolerance(many_layer)


def test_many_items_swiglu_requant(many_layer):
    TG.test_swiglu_requant_epilogue(many_layer)


def test_many_items_down_bf16(many_layer):
    TG.test_down_bf16_within_tolerance(many_layer)


def test_many_items_on_one_pair(many_layer):
    """512 items on one pair: more than the set-up item table holds, so every role walks
    the items and searches the expert records."""
    with PairLimit(1):
        TG.test_swiglu_requant_epilogue(many_layer)
        TG.test_down_bf16_within_tolerance(many_layer)


def test_many_items_forward(many_layer):
    TG.test_moe_forward_end_to_end(many_layer)
    TG.test_forward_is_deterministic(many_layer)


def test_pair_limit_arguments():
    with pytest.raises(M.MoesqError):
        M.moesq_set_gemm_pair_limit(-1)
    full = M.moesq_gemm_launch_pairs(0, M.EPI_BF16)
    assert full >= 1
    with PairLimit(full + 100):
        assert M.moesq_gemm_launch_pairs(0, M.EPI_BF16) == full
    torch.cuda.synchronize()


def test_many_items_swiglu_requant_wide(many_layer):
    assert M.moesq_gemm_tiles_per_item(0, M.EPI_SWIGLU_NVFP4, MANY.H, MANY.E, many_layer.S) == 1
    with TilesPerItem(2):
        assert M.moesq_gemm_tiles_per_item(0, M.EPI_SWIGLU_NVFP4, MANY.H, MANY.E, many_layer.S) == 2
        TG.test_swiglu_requant_epilogue(many_layer)
        TG.test_moe_forward_end_to_end(many_layer)


def wide_routing(cfg, seed):
    """Top-1 routing with WIDE_COUNTS tokens per expert, in a seeded token order."""
    ids = np.repeat(np.arange(cfg.E), WIDE_COUNTS)
    np.random.default_rng(seed).shuffle(ids)
    return ids.reshape(-1, 1), np.ones((ids.size, 1), np.float32)


@pytest.fixture(scope="module", params=sorted(WIDE))
def wide_layer(request):
    cfg, opt = WIDE[request.param]
    T = int(sum(WIDE_COUNTS))
    assert cfg.E == len(WIDE_COUNTS) and cfg.H % 512 == 0
    return TG.Layer(cfg, T, routing=wide_routing(cfg, cfg.seed), **opt)


@pytest.mark.parametrize("limit", (0, 1, 3))
def test_wide_items_swiglu_requant(wide_layer, limit):
    L = wide_layer
    with TilesPerItem(2), PairLimit(limit):
        assert M.moesq_gemm_tiles_per_item(0, M.EPI_SWIGLU_NVFP4, L.cfg.H, L.cfg.E, L.S) == 2
        TG.test_swiglu_requant_epilogue(L)


@pytest.mark.parametrize("limit", (0, 3))
def test_wide_items_forward(wide_layer, limit):
    with TilesPerItem(2), PairLimit(limit):
        TG.test_moe_forward_end_to_end(wide_layer)
        TG.test_forward_is_deterministic(wide_layer)


def test_tiles_per_item_arguments():
    sw, bf = M.EPI_SWIGLU_NVFP4, M.EPI_BF16
    for bad in (-1, 3):
        with pytest.raises(M.MoesqError):
            M.moesq_set_gemm_tiles_per_item(bad)
    assert M.moesq_gemm_tiles_per_item(0, sw, 4096, 128, 256 * 128) == 2      # 256 slots per expert
    assert M.moesq_gemm_tiles_per_item(0, sw, 4096, 128, 256 * 128 - 1) == 1
    assert M.moesq_gemm_tiles_per_item(0, sw, 4096 + 256, 128, 1 << 20) == 1  # K % 512 != 0
    assert M.moesq_gemm_tiles_per_item(0, sw, 2048, 128, 1 << 20) == 1        # K < 4096
    assert M.moesq_gemm_tiles_per_item(0, bf, 4096, 128, 1 << 20) == 1        # SwiGLU only
    assert M.moesq_gemm_tiles_per_item(1, sw, 4096, 128, 1 << 20) == 1        # sparse only
    with TilesPerItem(2):
        assert M.moesq_gemm_tiles_per_item(0, sw, 4096, 128, 1) == 2
        assert M.moesq_gemm_tiles_per_item(0, sw, 4096 + 256, 128, 1) == 1
    with TilesPerItem(1):
        assert M.moesq_gemm_tiles_per_item(0, sw, 4096, 128, 1 << 20) == 1


def table_used(counts, out_rows, pairs):
    """The kernel's rule for the per-item expert table, for pair 0: 2 to 128 items, and a
    walk that would advance over two or more experts an item on average."""
    tiles = int(((counts + 127) // 128).sum())
    nz = int((counts > 0).sum())
    mt2 = (out_rows // 128 + 1) // 2
    mine = -(-tiles * mt2 // pairs)
    return 2 <= mine <= 128 and 2 * tiles < (pairs // mt2) * nz


@pytest.fixture(scope="module")
def decode_layer():
    return TG.Layer(DECODE, 256)


@pytest.mark.parametrize("limit", (0, 8, 16))
def test_decode_items_from_table(decode_layer, limit):
    L = decode_layer
    counts = np.diff(L.perm["expert_offsets"])
    with PairLimit(limit):
        pairs = M.moesq_gemm_launch_pairs(0, M.EPI_BF16)
        assert table_used(counts, 2 * DECODE.I, pairs) and table_used(counts, DECODE.H, pairs)
        TG.test_gate_up_f32_within_tolerance(L)
        TG.test_swiglu_requant_epilogue(L)
        TG.test_down_bf16_within_tolerance(L)
        TG.test_moe_forward_end_to_end(L)
