"""The C-ABI library builds, loads and exports every symbol include/moesq.h
declares; argument validation answers synchronously (CPU only, no compute)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sparse_nvfp4_moe_b200 import build
    build.build()
    from sparse_nvfp4_moe_b200 import _lib
    return _lib.lib()


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "moesq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(moesq_[a-z0-9_]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(lib):
    syms = header_symbols()
    assert len(syms) >= 19
    for s in syms:
        assert hasattr(lib, s), s


def test_binding_covers_header():
    from sparse_nvfp4_moe_b200 import _lib
    assert set(_lib.declared_symbols()) == set(header_symbols())


def test_status_strings_and_version(lib):
    from sparse_nvfp4_moe_b200 import _lib
    assert lib.moesq_abi_version() == 1
    for code in range(8):
        assert _lib.status_string(code)
    assert _lib.status_string(99) == "unknown status"


def test_argument_validation_is_synchronous(lib):
    from sparse_nvfp4_moe_b200 import _lib
    INVALID, SHAPE, WS = 1, 2, 6
    assert lib.moesq_decode(None, None, None, 4, 128, None, None) == INVALID
    buf = ctypes.create_string_buffer(4096 + 16)
    p = (ctypes.addressof(buf) + 15) & ~15
    assert lib.moesq_decode(p, p, p, 4, 100, None, None) == SHAPE
    assert lib.moesq_decode(p + 1, p, p, 4, 128, None, None) == INVALID      # misaligned
    assert lib.moesq_decode(p, p, p, 0, 128, None, None) == 0                # empty: nothing to do
    assert lib.moesq_permute(p, 4, 2, 8, p, p, p, p, None, 0, None, None) == WS
    assert lib.moesq_permute(p, 4, 0, 8, p, p, p, p, p, 4096, None, None) == INVALID
    assert lib.moesq_quant_act(p, 100, None, None, None, 1, p, 4, 0, p, p, None) == SHAPE
    assert lib.moesq_repack_meta(p, p, p, 1, 192, 256, 0, p, p, p, None, None) == SHAPE
    W = _lib.Linear(p, p, p, p, 256, 256, 8, 0)
    assert lib.moesq_grouped_gemm(ctypes.byref(W), p, p, p, p, p, 0, 0, 0, None, p, None, None, 0,
                                  None, None) == 0                             # S == 0
    assert lib.moesq_grouped_gemm(ctypes.byref(W), p, p, p, p, p, 64, 64, 0, None, p, None, None, 0,
                                  None, None) == SHAPE                         # P_cap too small
    assert lib.moesq_grouped_gemm(ctypes.byref(W), p, p, p, p, p, 64, 2048, 2, None, p, None, None, 0,
                                  None, None) == INVALID                       # SwiGLU on down


def test_selftest_arguments_checked_before_launch(lib):
    INVALID = 1
    buf = ctypes.create_string_buffer(64)
    p = ctypes.addressof(buf)
    assert lib.moesq_selftest_wait_timeout(None, 1000, p, None) == INVALID
    assert lib.moesq_selftest_wait_timeout(p, 0, p, None) == INVALID
    assert lib.moesq_selftest_wait_timeout(p, 200000000, p, None) == INVALID   # limit above 0.1 s


def test_size_queries(lib):
    from sparse_nvfp4_moe_b200 import _lib
    assert _lib.repack_sizes(256, 256) == (2 * 1 * 2048, 2 * 2 * 512)
    assert _lib.repack_sizes(128, 384) == (2 * 2048, 3 * 512)
    assert _lib.padded_rows(0, 8) == 0
    assert _lib.padded_rows(1, 8) == 128
    assert _lib.padded_rows(300, 2) == ((300 + 2 * 127 + 127) // 128) * 128
    assert _lib.permute_workspace_size(64, 2, 8) == (1 * 8 + 8) * 4      # chunk counts + expert totals
    assert _lib.quant_weight_workspace_size(8, 2) == 64


def test_host_forward_workspace_layout(lib):
    """The host-buffer forward holds the forward workspace of one token chunk and one
    input/output buffer set per chunk: chunks of max(2048, ceil(T / 8)) tokens, at most
    8 of them (host logic only; no GPU needed)."""
    from sparse_nvfp4_moe_b200 import _lib
    layer = _lib.MoeLayer()
    layer.E, layer.k, layer.H, layer.I = 128, 8, 2048, 768

    def a256(x):
        return (x + 255) // 256 * 256

    def expected(T):
        tc = min(max(2048, -(-T // 8)), T)
        n = -(-T // tc)
        fw = _lib.moe_forward_workspace_size(layer, tc)
        per_set = 2 * a256(tc * layer.H * 2) + 2 * a256(tc * layer.k * 4)
        return a256(fw) + n * per_set, n

    for T, chunks in [(1, 1), (2048, 1), (2049, 2), (5000, 3), (16384, 8), (100000, 8)]:
        want, n = expected(T)
        assert n == chunks
        assert _lib.moe_forward_host_workspace_size(layer, T) == want
    # the forward workspace never shrinks with more tokens (a chunk's is enough for a shorter one)
    sizes = [_lib.moe_forward_workspace_size(layer, t) for t in (1, 100, 904, 2047, 2048)]
    assert sizes == sorted(sizes)
