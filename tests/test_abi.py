"""The C-ABI library without a GPU: it loads, exports every declared symbol,
rejects bad arguments before touching CUDA, and its host tile-list export
matches the oracle bit for bit."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
import long_context_prefill_trianglemix_b200 as tm
from long_context_prefill_trianglemix_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build_lib()
    yield


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "tm.h")).read()
    return sorted(set(re.findall(r"TM_API\s+[\w\s\*]+?\b(tm_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    syms = declared_symbols()
    assert len(syms) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", tm.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (tm_\w+)", out))
    for s in syms:
        assert s in exported, s
    assert set(tm.EXPORTED) == set(syms)
    L = tm.lib()
    for s in syms:
        assert getattr(L, s) is not None


def test_only_the_abi_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", tm.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    names = set(re.findall(r"\bT (\w+)", out))
    assert {n for n in names if not n.startswith("tm_")} <= {"_init", "_fini"}


def test_status_strings():
    for code in (0, -1, -2, -3, -4, 99):
        assert isinstance(tm.status_string(code), str) and tm.status_string(code)


FAKE = 0x10000  # a 16-byte-aligned address that is never dereferenced (calls fail validation)


@pytest.mark.parametrize("args,want", [
    ((0, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1), tm.TM_ERR_INVALID_ARG),   # null q
    ((FAKE, FAKE, FAKE, FAKE + 0x100000, 0, 4, 4, 64, 64, 0.1), tm.TM_ERR_INVALID_ARG),  # B < 1
    ((FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 3, 64, 64, 0.1), tm.TM_ERR_INVALID_ARG),  # Hq % Hkv
    ((FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 0, 64, 0.1), tm.TM_ERR_INVALID_ARG),   # N < 1
    ((FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 96, 0.1), tm.TM_ERR_UNSUPPORTED),  # D
    ((FAKE + 8, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1), tm.TM_ERR_INVALID_ARG),  # align
    ((FAKE, FAKE, FAKE, FAKE + 0x100, 1, 4, 4, 64, 64, 0.1), tm.TM_ERR_INVALID_ARG),     # o aliases q
    ((FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, float("nan")), tm.TM_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.0), tm.TM_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, -0.5), tm.TM_ERR_INVALID_ARG),
])
def test_causal_validation(args, want):
    assert tm.lib().tm_causal_attn_fwd(*args, None) == want


@pytest.mark.parametrize("S,W,L", [(-1, 4, 0), (0, 0, 0), (0, 4, -2)])
def test_triangle_pattern_validation(S, W, L):
    args = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1)
    assert tm.lib().tm_triangle_attn_fwd(*args, S, W, L, None) == tm.TM_ERR_INVALID_ARG


def test_layer_schedule_validation():
    args = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1, 4, 8, 2)
    assert tm.lib().tm_trianglemix_attn_fwd(*args, -1, 3, None) == tm.TM_ERR_INVALID_ARG
    assert tm.lib().tm_trianglemix_attn_fwd(*args, 0, -3, None) == tm.TM_ERR_INVALID_ARG
    # the bad window is only checked when the triangle kernel is chosen
    bad = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1, 4, 0, 2)
    assert tm.lib().tm_trianglemix_attn_fwd(*bad, 5, 3, None) == tm.TM_ERR_INVALID_ARG


def test_binding_raises_on_error():
    with pytest.raises(tm.TmError) as e:
        tm.tm_causal_attn_fwd(0, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1, stream=0)
    assert e.value.status == tm.TM_ERR_INVALID_ARG


TILE_CASES = [(1, 0, 1, 0), (100, 3, 10, 5), (128, 16, 64, 64), (129, 16, 64, 0), (500, 0, 1, 0),
              (512, 16, 64, 64), (1000, 64, 200, 130), (2049, 64, 300, 1), (777, 130, 129, 0),
              (4096, 64, 1024, 128), (3000, 5000, 1, 0), (3000, 0, 5000, 0), (3000, 1, 1, 5000)]


@pytest.mark.parametrize("N,S,W,L", TILE_CASES)
@pytest.mark.parametrize("BM,BN", [(128, 128), (64, 128), (128, 64), (32, 32)])
def test_host_tile_list_bit_exact(N, S, W, L, BM, BN):
    for causal in (False, True):
        got = tm.tm_tile_list(N, causal, S, W, L, BM, BN)
        want = oracle.tile_list_bruteforce(N, causal, S, W, L, BM, BN)
        np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(tm.tm_triangle_tile_list(N, S, W, L, BM, BN),
                                  tm.tm_tile_list(N, False, S, W, L, BM, BN))


@pytest.mark.parametrize("N,S,W,L", [(32768, 64, 1024, 128), (65536, 64, 1024, 128),
                                     (131072, 64, 512, 256), (131072, 64, 2048, 256),
                                     (131072, 64, 4096, 256), (131072, 64, 1024, 128)])
def test_host_tile_list_bit_exact_large(N, S, W, L):
    got = tm.tm_triangle_tile_list(N, S, W, L)
    want = oracle.tile_list_rows(N, False, S, W, L)
    np.testing.assert_array_equal(got, want)
    assert tm.tm_kept_tiles(N, False, S, W, L) == len(want)


def test_tile_list_capacity_and_count():
    cnt = ctypes.c_longlong(0)
    buf = np.zeros((3, 3), np.int32)
    rc = tm.lib().tm_tile_list(512, 0, 16, 64, 64, 128, 128, buf.ctypes.data, 3, ctypes.byref(cnt))
    assert rc == 0 and cnt.value == 10
    np.testing.assert_array_equal(buf, tm.tm_tile_list(512, False, 16, 64, 64)[:3])
    assert tm.lib().tm_tile_list(512, 0, 16, 64, 64, 128, 128, None, 5,
                                 ctypes.byref(cnt)) == tm.TM_ERR_INVALID_ARG


def test_kept_pairs_and_tiles():
    for N, S, W, L in [(512, 16, 64, 64), (131072, 64, 2048, 256), (1000, 0, 1, 0)]:
        assert tm.tm_triangle_kept_pairs(N, S, W, L) == oracle.kept_pairs(N, False, S, W, L)
    assert tm.tm_kept_tiles(131072, True, 0, 1, 0) == 1024 * 1025 // 2
    assert tm.tm_triangle_kept_pairs(10, 0, 0, 0) == -1


WS_ARGS = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1)


@pytest.mark.parametrize("ws,nbytes", [(0, 256), (FAKE + 0x200008, 256), (FAKE + 0x200000, -1),
                                       (FAKE + 0x100, 4096), (FAKE + 0x100000 - 64, 4096)])
def test_workspace_validation(ws, nbytes):
    L = tm.lib()
    assert L.tm_triangle_attn_fwd_ws(*WS_ARGS, 4, 8, 2, ws, nbytes, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_causal_attn_fwd_ws(*WS_ARGS, ws, nbytes, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_trianglemix_attn_fwd_ws(*WS_ARGS, 4, 8, 2, 3, 1, ws, nbytes,
                                        None) == tm.TM_ERR_INVALID_ARG


def test_workspace_size_arguments():
    n = ctypes.c_longlong(-1)
    L = tm.lib()
    assert L.tm_attn_workspace_size(1, 4, 3, 4096, 128, 0, 0, 1, 0, 148, ctypes.byref(n)) == \
        tm.TM_ERR_INVALID_ARG
    assert L.tm_attn_workspace_size(1, 4, 1, 4096, 96, 0, 0, 1, 0, 148, ctypes.byref(n)) == \
        tm.TM_ERR_UNSUPPORTED
    assert L.tm_attn_workspace_size(1, 4, 1, 4096, 128, 0, 0, 0, 0, 148, ctypes.byref(n)) == \
        tm.TM_ERR_INVALID_ARG
    assert L.tm_attn_workspace_size(1, 4, 1, 4096, 128, 0, 0, 1, 0, 148, None) == \
        tm.TM_ERR_INVALID_ARG
    assert L.tm_attn_workspace_size(1, 4, 1, 4096, 128, 0, 16, 64, 64, 148, ctypes.byref(n)) == 0
    assert n.value >= 0


def test_block_sparse_validation():
    L = tm.lib()
    args = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1)
    off = FAKE + 0x200000
    assert L.tm_block_sparse_attn_fwd(*args, None, off, 4, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_block_sparse_attn_fwd(*args, off, None, 4, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_block_sparse_attn_fwd(*args, off, off, -1, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_block_sparse_attn_fwd(*args, off + 2, off, 4, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_block_sparse_attn_fwd(*args, off, off, 1 << 31, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_trianglemix_sparse_attn_fwd(*args, 4, 8, 2, -1, 1, off, off, 4,
                                            None) == tm.TM_ERR_INVALID_ARG
    # the triangle branch ignores the index but still checks the pattern
    assert L.tm_trianglemix_sparse_attn_fwd(*args, 4, 0, 2, 3, 1, None, None, 0,
                                            None) == tm.TM_ERR_INVALID_ARG


def test_per_head_band_validation():
    L = tm.lib()
    args = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1)
    good = (ctypes.c_int * 4)(1, 2, 3, 4)
    bad_w = (ctypes.c_int * 4)(1, 0, 3, 4)
    bad_s = (ctypes.c_int * 4)(1, -2, 3, 4)
    assert L.tm_triangle_attn_fwd_heads(*args, None, good, 2, None, 0, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_triangle_attn_fwd_heads(*args, good, bad_w, 2, None, 0, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_triangle_attn_fwd_heads(*args, bad_s, good, 2, None, 0, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_triangle_attn_fwd_heads(*args, good, good, -1, None, 0, None) == tm.TM_ERR_INVALID_ARG


def test_seeded_head_bands():
    from long_context_prefill_trianglemix_b200 import inputs as I
    S, W = I.head_bands(32, 0)
    assert S.shape == (32,) and W.shape == (32,)
    assert set(S.tolist()) <= {0, 64} and (W >= 512).all() and (W <= 4096).all()
    assert len(set(W.tolist())) > 20
    S2, W2 = I.head_bands(32, 0)
    assert np.array_equal(S, S2) and np.array_equal(W, W2)


def test_inject_stall_validates_before_launch():
    args = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1)
    assert tm.lib().tm_debug_inject_stall(*args, 4, 0, 2, None) == tm.TM_ERR_INVALID_ARG
    assert tm.lib().tm_debug_inject_stall(0, *args[1:], 4, 8, 2, None) == tm.TM_ERR_INVALID_ARG


def test_host_streamed_call_validation():
    """Every rejection happens before any CUDA call (none of these pointers is
    ever dereferenced)."""
    L = tm.lib()
    H = 0x40000000  # stands for host buffers
    dev = (FAKE, FAKE, FAKE, FAKE + 0x100000)
    geo = (1, 4, 4, 64, 64, 0.1, 4, 8, 2)

    def call(host=(H, H, H, H + 0x100000), devp=dev, geometry=geo, layer=1, tri_start=1, chunk=0):
        return L.tm_trianglemix_attn_fwd_host(*host, *devp, *geometry, layer, tri_start, chunk,
                                              None)
    for i in range(4):  # a NULL host buffer
        host = [H, H, H, H + 0x100000]
        host[i] = 0
        assert call(host=tuple(host)) == tm.TM_ERR_INVALID_ARG
    assert call(devp=(0, FAKE, FAKE, FAKE + 0x100000)) == tm.TM_ERR_INVALID_ARG   # NULL device q
    assert call(devp=(FAKE, FAKE, FAKE, FAKE + 0x100)) == tm.TM_ERR_INVALID_ARG   # o_dev aliases q
    for chunk in (-128, 100, 129):                                                # not k * 128
        assert call(chunk=chunk) == tm.TM_ERR_INVALID_ARG
    assert call(layer=-1) == tm.TM_ERR_INVALID_ARG
    assert call(geometry=(1, 4, 4, 64, 64, 0.1, 4, 0, 2)) == tm.TM_ERR_INVALID_ARG  # W = 0
