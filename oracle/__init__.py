"""ctypes front end of the fp64 CPU oracle (``tm_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke``
and by the benchmark's CPU-baseline leg, never by the product path. It shares
no code with the CUDA library; the only thing both sides share is the seeded
input generator, which holds no attention arithmetic.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with the host C++ compiler (no CUDA). It is
    rebuilt unless ``liboracle.so.stamp`` holds the SHA-256 of the compiler
    flags and the source (file times are not trusted across copies)."""
    src = os.path.join(_HERE, "tm_oracle.cpp")
    flags = ["-O2", "-std=c++17", "-fPIC", "-shared", "-pthread"]
    with open(src, "rb") as f:
        digest = hashlib.sha256((" ".join(flags) + "\n").encode() + f.read()).hexdigest()
    stamp = LIB_PATH + ".stamp"
    fresh = os.path.exists(LIB_PATH) and os.path.exists(stamp) and open(stamp).read().strip() == digest
    if force or not fresh:
        subprocess.run(["g++", *flags, src, "-o", LIB_PATH], check=True)
        with open(stamp, "w") as f:
            f.write(digest + "\n")
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB_PATH)
        c_int, c_ll, c_dbl, vp = ctypes.c_int, ctypes.c_longlong, ctypes.c_double, ctypes.c_void_p
        lib.oracle_keep.restype = c_int
        lib.oracle_keep.argtypes = [c_int] * 5 + [c_ll, c_ll]
        lib.oracle_mask_row.restype = c_int
        lib.oracle_mask_row.argtypes = [c_int] * 5 + [c_ll, vp]
        lib.oracle_kept_count_row.restype = c_ll
        lib.oracle_kept_count_row.argtypes = [c_int] * 5 + [c_ll]
        lib.oracle_kept_pairs.restype = c_ll
        lib.oracle_kept_pairs.argtypes = [c_int] * 6
        lib.oracle_attention.restype = c_int
        lib.oracle_attention.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_dbl,
                                         c_int, c_int, c_int, c_int, vp, c_ll, vp, vp, c_int]
        lib.oracle_block_sparse_attention.restype = c_int
        lib.oracle_block_sparse_attention.argtypes = [
            vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_dbl, c_int, c_int, vp, vp, c_ll, vp,
            c_ll, vp, c_int]
        lib.oracle_attention_heads.restype = c_int
        lib.oracle_attention_heads.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int,
                                               c_dbl, vp, vp, c_int, vp, c_ll, vp, c_int]
        lib.oracle_flashprefill_scores.restype = c_int
        lib.oracle_flashprefill_scores.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int,
                                                   c_dbl, c_int, c_int, vp, c_int]
        for name in ("oracle_tile_list_bruteforce", "oracle_tile_list_rows"):
            f = getattr(lib, name)
            f.restype = c_int
            f.argtypes = [c_int] * 7 + [vp, c_ll, ctypes.POINTER(c_ll)]
        lib.oracle_hardware_threads.restype = c_int
        _lib = lib
    return _lib


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def keep(N, causal, S, W, L, i, j) -> int:
    return int(_load().oracle_keep(N, int(causal), S, W, L, i, j))


def mask_row(N, causal, S, W, L, i) -> np.ndarray:
    out = np.zeros(N, np.uint8)
    rc = _load().oracle_mask_row(N, int(causal), S, W, L, i, out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_mask_row: bad argument")
    return out.astype(bool)


def kept_count_row(N, causal, S, W, L, i) -> int:
    return int(_load().oracle_kept_count_row(N, int(causal), S, W, L, i))


def kept_pairs(N, causal, S, W, L, nthreads=None) -> int:
    return int(_load().oracle_kept_pairs(N, int(causal), S, W, L, nthreads or hardware_threads()))


def _tile_list(fn, N, causal, S, W, L, BM, BN):
    cnt = ctypes.c_longlong(0)
    rc = fn(N, int(causal), S, W, L, BM, BN, None, 0, ctypes.byref(cnt))
    if rc != 0:
        raise ValueError("tile list: bad argument")
    out = np.zeros((max(cnt.value, 1), 3), np.int32)
    rc = fn(N, int(causal), S, W, L, BM, BN, out.ctypes.data, cnt.value, ctypes.byref(cnt))
    if rc != 0:
        raise ValueError("tile list: bad argument")
    return out[: cnt.value]


def tile_list_bruteforce(N, causal, S, W, L, BM=128, BN=128) -> np.ndarray:
    """(qb, kb, flag) records by brute force over pairs; flag 1 = every pair kept."""
    return _tile_list(_load().oracle_tile_list_bruteforce, N, causal, S, W, L, BM, BN)


def tile_list_rows(N, causal, S, W, L, BM=128, BN=128) -> np.ndarray:
    """Same records by the row-interval method (fast enough for N = 128K)."""
    return _tile_list(_load().oracle_tile_list_rows, N, causal, S, W, L, BM, BN)


def attention(q, k, v, B, Hq, Hkv, N, D, scale, causal, S=0, W=1, L=0, rows=None,
              nthreads=None, with_rowsum=False):
    """fp64 masked softmax attention.

    q: uint16 [B, N, Hq, D] bf16 bits; k, v: uint16 [B, N, Hkv, D].
    rows: optional list of query rows (same rows for every batch and head).
    Returns out [B, nrows, Hq, D] float64 (and rowsum [B, nrows, Hq] if asked).
    """
    lib = _load()
    for a in (q, k, v):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    assert q.size == B * N * Hq * D and k.size == B * N * Hkv * D and v.size == k.size
    if rows is None:
        nrows, rows_arr, rows_ptr = N, None, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        nrows, rows_ptr = len(rows_arr), rows_arr.ctypes.data
    out = np.zeros((B, nrows, Hq, D), np.float64)
    rs = np.zeros((B, nrows, Hq), np.float64) if with_rowsum else None
    rc = lib.oracle_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, N, D,
                              float(scale), int(causal), S, W, L, rows_ptr, nrows,
                              out.ctypes.data, None if rs is None else rs.ctypes.data,
                              nthreads or hardware_threads())
    if rc != 0:
        raise ValueError("oracle_attention: bad argument")
    return (out, rs) if with_rowsum else out


def block_sparse_attention(q, k, v, B, Hq, Hkv, N, D, scale, offsets, indices, rows=None, BM=128,
                           BS=128, nthreads=None):
    """fp64 block-sparse causal attention from a CSR block index.

    offsets: int32 [B * Hkv * ceil(N / BM) + 1]; indices: int32 [nnz] (k-block
    numbers of each (batch, kv head, q-block)). Returns out [B, nrows, Hq, D].
    """
    lib = _load()
    for a in (q, k, v):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    idx = np.ascontiguousarray(indices, dtype=np.int32)
    assert off.size == B * Hkv * ((N + BM - 1) // BM) + 1
    if rows is None:
        nrows, rows_ptr = N, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        nrows, rows_ptr = len(rows_arr), rows_arr.ctypes.data
    out = np.zeros((B, nrows, Hq, D), np.float64)
    rc = lib.oracle_block_sparse_attention(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, N, D, float(scale), BM, BS,
        off.ctypes.data, idx.ctypes.data if idx.size else None, int(idx.size), rows_ptr, nrows,
        out.ctypes.data, nthreads or hardware_threads())
    if rc != 0:
        raise ValueError("oracle_block_sparse_attention: bad argument")
    return out


def flashprefill_scores(q, k, B, Hq, Hkv, N, D, scale, probes, BS=128, nthreads=None):
    """fp64 block scores Score(I, J) [B * Hkv, nqb, nqb] of the discovery step."""
    lib = _load()
    for a in (q, k):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    nb = (N + BS - 1) // BS
    out = np.zeros((B * Hkv, nb, nb), np.float64)
    rc = lib.oracle_flashprefill_scores(q.ctypes.data, k.ctypes.data, B, Hq, Hkv, N, D,
                                        float(scale), probes, BS, out.ctypes.data,
                                        nthreads or hardware_threads())
    if rc != 0:
        raise ValueError("oracle_flashprefill_scores: bad argument")
    return out


def flashprefill_select(scores, alpha):
    """Kept blocks per list from the scores: J <= I with Score >= alpha * max_J Score.
    Returns (offsets int32 [n_lists + 1], indices int32)."""
    BH, nb, _ = scores.shape
    lists = []
    for bg in range(BH):
        for I in range(nb):
            row = scores[bg, I, :I + 1]
            lists.append(np.flatnonzero(row >= alpha * row.max()).astype(np.int32))
    off = np.zeros(len(lists) + 1, np.int32)
    off[1:] = np.cumsum([len(x) for x in lists])
    return off, (np.concatenate(lists) if lists else np.zeros(0, np.int32))


def attention_heads(q, k, v, B, Hq, Hkv, N, D, scale, S_heads, W_heads, L, rows=None,
                    nthreads=None):
    """fp64 triangle attention with per-head sinks S_heads[h] and windows W_heads[h]."""
    lib = _load()
    for a in (q, k, v):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    Sh = np.ascontiguousarray(S_heads, dtype=np.int32)
    Wh = np.ascontiguousarray(W_heads, dtype=np.int32)
    assert Sh.size == Hq and Wh.size == Hq
    if rows is None:
        nrows, rows_ptr = N, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        nrows, rows_ptr = len(rows_arr), rows_arr.ctypes.data
    out = np.zeros((B, nrows, Hq, D), np.float64)
    rc = lib.oracle_attention_heads(q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, N, D,
                                    float(scale), Sh.ctypes.data, Wh.ctypes.data, L, rows_ptr,
                                    nrows, out.ctypes.data, nthreads or hardware_threads())
    if rc != 0:
        raise ValueError("oracle_attention_heads: bad argument")
    return out
