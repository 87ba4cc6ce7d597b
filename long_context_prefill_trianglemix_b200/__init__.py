"""TriangleMix prefill attention on NVIDIA B200 (sm_100a).

Python binding of ``libtm.so`` (C ABI in ``include/tm.h``). The functions named
``tm_*`` take the C ABI's arguments one for one; tensors may be passed as
torch tensors (their ``data_ptr()`` is used) or as raw device addresses.
This module only marshals arguments: every step of the attention runs in the
library's CUDA kernels. PyTorch provides device memory and streams.

If the library has not been built, every call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtm.so")

TM_OK, TM_ERR_INVALID_ARG, TM_ERR_UNSUPPORTED, TM_ERR_CUDA, TM_ERR_TIMEOUT = 0, -1, -2, -3, -4
TM_BLOCK_M = TM_BLOCK_N = 128

EXPORTED = (
    "tm_causal_attn_fwd", "tm_triangle_attn_fwd", "tm_trianglemix_attn_fwd",
    "tm_trianglemix_attn_fwd_host",
    "tm_triangle_kept_pairs", "tm_kept_tiles", "tm_triangle_tile_list", "tm_tile_list",
    "tm_debug_dump_tiles", "tm_debug_mma_probe", "tm_debug_schedule", "tm_debug_schedule_window",
    "tm_get_device_status",
    "tm_status_string", "tm_attn_workspace_size", "tm_causal_attn_fwd_ws", "tm_triangle_attn_fwd_ws",
    "tm_trianglemix_attn_fwd_ws", "tm_trianglemix_attn_fwd_noalloc", "tm_block_sparse_attn_fwd",
    "tm_trianglemix_sparse_attn_fwd", "tm_flashprefill_workspace_size",
    "tm_flashprefill_index_capacity", "tm_flashprefill_block_index", "tm_triangle_attn_fwd_heads",
    "tm_debug_inject_stall", "tm_debug_launch_count", "tm_debug_schedule_heads",
)


class TmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded ``libtm.so``; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m long_context_prefill_trianglemix_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, cf, cll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
        sig = {
            "tm_causal_attn_fwd": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp]),
            "tm_triangle_attn_fwd": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci, ci, vp]),
            "tm_trianglemix_attn_fwd": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci, ci,
                                             ci, ci, vp]),
            "tm_trianglemix_attn_fwd_host": (ci, [vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                                  ci, cf, ci, ci, ci, ci, ci, ci, vp]),
            "tm_triangle_kept_pairs": (cll, [ci, ci, ci, ci]),
            "tm_kept_tiles": (cll, [ci, ci, ci, ci, ci]),
            "tm_triangle_tile_list": (ci, [ci, ci, ci, ci, ci, ci, vp, cll,
                                           ctypes.POINTER(cll)]),
            "tm_tile_list": (ci, [ci, ci, ci, ci, ci, ci, ci, vp, cll, ctypes.POINTER(cll)]),
            "tm_debug_dump_tiles": (ci, [ci, ci, ci, ci, ci, vp, cll, ctypes.POINTER(cll), vp]),
            "tm_debug_mma_probe": (ci, [vp, vp, vp, vp, vp, ci, vp]),
            "tm_debug_schedule": (ci, [ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, vp, cll,
                                       ctypes.POINTER(cll)]),
            "tm_debug_schedule_window": (ci, [ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, vp,
                                              cll, ctypes.POINTER(cll)]),
            "tm_attn_workspace_size": (ci, [ci, ci, ci, ci, ci, ci, ci, ci, ci, ci,
                                            ctypes.POINTER(cll)]),
            "tm_causal_attn_fwd_ws": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, cll, vp]),
            "tm_triangle_attn_fwd_ws": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci, ci,
                                             vp, cll, vp]),
            "tm_trianglemix_attn_fwd_ws": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci,
                                                ci, ci, ci, vp, cll, vp]),
            "tm_trianglemix_attn_fwd_noalloc": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci,
                                                     ci, ci, ci, ci, vp]),
            "tm_block_sparse_attn_fwd": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, vp, cll,
                                              vp]),
            "tm_trianglemix_sparse_attn_fwd": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci,
                                                    ci, ci, ci, vp, vp, cll, vp]),
            "tm_flashprefill_workspace_size": (ci, [ci, ci, ci, ci, ci, ci, ctypes.POINTER(cll)]),
            "tm_triangle_attn_fwd_heads": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, vp, ci,
                                                vp, cll, vp]),
            "tm_flashprefill_index_capacity": (cll, [ci, ci, ci]),
            "tm_flashprefill_block_index": (ci, [vp, vp, ci, ci, ci, ci, ci, cf, cf, ci, vp, cll,
                                                 vp, vp, cll, vp, vp]),
            "tm_get_device_status": (ci, [vp]),
            "tm_debug_inject_stall": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci, ci, vp]),
            "tm_status_string": (ctypes.c_char_p, [ci]),
            "tm_debug_launch_count": (cll, []),
            "tm_debug_schedule_heads": (ci, [ci, ci, ci, ci, vp, vp, ci, ci, ci, vp, cll,
                                             ctypes.POINTER(cll)]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().tm_status_string(int(status)).decode()


def _ptr(x):
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    return int(x)


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    return int(s)


def _check(fn: str, rc: int) -> int:
    if rc != TM_OK:
        raise TmError(fn, rc)
    return rc


# ----------------------------------------------------------------------- C ABI, one for one

def tm_causal_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D, scale, stream=None):
    return _check("tm_causal_attn_fwd", lib().tm_causal_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, _stream(stream)))


def tm_triangle_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, stream=None):
    return _check("tm_triangle_attn_fwd", lib().tm_triangle_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, S, W, L, _stream(stream)))


def tm_trianglemix_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
                            stream=None):
    return _check("tm_trianglemix_attn_fwd", lib().tm_trianglemix_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
        _stream(stream)))


def tm_trianglemix_attn_fwd_host(q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, B,
                                 Hq, Hkv, N, D, scale, S, W, L, layer, tri_start, chunk_rows=0,
                                 stream=None):
    return _check("tm_trianglemix_attn_fwd_host", lib().tm_trianglemix_attn_fwd_host(
        _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host), _ptr(q_dev), _ptr(k_dev),
        _ptr(v_dev), _ptr(o_dev), B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
        int(chunk_rows), _stream(stream)))


def tm_causal_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, workspace, workspace_bytes,
                          stream=None):
    return _check("tm_causal_attn_fwd_ws", lib().tm_causal_attn_fwd_ws(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def tm_triangle_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, workspace,
                            workspace_bytes, stream=None):
    return _check("tm_triangle_attn_fwd_ws", lib().tm_triangle_attn_fwd_ws(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, S, W, L, _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def tm_trianglemix_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
                               workspace, workspace_bytes, stream=None):
    return _check("tm_trianglemix_attn_fwd_ws", lib().tm_trianglemix_attn_fwd_ws(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
        _ptr(workspace), int(workspace_bytes), _stream(stream)))


def tm_trianglemix_attn_fwd_noalloc(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, layer,
                                    tri_start, stream=None):
    return _check("tm_trianglemix_attn_fwd_noalloc", lib().tm_trianglemix_attn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
        _stream(stream)))


TM_NOALLOC_SCRATCH_BYTES = 16 << 20


def tm_block_sparse_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D, scale, block_offsets, block_indices,
                             nnz, stream=None):
    return _check("tm_block_sparse_attn_fwd", lib().tm_block_sparse_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, _ptr(block_offsets),
        _ptr(block_indices), int(nnz), _stream(stream)))


def tm_trianglemix_sparse_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, layer,
                                   tri_start, block_offsets, block_indices, nnz, stream=None):
    return _check("tm_trianglemix_sparse_attn_fwd", lib().tm_trianglemix_sparse_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
        _ptr(block_offsets), _ptr(block_indices), int(nnz), _stream(stream)))


def tm_triangle_attn_fwd_heads(q, k, v, o, B, Hq, Hkv, N, D, scale, S_heads, W_heads, L,
                               workspace=None, workspace_bytes=0, stream=None):
    """Triangle attention with per-head sinks and windows (host int sequences of Hq)."""
    Sh = np.ascontiguousarray(S_heads, dtype=np.int32)
    Wh = np.ascontiguousarray(W_heads, dtype=np.int32)
    assert Sh.size == Hq and Wh.size == Hq
    return _check("tm_triangle_attn_fwd_heads", lib().tm_triangle_attn_fwd_heads(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, Sh.ctypes.data,
        Wh.ctypes.data, L, _ptr(workspace), int(workspace_bytes), _stream(stream)))


def tm_flashprefill_workspace_size(B, Hq, Hkv, N, D, probes) -> int:
    n = ctypes.c_longlong(0)
    _check("tm_flashprefill_workspace_size", lib().tm_flashprefill_workspace_size(
        B, Hq, Hkv, N, D, probes, ctypes.byref(n)))
    return n.value


def tm_flashprefill_index_capacity(B, Hkv, N) -> int:
    return int(lib().tm_flashprefill_index_capacity(B, Hkv, N))


def tm_flashprefill_block_index(q, k, B, Hq, Hkv, N, D, scale, alpha, probes, workspace,
                                workspace_bytes, block_offsets, block_indices, cap,
                                scores_out=None, stream=None):
    return _check("tm_flashprefill_block_index", lib().tm_flashprefill_block_index(
        _ptr(q), _ptr(k), B, Hq, Hkv, N, D, scale, alpha, probes, _ptr(workspace),
        int(workspace_bytes), _ptr(block_offsets), _ptr(block_indices), int(cap),
        _ptr(scores_out), _stream(stream)))


def tm_attn_workspace_size(B, Hq, Hkv, N, D, causal, S, W, L, num_ctas=0) -> int:
    """Workspace bytes of the split schedule (0: nothing is split)."""
    n = ctypes.c_longlong(0)
    _check("tm_attn_workspace_size", lib().tm_attn_workspace_size(
        B, Hq, Hkv, N, D, int(causal), S, W, L, num_ctas, ctypes.byref(n)))
    return n.value


def tm_triangle_kept_pairs(N, S, W, L) -> int:
    return int(lib().tm_triangle_kept_pairs(N, S, W, L))


def tm_kept_tiles(N, causal, S, W, L) -> int:
    return int(lib().tm_kept_tiles(N, int(causal), S, W, L))


def tm_tile_list(N, causal, S, W, L, BM=TM_BLOCK_M, BN=TM_BLOCK_N) -> np.ndarray:
    """(qb, kb, full) records of the static tile list, as an int32 [n, 3] array."""
    cnt = ctypes.c_longlong(0)
    _check("tm_tile_list", lib().tm_tile_list(N, int(causal), S, W, L, BM, BN, None, 0,
                                              ctypes.byref(cnt)))
    out = np.zeros((max(cnt.value, 1), 3), np.int32)
    _check("tm_tile_list", lib().tm_tile_list(N, int(causal), S, W, L, BM, BN,
                                              out.ctypes.data, cnt.value, ctypes.byref(cnt)))
    return out[: cnt.value]


def tm_triangle_tile_list(N, S, W, L, BM=TM_BLOCK_M, BN=TM_BLOCK_N) -> np.ndarray:
    cnt = ctypes.c_longlong(0)
    _check("tm_triangle_tile_list", lib().tm_triangle_tile_list(N, S, W, L, BM, BN, None, 0,
                                                                ctypes.byref(cnt)))
    out = np.zeros((max(cnt.value, 1), 3), np.int32)
    _check("tm_triangle_tile_list", lib().tm_triangle_tile_list(
        N, S, W, L, BM, BN, out.ctypes.data, cnt.value, ctypes.byref(cnt)))
    return out[: cnt.value]


def tm_debug_dump_tiles(N, causal, S, W, L, out_dev, cap, stream=None) -> int:
    cnt = ctypes.c_longlong(0)
    _check("tm_debug_dump_tiles", lib().tm_debug_dump_tiles(
        N, int(causal), S, W, L, _ptr(out_dev), cap, ctypes.byref(cnt), _stream(stream)))
    return cnt.value


def tm_debug_mma_probe(q, k, v, s_out, o_out, D, stream=None):
    return _check("tm_debug_mma_probe", lib().tm_debug_mma_probe(
        _ptr(q), _ptr(k), _ptr(v), _ptr(s_out), _ptr(o_out), D, _stream(stream)))


def tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, num_ctas=148, split=False,
                      mix_pairs=False, qb_lo=0, qb_hi=-1) -> np.ndarray:
    """Persistent work split as an int32 [n, 7] array:
    (cta, item, q-block, head0, Q tiles, first tile, end tile); with a window,
    the split of the q-blocks [qb_lo, qb_hi) only."""
    split = int(bool(split)) | (2 if mix_pairs else 0)
    cnt = ctypes.c_longlong(0)
    f = lib().tm_debug_schedule_window
    _check("tm_debug_schedule_window", f(B, Hq, Hkv, N, int(causal), S, W, L, num_ctas,
                                         int(split), qb_lo, qb_hi, None, 0, ctypes.byref(cnt)))
    out = np.zeros((max(cnt.value, 1), 7), np.int32)
    _check("tm_debug_schedule_window", f(B, Hq, Hkv, N, int(causal), S, W, L, num_ctas,
                                         int(split), qb_lo, qb_hi, out.ctypes.data, cnt.value,
                                         ctypes.byref(cnt)))
    return out[: cnt.value]


def tm_debug_schedule_heads(B, Hq, Hkv, N, S_heads, W_heads, L, num_ctas=148,
                            split=False) -> np.ndarray:
    """tm_debug_schedule of a per-head band launch with these bands (records as there)."""
    hs = np.ascontiguousarray(S_heads, dtype=np.int32)
    hw = np.ascontiguousarray(W_heads, dtype=np.int32)
    cnt = ctypes.c_longlong(0)
    f = lib().tm_debug_schedule_heads
    _check("tm_debug_schedule_heads", f(B, Hq, Hkv, N, hs.ctypes.data, hw.ctypes.data, L, num_ctas,
                                        int(bool(split)), None, 0, ctypes.byref(cnt)))
    out = np.zeros((max(cnt.value, 1), 7), np.int32)
    _check("tm_debug_schedule_heads", f(B, Hq, Hkv, N, hs.ctypes.data, hw.ctypes.data, L, num_ctas,
                                        int(bool(split)), out.ctypes.data, cnt.value,
                                        ctypes.byref(cnt)))
    return out[: cnt.value]


def tm_debug_inject_stall(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, stream=None):
    return _check("tm_debug_inject_stall", lib().tm_debug_inject_stall(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, D, scale, S, W, L, _stream(stream)))


def tm_get_device_status(stream=None) -> int:
    return int(lib().tm_get_device_status(_stream(stream)))


def tm_debug_launch_count() -> int:
    return int(lib().tm_debug_launch_count())


# ----------------------------------------------------------------------- torch conveniences

def _shapes(q, k):
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    return B, N, Hq, Hkv, D


def _out(q, out):
    import torch
    return torch.empty_like(q) if out is None else out


def causal_attention(q, k, v, scale=None, out=None, stream=None):
    """Dense causal attention of bf16 CUDA tensors q [B,N,Hq,D], k/v [B,N,Hkv,D]."""
    B, N, Hq, Hkv, D = _shapes(q, k)
    o = _out(q, out)
    tm_causal_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D,
                       1.0 / math.sqrt(D) if scale is None else scale, stream)
    return o


def triangle_attention(q, k, v, S, W, L, scale=None, out=None, stream=None):
    """Triangle attention (sinks S, window W, last L rows) of bf16 CUDA tensors."""
    B, N, Hq, Hkv, D = _shapes(q, k)
    o = _out(q, out)
    tm_triangle_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D,
                         1.0 / math.sqrt(D) if scale is None else scale, S, W, L, stream)
    return o


def trianglemix_attention(q, k, v, S, W, L, layer, tri_start, scale=None, out=None, stream=None):
    """One layer of the TriangleMix schedule: causal below tri_start, triangle from it on."""
    B, N, Hq, Hkv, D = _shapes(q, k)
    o = _out(q, out)
    tm_trianglemix_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D,
                            1.0 / math.sqrt(D) if scale is None else scale, S, W, L, layer,
                            tri_start, stream)
    return o
