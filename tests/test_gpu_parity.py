"""Parity of the sm_100a kernels (through the C ABI) with the fp64 CPU oracle.

Bar: bf16 outputs within max-abs 2e-2 and mean-abs 2e-3 of the oracle; tile
lists bit-exact; the pattern's invariants bit-exact where the kernel computes
the same rows the same way.
"""
import math

import numpy as np
import pytest

import oracle
import long_context_prefill_trianglemix_b200 as tm
from long_context_prefill_trianglemix_b200 import inputs as I
from gpu_util import assert_close, from_dev, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_prefill_trianglemix_b200 import build
    build.build_lib()
    yield
    assert tm.tm_get_device_status() == tm.TM_OK


def rand_bits(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return I.f32_to_bf16_bits((g.standard_normal(shape) * scale).astype(np.float32))


def run(q, k, v, B, Hq, Hkv, N, D, scale, causal, S=0, W=1, L=0):
    import torch
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    o = torch.empty_like(dq)
    if causal:
        tm.tm_causal_attn_fwd(dq, dk, dv, o, B, Hq, Hkv, N, D, scale)
    else:
        tm.tm_triangle_attn_fwd(dq, dk, dv, o, B, Hq, Hkv, N, D, scale, S, W, L)
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    return from_dev(o)


# ------------------------------------------------------------------ building blocks


@pytest.mark.parametrize("D", [64, 128])
def test_mma_probe_qk_and_pv(D):
    import torch
    q, k, v = rand_bits((128, D), 1), rand_bits((128, D), 2), rand_bits((128, D), 3)
    s_out = torch.zeros(128 * 128, dtype=torch.float32, device="cuda")
    o_out = torch.zeros(128 * D, dtype=torch.float32, device="cuda")
    tm.tm_debug_mma_probe(to_dev(q), to_dev(k), to_dev(v), s_out, o_out, D)
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    qf, kf, vf = (I.bf16_bits_to_f32(x).astype(np.float64) for x in (q, k, v))
    s_gpu = s_out.cpu().numpy().reshape(128, 128)
    np.testing.assert_allclose(s_gpu, qf @ kf.T, rtol=0, atol=1e-3)
    p = I.bf16_bits_to_f32(I.f32_to_bf16_bits(s_gpu)).astype(np.float64)  # same rounding as the GPU
    o_gpu = o_out.cpu().numpy().reshape(128, D)
    np.testing.assert_allclose(o_gpu, p @ vf, rtol=0, atol=1e-2)


@pytest.mark.parametrize("N,causal,S,W,L", [(512, False, 16, 64, 64), (512, True, 0, 1, 0),
                                            (777, False, 130, 129, 0), (1, False, 0, 1, 0),
                                            (32768, False, 64, 1024, 128),
                                            (131072, False, 64, 2048, 256),
                                            (131072, True, 0, 1, 0)])
def test_device_tile_dump_bit_exact(N, causal, S, W, L):
    import torch
    n = tm.tm_kept_tiles(N, causal, S, W, L)
    buf = torch.full((n * 3 + 4,), -7, dtype=torch.int32, device="cuda")
    cnt = tm.tm_debug_dump_tiles(N, causal, S, W, L, buf, n)
    torch.cuda.synchronize()
    assert cnt == n
    got = buf[: 3 * n].cpu().numpy().reshape(n, 3)
    if N <= 4096:
        want = oracle.tile_list_bruteforce(N, causal, S, W, L)
    else:
        want = oracle.tile_list_rows(N, causal, S, W, L)
    np.testing.assert_array_equal(got, want)
    assert (buf[3 * n:].cpu().numpy() == -7).all()


# ------------------------------------------------------------------ tiny workload, edge cases


def test_tiny_workload_both_layers():
    wl = I.WORKLOADS["tiny"]
    q, k, v = I.make_qkv(wl)
    import torch
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    for layer in range(wl.layers):
        o = torch.empty_like(dq)
        tm.tm_trianglemix_attn_fwd(dq, dk, dv, o, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                                   wl.S, wl.W, wl.L, layer, wl.tri_start)
        torch.cuda.synchronize()
        causal = layer < wl.tri_start
        want = oracle.attention(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, causal,
                                wl.S, wl.W, wl.L)
        assert_close(from_dev(o), want, f"tiny layer {layer}")


EDGE = [  # B, Hq, Hkv, N, D, S, W, L
    (1, 2, 1, 1, 64, 0, 1, 0),
    (1, 2, 2, 127, 128, 3, 17, 5),
    (2, 4, 2, 129, 64, 16, 64, 64),
    (1, 6, 2, 300, 128, 0, 50, 0),
    (1, 8, 2, 500, 128, 64, 128, 37),
    (1, 4, 4, 512, 64, 16, 64, 64),
    (1, 2, 1, 1000, 128, 130, 129, 0),
    (1, 14, 2, 777, 128, 5, 200, 100),
    (3, 4, 1, 383, 64, 1, 1, 1),
    (1, 2, 2, 2049, 128, 64, 300, 129),
    (2, 6, 2, 1100, 64, 16, 200, 100),  # odd group at D = 64: causal items pair q-blocks
]


@pytest.mark.parametrize("B,Hq,Hkv,N,D,S,W,L", EDGE)
def test_edge_cases_match_oracle(B, Hq, Hkv, N, D, S, W, L):
    q = rand_bits((B, N, Hq, D), 11, 2.0)
    k = rand_bits((B, N, Hkv, D), 12, 2.0)
    v = rand_bits((B, N, Hkv, D), 13)
    scale = 1.0 / math.sqrt(D)
    for causal in (False, True):
        got = run(q, k, v, B, Hq, Hkv, N, D, scale, causal, S, W, L)
        want = oracle.attention(q, k, v, B, Hq, Hkv, N, D, scale, causal, S, W, L)
        assert_close(got, want, f"edge {(B, Hq, Hkv, N, D, S, W, L)} causal={causal}")


@pytest.fixture(scope="module")
def mid():
    B, Hq, Hkv, N, D = 1, 8, 2, 1500, 128
    return (B, Hq, Hkv, N, D, rand_bits((B, N, Hq, D), 21, 1.5), rand_bits((B, N, Hkv, D), 22, 1.5),
            rand_bits((B, N, Hkv, D), 23))


def test_invariant_causal_equivalents_bitwise(mid):
    B, Hq, Hkv, N, D, q, k, v = mid
    causal = run(q, k, v, B, Hq, Hkv, N, D, 0.1, True)
    for S, W, L in [(3, 40, N), (3, 40, N + 9), (700, 800, 0), (0, N, 0)]:
        tri = run(q, k, v, B, Hq, Hkv, N, D, 0.1, False, S, W, L)
        np.testing.assert_array_equal(tri, causal)


def test_invariant_last_rows_bitwise(mid):
    B, Hq, Hkv, N, D, q, k, v = mid
    L = 300
    causal = run(q, k, v, B, Hq, Hkv, N, D, 0.1, True)
    tri = run(q, k, v, B, Hq, Hkv, N, D, 0.1, False, 4, 100, L)
    np.testing.assert_array_equal(tri[:, N - L:], causal[:, N - L:])


def test_special_identity_window_bitwise(mid):
    B, Hq, Hkv, N, D, q, k, v = mid
    kk = np.ascontiguousarray(np.repeat(k, Hq // Hkv, axis=2))
    vv = np.ascontiguousarray(np.repeat(v, Hq // Hkv, axis=2))
    out = run(q, kk, vv, B, Hq, Hq, N, D, 0.1, False, 0, 1, 0)
    np.testing.assert_array_equal(out, I.bf16_bits_to_f32(vv))


def test_special_unit_values(mid):
    B, Hq, Hkv, N, D, q, k, _ = mid
    ones = np.full((B, N, Hkv, D), 0x3F80, np.uint16)
    out = run(q, k, ones, B, Hq, Hkv, N, D, 0.1, False, 5, 77, 9)
    assert np.abs(out - 1.0).max() <= 4e-3


def test_special_rising_scores_scale_with_v():
    """Scores that rise by ~100 log2 units along the keys: the running reference
    lags the row max by up to the lazy threshold, so weights reach 2^48 before it
    moves. Attention is linear in v and a power-of-two scale is exact in bf16 and
    fp32, so v * 2^40 must give the output * 2^40 bit for bit, with no overflow."""
    B, Hq, Hkv, N, D = 1, 2, 1, 1500, 128
    q = np.zeros((B, N, Hq, D), np.uint16)
    q[..., 0] = I.f32_to_bf16_bits(np.float32(16.0))
    k = np.zeros((B, N, Hkv, D), np.uint16)
    k[0, :, 0, 0] = I.f32_to_bf16_bits((49.0 * np.arange(N) / N).astype(np.float32))
    v = rand_bits((B, N, Hkv, D), 41)
    v40 = I.f32_to_bf16_bits(I.bf16_bits_to_f32(v) * np.float32(2.0 ** 40))
    scale = 1.0 / math.sqrt(D)
    for causal, S, W, L in ((True, 0, 1, 0), (False, 3, 900, 200)):
        out = run(q, k, v, B, Hq, Hkv, N, D, scale, causal, S, W, L)
        big = run(q, k, v40, B, Hq, Hkv, N, D, scale, causal, S, W, L)
        assert np.isfinite(big).all()
        np.testing.assert_array_equal(big, out * np.float32(2.0 ** 40))
        want = oracle.attention(q, k, v, B, Hq, Hkv, N, D, scale, causal, S, W, L)
        assert_close(out, want, f"rising scores causal={causal}")


def zero_query_expected(vf, pre, N, S, W, L, rows):
    """Closed form for q = 0: the mean of v over each row's kept set (prefix sums).
    vf: v as float64 [B, N, Hkv, D]; pre: its prefix sums along N. Returns [B, rows, Hkv, D]."""
    rows = np.asarray(rows)
    last = rows >= N - min(L, N)
    se = np.where(last, rows + 1, np.minimum(S, rows + 1))
    lo = np.where(last, rows + 1, np.maximum(np.maximum(rows - W + 1, 0), se))
    tot = pre[:, se] + pre[:, rows + 1] - pre[:, lo]
    cnt = (se + (rows + 1 - lo)).astype(np.float64)
    return tot / cnt[None, :, None, None]


# ------------------------------------------------------------------ workload sizes


def device_inputs(wl, layer=0, N=None):
    q, k, v = I.make_qkv(wl, layer, N=N)
    return (q, k, v), (to_dev(q), to_dev(k), to_dev(v))


def run_dev(dq, dk, dv, wl, layer, N=None, S=None, W=None, L=None):
    import torch
    N = wl.N if N is None else N
    o = torch.empty_like(dq)
    tm.tm_trianglemix_attn_fwd(dq, dk, dv, o, wl.B, wl.Hq, wl.Hkv, N, wl.D, wl.scale,
                               wl.S if S is None else S, wl.W if W is None else W,
                               wl.L if L is None else L, layer, wl.tri_start)
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    return o


def check_rows(o_dev, host, wl, causal, rows, N=None, S=None, W=None, L=None, what=""):
    q, k, v = host
    N = wl.N if N is None else N
    idx = __import__("torch").tensor(rows, device="cuda")
    got = from_dev(o_dev[:, idx])
    want = oracle.attention(q, k, v, wl.B, wl.Hq, wl.Hkv, N, wl.D, wl.scale, causal,
                            wl.S if S is None else S, wl.W if W is None else W,
                            wl.L if L is None else L, rows=rows)
    return assert_close(got, want, what)


def test_llama_32k_triangle_all_rows_causal_sampled():
    wl = I.WORKLOADS["llama3-8b-32k"]
    host, (dq, dk, dv) = device_inputs(wl)
    o = run_dev(dq, dk, dv, wl, layer=1)  # triangle
    want = oracle.attention(*host, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, False,
                            wl.S, wl.W, wl.L)
    assert_close(from_dev(o), want, "llama 32K triangle (all rows)")
    o = run_dev(dq, dk, dv, wl, layer=0)  # causal
    check_rows(o, host, wl, True, sample_rows(wl.N, wl.L, 1, 64, 64), what="llama 32K causal")


@pytest.fixture(scope="module")
def llama128k():
    wl = I.WORKLOADS["llama3-8b-128k"]
    return wl, device_inputs(wl)


@pytest.fixture(scope="module")
def llama128k_last_rows(llama128k):
    """The oracle's output on all L = 256 last rows at 128K. Those rows keep every
    causal key whatever S and W are (the pattern's last-Q-K region), so this one
    fp64 computation is the expected value of the last rows of the triangle layer
    at every window and of the causal layer."""
    wl, (host, _) = llama128k
    rows = list(range(wl.N - wl.L, wl.N))
    return rows, oracle.attention(*host, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, True,
                                  rows=rows)


def check_last_rows(o_dev, last, what):
    rows, want = last
    return assert_close(from_dev(o_dev[:, rows[0]:rows[-1] + 1]), want, what + " (all last-L rows)")


def test_llama_128k_triangle_sampled_rows(llama128k, llama128k_last_rows):
    wl, (host, (dq, dk, dv)) = llama128k
    rows = sample_rows(wl.N, wl.L, 2, 64, 96, n_last=0)
    o = run_dev(dq, dk, dv, wl, layer=1)
    check_rows(o, host, wl, False, rows, what="llama 128K triangle W=2048")
    check_last_rows(o, llama128k_last_rows, "llama 128K triangle W=2048")


@pytest.mark.parametrize("W", [512, 1024, 4096])
def test_llama_128k_window_sweep_sampled_rows(llama128k, llama128k_last_rows, W):
    wl, (host, (dq, dk, dv)) = llama128k
    rows = sample_rows(wl.N, wl.L, 3, 32, 48, n_last=0)
    o = run_dev(dq, dk, dv, wl, layer=1, W=W)
    check_rows(o, host, wl, False, rows, W=W, what=f"llama 128K triangle W={W}")
    check_last_rows(o, llama128k_last_rows, f"llama 128K triangle W={W}")


def test_llama_128k_causal_sampled_rows(llama128k, llama128k_last_rows):
    wl, (host, (dq, dk, dv)) = llama128k
    rows = sample_rows(wl.N, wl.L, 4, 32, 32, n_last=0)
    o = run_dev(dq, dk, dv, wl, layer=0)
    check_rows(o, host, wl, True, rows, what="llama 128K causal")
    check_last_rows(o, llama128k_last_rows, "llama 128K causal")


def test_llama_128k_zero_query_every_row(llama128k):
    """q = 0 makes every kept key equally weighted: the output is the mean of v over
    each row's kept set, a closed form that pins the mask of all 131072 rows."""
    import torch
    wl, (host, (dq, dk, dv)) = llama128k
    zq = torch.zeros_like(dq)
    o = run_dev(zq, dk, dv, wl, layer=1)
    vf = I.bf16_bits_to_f32(host[2]).astype(np.float64)
    pre = np.concatenate([np.zeros_like(vf[:, :1]), np.cumsum(vf, axis=1)], axis=1)
    G = wl.Hq // wl.Hkv
    worst, total, n = 0.0, 0.0, 0
    for r0 in range(0, wl.N, 8192):
        rows = np.arange(r0, min(wl.N, r0 + 8192))
        got = from_dev(o[:, r0:r0 + len(rows)]).reshape(wl.B, len(rows), wl.Hkv, G, wl.D)
        want = zero_query_expected(vf, pre, wl.N, wl.S, wl.W, wl.L, rows)[:, :, :, None, :]
        e = np.abs(got - want)
        assert np.isfinite(got).all()
        worst, total, n = max(worst, float(e.max())), total + float(e.sum()), n + e.size
    assert worst <= 2e-2 and total / n <= 2e-3, (worst, total / n)


def test_llama_64k_32layer_two_layers_sampled():
    wl = I.WORKLOADS["llama3-8b-64k-32layer"]
    for layer in (wl.tri_start - 1, wl.tri_start):
        host, (dq, dk, dv) = device_inputs(wl, layer)
        o = run_dev(dq, dk, dv, wl, layer)
        causal = layer < wl.tri_start
        rows = sample_rows(wl.N, wl.L, layer, 32, 48 if causal else 128, n_last=16 if causal else None)
        check_rows(o, host, wl, causal, rows, what=f"llama 64K layer {layer}")


def test_qwen_128k_two_layers_sampled():
    wl = I.WORKLOADS["qwen2.5-7b-128k-28layer"]
    host, (dq, dk, dv) = device_inputs(wl)
    for layer in (wl.tri_start - 1, wl.tri_start):
        o = run_dev(dq, dk, dv, wl, layer)
        causal = layer < wl.tri_start
        rows = sample_rows(wl.N, wl.L, 5 + layer, 32, 32 if causal else 96,
                           n_last=16 if causal else None)
        check_rows(o, host, wl, causal, rows, what=f"qwen 128K layer {layer}")


def test_256k_context_sampled_rows_and_zero_query_every_row():
    """The longest context in the pages' experiments (the FlashPrefill summary
    reports 256K): N = 262144 with the Llama group shape on 8 q heads, the
    split schedule on, sampled rows (all 256 last-L rows) against the oracle and
    the q = 0 closed form on every row."""
    import dataclasses
    import torch
    wl = dataclasses.replace(I.WORKLOADS["llama3-8b-128k"], N=262144, Hq=8, Hkv=2)
    q, k, v = I.make_qkv(wl)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    n = tm.tm_attn_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, False, wl.S, wl.W, wl.L)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(dq)
    tm.tm_triangle_attn_fwd_ws(dq, dk, dv, o, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, wl.S,
                               wl.W, wl.L, ws, n)
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    rows = sample_rows(wl.N, wl.L, 13, 16, 48)  # every one of the L last rows
    check_rows(o, (q, k, v), wl, False, rows, what="256K triangle")
    zq = torch.zeros_like(dq)
    tm.tm_triangle_attn_fwd_ws(zq, dk, dv, o, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, wl.S,
                               wl.W, wl.L, ws, n)
    torch.cuda.synchronize()
    vf = I.bf16_bits_to_f32(v).astype(np.float64)
    pre = np.concatenate([np.zeros_like(vf[:, :1]), np.cumsum(vf, axis=1)], axis=1)
    G = wl.Hq // wl.Hkv
    worst = 0.0
    for r0 in range(0, wl.N, 16384):
        rr = np.arange(r0, min(wl.N, r0 + 16384))
        got = from_dev(o[:, r0:r0 + len(rr)]).reshape(wl.B, len(rr), wl.Hkv, G, wl.D)
        want = zero_query_expected(vf, pre, wl.N, wl.S, wl.W, wl.L, rr)[:, :, :, None, :]
        assert np.isfinite(got).all()
        worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= 2e-2, worst
