"""Parity of triangle attention with per-head bands (tm_triangle_attn_fwd_heads,
through the C ABI) with the fp64 oracle: random bands with the extremes
(S = 0, W = 1, S or W past N), odd group sizes, D = 64, ragged N; equal bands
bit for bit against tm_triangle_attn_fwd; the Llama-3-8B 32K shape with
seeded per-head windows on every row; a tensor-parallel shard at 128K with
the split schedule on sampled rows."""
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


def run_heads(dq, dk, dv, B, Hq, Hkv, N, D, scale, Sh, Wh, L, split=False):
    import torch
    o = torch.full_like(dq, float("nan"))
    ws, n = None, 0
    if split:
        n = tm.tm_attn_workspace_size(B, Hq, Hkv, N, D, False, int(max(Sh)), int(max(Wh)), L)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    tm.tm_triangle_attn_fwd_heads(dq, dk, dv, o, B, Hq, Hkv, N, D, scale, Sh, Wh, L, ws, n)
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    return o


CASES = [  # B, Hq, Hkv, N, D, L, seed
    (1, 4, 2, 1000, 128, 37, 1),
    (2, 6, 2, 777, 64, 0, 2),
    (1, 7, 1, 1500, 128, 200, 3),
    (1, 8, 8, 300, 128, 0, 4),
    (1, 2, 1, 4173, 128, 300, 5),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,D,L,seed", CASES)
def test_random_bands_match_oracle_all_rows(B, Hq, Hkv, N, D, L, seed):
    rng = np.random.default_rng(seed)
    Sh = rng.integers(0, 300, Hq).astype(np.int32)
    Wh = rng.integers(1, 600, Hq).astype(np.int32)
    Sh[0], Wh[0] = 0, 1                  # identity head
    if Hq > 2:
        Sh[1], Wh[1] = N + 5, 3          # sinks past N
        Wh[2] = N + 100                  # window past N (causal head)
    q, k, v = (rand_bits((B, N, h, D), seed * 10 + t, a)
               for h, t, a in ((Hq, 1, 2.0), (Hkv, 2, 2.0), (Hkv, 3, 1.0)))
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    want = oracle.attention_heads(q, k, v, B, Hq, Hkv, N, D, scale, Sh, Wh, L)
    for split in (False, True):
        o = run_heads(dq, dk, dv, B, Hq, Hkv, N, D, scale, Sh, Wh, L, split)
        assert_close(from_dev(o), want, f"heads {(B, Hq, Hkv, N, D, L)} split={split}")


def test_equal_bands_bitwise_equal_to_shared_band():
    import torch
    B, Hq, Hkv, N, D, S, W, L = 1, 8, 2, 3000, 128, 64, 700, 130
    dq = to_dev(rand_bits((B, N, Hq, D), 21, 2.0))
    dk, dv = to_dev(rand_bits((B, N, Hkv, D), 22, 2.0)), to_dev(rand_bits((B, N, Hkv, D), 23))
    o = run_heads(dq, dk, dv, B, Hq, Hkv, N, D, 0.1, [S] * Hq, [W] * Hq, L)
    ref = torch.empty_like(dq)
    tm.tm_triangle_attn_fwd(dq, dk, dv, ref, B, Hq, Hkv, N, D, 0.1, S, W, L)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), ref.view(torch.int16))


def test_llama_32k_seeded_bands_all_rows():
    wl = I.WORKLOADS["llama3-8b-32k"]
    q, k, v = I.make_qkv(wl)
    Sh, Wh = I.head_bands(wl.Hq, 0)
    o = run_heads(to_dev(q), to_dev(k), to_dev(v), wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                  Sh, Wh, wl.L)
    want = oracle.attention_heads(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, Sh, Wh,
                                  wl.L)
    assert_close(from_dev(o), want, "llama 32K per-head bands (all rows)")


def test_tp8_shard_128k_bands_with_split_sampled_rows():
    import torch
    wl = I.WORKLOADS["llama3-8b-128k-tp8"]
    q, k, v = I.make_qkv(wl, 1)
    Sh, Wh = I.head_bands(wl.Hq, 1)
    o = run_heads(to_dev(q), to_dev(k), to_dev(v), wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                  Sh, Wh, wl.L, split=True)
    rows = sample_rows(wl.N, wl.L, 12, 32, 96)
    want = oracle.attention_heads(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, Sh, Wh,
                                  wl.L, rows=rows)
    assert_close(from_dev(o[:, torch.tensor(rows, device="cuda")]), want, "tp8 128K bands")


def test_llama_128k_bench_bands_sampled_rows():
    """The bench's per-head leg: all 32 q heads of the 128K Llama-3-8B shape with
    the seeded bands (windows 512..4096, sinks {0, 64}), sampled rows."""
    import torch
    wl = I.WORKLOADS["llama3-8b-128k"]
    q, k, v = I.make_qkv(wl, wl.tri_start)
    Sh, Wh = I.head_bands(wl.Hq, 0)
    o = run_heads(to_dev(q), to_dev(k), to_dev(v), wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                  Sh, Wh, wl.L)
    rows = sample_rows(wl.N, wl.L, 14, 32, 64, n_last=32)
    want = oracle.attention_heads(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, Sh, Wh,
                                  wl.L, rows=rows)
    assert_close(from_dev(o[:, torch.tensor(rows, device="cuda")]), want, "llama 128K bands")
