"""Parity of block-sparse attention (tm_block_sparse_attn_fwd, through the C
ABI) with the fp64 oracle: random indices with empty lists, entries above the
diagonal and out-of-range entries (fully masked tiles), odd group sizes,
ragged N, D = 64; the full causal index against the causal kernel bit for bit;
the synthetic vertical/slash index at 32K on every row and at 128K on sampled
rows; and the layer schedule that pairs it with the triangle layers.
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


def random_index(B, Hkv, N, seed, density, extra_bad=False):
    rng = np.random.default_rng(seed)
    nqb = (N + 127) // 128
    lists = []
    for _ in range(B * Hkv):
        for qb in range(nqb):
            kb = np.flatnonzero(rng.random(qb + 1) < density).tolist()
            if extra_bad and rng.random() < 0.3:
                kb += [qb + 1 + int(rng.integers(0, 3)), -1 - int(rng.integers(0, 3)), 10 ** 6]
            lists.append(sorted(set(kb)))
    off = np.zeros(len(lists) + 1, np.int32)
    off[1:] = np.cumsum([len(x) for x in lists])
    return off, np.array([c for x in lists for c in x], np.int32)


def dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()


def run_sparse(dq, dk, dv, B, Hq, Hkv, N, D, scale, off, idx):
    import torch
    o = torch.full_like(dq, float("nan"))
    doff, didx = dev_i32(off), dev_i32(idx if len(idx) else np.zeros(1, np.int32))
    tm.tm_block_sparse_attn_fwd(dq, dk, dv, o, B, Hq, Hkv, N, D, scale, doff, didx, len(idx))
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    return o


CASES = [  # B, Hq, Hkv, N, D, density, bad
    (1, 2, 1, 1000, 128, 0.5, False),
    (2, 6, 2, 777, 64, 0.3, True),
    (1, 7, 1, 1500, 128, 0.2, True),
    (1, 8, 2, 2049, 128, 0.05, False),
    (3, 4, 4, 300, 64, 1.0, False),
    (1, 2, 2, 1, 128, 1.0, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,D,density,bad", CASES)
def test_random_index_matches_oracle_all_rows(B, Hq, Hkv, N, D, density, bad):
    q = rand_bits((B, N, Hq, D), 51, 2.0)
    k = rand_bits((B, N, Hkv, D), 52, 2.0)
    v = rand_bits((B, N, Hkv, D), 53)
    off, idx = random_index(B, Hkv, N, 54, density, bad)
    scale = 1.0 / math.sqrt(D)
    o = run_sparse(to_dev(q), to_dev(k), to_dev(v), B, Hq, Hkv, N, D, scale, off, idx)
    want = oracle.block_sparse_attention(q, k, v, B, Hq, Hkv, N, D, scale, off, idx)
    got = from_dev(o)
    assert_close(got, want, f"block sparse {(B, Hq, Hkv, N, D, density, bad)}")
    empty = np.diff(off) == 0
    if empty.any():  # rows of empty lists are written as zeros
        nqb = (N + 127) // 128
        for r in np.flatnonzero(empty)[:8]:
            b, g, qb = r // (Hkv * nqb), (r // nqb) % Hkv, r % nqb
            G = Hq // Hkv
            assert (got[b, qb * 128:(qb + 1) * 128, g * G:(g + 1) * G] == 0).all()


def test_empty_index_writes_zeros():
    import torch
    B, Hq, Hkv, N, D = 1, 4, 2, 600, 128
    dq = to_dev(rand_bits((B, N, Hq, D), 1))
    dk, dv = to_dev(rand_bits((B, N, Hkv, D), 2)), to_dev(rand_bits((B, N, Hkv, D), 3))
    off = np.zeros(B * Hkv * 5 + 1, np.int32)
    o = run_sparse(dq, dk, dv, B, Hq, Hkv, N, D, 0.1, off, np.zeros(0, np.int32))
    assert torch.equal(o, torch.zeros_like(o))


def test_full_causal_index_equals_causal_kernel_bitwise():
    import torch
    B, Hq, Hkv, N, D = 1, 8, 2, 3000, 128
    dq = to_dev(rand_bits((B, N, Hq, D), 61, 2.0))
    dk, dv = to_dev(rand_bits((B, N, Hkv, D), 62, 2.0)), to_dev(rand_bits((B, N, Hkv, D), 63))
    off, idx = I.full_causal_index(B, Hkv, N)
    o = run_sparse(dq, dk, dv, B, Hq, Hkv, N, D, 0.09, off, idx)
    c = torch.empty_like(dq)
    tm.tm_causal_attn_fwd(dq, dk, dv, c, B, Hq, Hkv, N, D, 0.09)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), c.view(torch.int16))


def test_synthetic_index_32k_all_rows():
    wl = I.WORKLOADS["llama3-8b-32k"]
    q, k, v = I.make_qkv(wl)
    off, idx = I.make_block_index(wl.B, wl.Hkv, wl.N, 0)
    o = run_sparse(to_dev(q), to_dev(k), to_dev(v), wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                   off, idx)
    want = oracle.block_sparse_attention(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, off,
                                         idx)
    assert_close(from_dev(o), want, "block sparse 32K synthetic index (all rows)")


def test_synthetic_index_128k_sampled_rows_and_layer_schedule():
    import torch
    wl = I.WORKLOADS["llama3-8b-128k"]
    q, k, v = I.make_qkv(wl)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    off, idx = I.make_block_index(wl.B, wl.Hkv, wl.N, 0)
    doff, didx = dev_i32(off), dev_i32(idx)
    rows = sample_rows(wl.N, wl.L, 11, 32, 96, n_last=32)
    ridx = torch.tensor(rows, device="cuda")
    for layer in (0, 1):  # tri_start = 1: layer 0 block-sparse, layer 1 triangle
        o = torch.empty_like(dq)
        tm.tm_trianglemix_sparse_attn_fwd(dq, dk, dv, o, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D,
                                          wl.scale, wl.S, wl.W, wl.L, layer, 1, doff, didx,
                                          len(idx))
        torch.cuda.synchronize()
        assert tm.tm_get_device_status() == tm.TM_OK
        if layer == 0:
            want = oracle.block_sparse_attention(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D,
                                                 wl.scale, off, idx, rows=rows)
        else:
            want = oracle.attention(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, False,
                                    wl.S, wl.W, wl.L, rows=rows)
        assert_close(from_dev(o[:, ridx]), want, f"128K layer {layer}")
