"""Pins of the oracle's block-sparse attention (CPU only).

The routine is pinned to things other than itself: a block index that lists
every causal block reduces it to the (separately pinned) causal oracle exactly;
torch's float64 scaled_dot_product_attention under a block mask built here
from the index with numpy; the closed form for q = 0 (the mean of v over the
kept keys); zeros for rows that keep nothing; and the synthetic index recipe's
structure (sorted, causal, with its local band, sinks, verticals and slashes).
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_prefill_trianglemix_b200 import inputs as I


def rand_bits(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return I.f32_to_bf16_bits((g.standard_normal(shape) * scale).astype(np.float32))


def mask_from_index(B, Hkv, N, offsets, indices, BM=128, BS=128):
    """[B, Hkv, N, N] boolean mask, written from the definition with numpy."""
    nqb = (N + BM - 1) // BM
    nkb = (N + BS - 1) // BS
    m = np.zeros((B, Hkv, N, N), bool)
    causal = np.tril(np.ones((N, N), bool))
    for b in range(B):
        for g in range(Hkv):
            for qb in range(nqb):
                r = (b * Hkv + g) * nqb + qb
                cols = np.zeros(N, bool)
                for kb in indices[offsets[r]:offsets[r + 1]]:
                    if 0 <= kb < nkb:
                        cols[kb * BS:(kb + 1) * BS] = True
                rows = slice(qb * BM, min(N, (qb + 1) * BM))
                m[b, g, rows] = cols[None, :] & causal[rows]
    return m


def random_index(B, Hkv, N, seed, density, BM=128, extra_bad=False):
    rng = np.random.default_rng(seed)
    nqb = (N + BM - 1) // BM
    lists = []
    for _ in range(B * Hkv):
        for qb in range(nqb):
            kb = np.flatnonzero(rng.random(qb + 1) < density).tolist()
            if extra_bad and rng.random() < 0.3:
                kb += [qb + 1 + int(rng.integers(0, 3)), -1 - int(rng.integers(0, 3))]
            lists.append(sorted(set(kb)))
    off = np.zeros(len(lists) + 1, np.int32)
    off[1:] = np.cumsum([len(x) for x in lists])
    idx = np.array([c for x in lists for c in x], np.int32)
    return off, idx


def test_full_causal_index_is_causal_attention_exactly():
    B, Hq, Hkv, N, D = 2, 4, 2, 300, 32
    q, k, v = rand_bits((B, N, Hq, D), 1), rand_bits((B, N, Hkv, D), 2), rand_bits((B, N, Hkv, D), 3)
    off, idx = I.full_causal_index(B, Hkv, N)
    got = oracle.block_sparse_attention(q, k, v, B, Hq, Hkv, N, D, 0.2, off, idx)
    want = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, True)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("N,density,bad", [(300, 0.5, False), (257, 0.3, True), (128, 1.0, False)])
def test_matches_library_attention_under_a_block_mask(N, density, bad):
    B, Hq, Hkv, D = 2, 6, 2, 16
    q, k, v = (rand_bits((B, N, h, D), s, 2.0) for h, s in ((Hq, 4), (Hkv, 5), (Hkv, 6)))
    off, idx = random_index(B, Hkv, N, 7, density, extra_bad=bad)
    got = oracle.block_sparse_attention(q, k, v, B, Hq, Hkv, N, D, 0.3, off, idx)
    m = mask_from_index(B, Hkv, N, off, idx)
    G = Hq // Hkv
    mq = torch.from_numpy(np.repeat(m, G, axis=1))                      # [B, Hq, N, N]
    tq, tk, tv = (torch.from_numpy(I.bf16_bits_to_f32(x).astype(np.float64)).transpose(1, 2)
                  for x in (q, k, v))
    tk, tv = tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1)
    empty = ~mq.any(-1)                                                  # rows that keep nothing
    safe = mq | empty[..., None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=safe, scale=0.3)
    ref = ref.masked_fill(empty[..., None], 0.0).transpose(1, 2).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    if density < 1.0:
        assert empty.any()  # the case covers rows with an empty kept set


def test_zero_query_gives_the_mean_of_v_over_kept_keys():
    B, Hq, Hkv, N, D = 1, 4, 2, 400, 8
    q = np.zeros((B, N, Hq, D), np.uint16)
    k, v = rand_bits((B, N, Hkv, D), 8), rand_bits((B, N, Hkv, D), 9)
    off, idx = I.make_block_index(B, Hkv, N, 3, I.BlockIndexRecipe(local=1, sink=1, vertical=1,
                                                                   slash=1))
    got = oracle.block_sparse_attention(q, k, v, B, Hq, Hkv, N, D, 1.0, off, idx)
    m = mask_from_index(B, Hkv, N, off, idx)
    vf = I.bf16_bits_to_f32(v).astype(np.float64)
    for g in range(Hkv):
        want = (m[0, g].astype(np.float64) @ vf[0, :, g]) / m[0, g].sum(1, keepdims=True)
        for hq in range(g * 2, g * 2 + 2):
            np.testing.assert_allclose(got[0, :, hq], want, rtol=0, atol=1e-12)


def test_empty_lists_give_zero_rows():
    B, Hq, Hkv, N, D = 1, 2, 1, 256, 16
    q, k, v = rand_bits((B, N, Hq, D), 10), rand_bits((B, N, Hkv, D), 11), rand_bits((B, N, Hkv, D), 12)
    off = np.array([0, 0, 1], np.int32)     # q-block 0: nothing; q-block 1: block 0
    idx = np.array([0], np.int32)
    got = oracle.block_sparse_attention(q, k, v, B, Hq, Hkv, N, D, 0.1, off, idx)
    assert (got[0, :128] == 0).all()
    assert np.abs(got[0, 128:]).sum() > 0


def test_malformed_offsets_are_rejected():
    B, Hq, Hkv, N, D = 1, 2, 1, 256, 16
    q, k, v = rand_bits((B, N, Hq, D), 1), rand_bits((B, N, Hkv, D), 2), rand_bits((B, N, Hkv, D), 3)
    for off in ([0, 2, 1], [0, 1, 3], [-1, 0, 1]):
        with pytest.raises(ValueError):
            oracle.block_sparse_attention(q, k, v, B, Hq, Hkv, N, D, 0.1,
                                          np.array(off, np.int32), np.array([0, 1], np.int32))


@pytest.mark.parametrize("N", [1000, 32768])
def test_synthetic_index_structure(N):
    rec = I.BlockIndexRecipe()
    off, idx = I.make_block_index(2, 3, N, 5, rec)
    nqb = (N + 127) // 128
    assert off.size == 2 * 3 * nqb + 1 and off[0] == 0 and (np.diff(off) >= 1).all()
    for r in range(2 * 3 * nqb):
        qb = r % nqb
        lst = idx[off[r]:off[r + 1]]
        assert (np.diff(lst) > 0).all() and lst[0] >= 0 and lst[-1] == qb
        assert set(range(max(0, qb - rec.local + 1), qb + 1)) <= set(lst.tolist())
        assert 0 in lst
    # the same seed gives the same index; another seed another one
    off2, idx2 = I.make_block_index(2, 3, N, 5, rec)
    np.testing.assert_array_equal(idx, idx2)
    assert not np.array_equal(I.make_block_index(2, 3, N, 6, rec)[1][:200], idx[:200]) or N < 2000
