"""Pins for the fp64 CPU oracle: each check ties it to something other than itself.

* closed-form kept count per row (the TriangleMix pattern written as a count);
* a hand-worked mask and a hand-worked attention example (tests/golden/);
* a library routine: torch's scaled_dot_product_attention in float64;
* invariants of the pattern (L=N and S+W>=N give causal, last-L rows are
  causal rows, rows sum to 1) and special cases with closed forms
  (identity window, q = 0 gives a mean over the kept set, v = 1 gives 1).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_prefill_trianglemix_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def closed_form_count(i, N, S, W, L):
    """|K_i| of the triangle pattern, written as a count (not as a mask)."""
    S, L, W = min(max(S, 0), N), min(max(L, 0), N), max(W, 1)
    if i >= N - L:
        return i + 1
    return min(i + 1, W) + max(0, min(S, i + 1 - W))


def kept_intervals(i, N, S, W, L, causal):
    """K_i as half-open intervals (used only to build a library mask)."""
    if causal or i >= N - min(L, N):
        return [(0, i + 1)]
    return [(0, min(S, i + 1)), (max(0, i - W + 1), i + 1)]


def interval_mask(N, S, W, L, causal):
    m = np.zeros((N, N), bool)
    for i in range(N):
        for a, b in kept_intervals(i, N, S, W, L, causal):
            m[i, a:b] = True
    return m


def rand_bf16(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return I.f32_to_bf16_bits((g.standard_normal(shape) * scale).astype(np.float32))


def to_f64(a):
    return I.bf16_bits_to_f32(a).astype(np.float64)


# ----------------------------------------------------------------------------- mask


GRID = [(N, S, W, L)
        for N in (1, 2, 3, 7, 64, 127, 128, 129, 300)
        for S in (0, 1, 3, 16, 1000)
        for W in (1, 2, 5, 64, 1000)
        for L in (0, 1, 5, 1000)]


@pytest.mark.parametrize("N,S,W,L", GRID)
def test_kept_count_matches_closed_form(N, S, W, L):
    for i in range(N):
        row = oracle.mask_row(N, False, S, W, L, i)
        assert int(row.sum()) == closed_form_count(i, N, S, W, L), (i, N, S, W, L)
        assert row[i], "every row keeps its diagonal (W >= 1)"
        assert not row[i + 1:].any(), "no key after the query"


def test_mask_matches_hand_worked_golden():
    lines = [l.strip() for l in open(os.path.join(GOLDEN, "mask_n10_s1_w3_l2.txt"))
             if l.strip() and not l.startswith("#")]
    want = np.array([[c == "1" for c in l] for l in lines])
    got = np.stack([oracle.mask_row(10, False, 1, 3, 2, i) for i in range(10)])
    np.testing.assert_array_equal(got, want)


def test_causal_mask_is_lower_triangle():
    N = 37
    got = np.stack([oracle.mask_row(N, True, 0, 1, 0, i) for i in range(N)])
    np.testing.assert_array_equal(got, np.tril(np.ones((N, N), bool)))


@pytest.mark.parametrize("N,S,W,L", [(512, 16, 64, 64), (1000, 64, 100, 10), (4097, 7, 300, 0),
                                     (131072, 64, 2048, 256)])
def test_kept_pairs_total(N, S, W, L):
    want = sum(closed_form_count(i, N, S, W, L) for i in range(N))
    assert oracle.kept_pairs(N, False, S, W, L) == want
    assert oracle.kept_pairs(N, True, 0, 1, 0) == N * (N + 1) // 2


def test_bad_pattern_rejected():
    with pytest.raises(ValueError):
        oracle.mask_row(10, False, 1, 0, 2, 0)      # W < 1
    with pytest.raises(ValueError):
        oracle.mask_row(10, False, -1, 3, 2, 0)     # S < 0
    assert oracle.kept_count_row(0, False, 0, 1, 0, 0) == -1


# ----------------------------------------------------------------------------- tiles

TILE_CASES = [(N, S, W, L, BM, BN)
              for (N, S, W, L) in [(1, 0, 1, 0), (100, 3, 10, 5), (128, 16, 64, 64),
                                   (129, 16, 64, 0), (500, 0, 1, 0), (512, 16, 64, 64),
                                   (1000, 64, 200, 130), (2049, 64, 300, 1), (777, 130, 129, 0)]
              for (BM, BN) in [(128, 128), (64, 128), (128, 64)]]


@pytest.mark.parametrize("N,S,W,L,BM,BN", TILE_CASES)
def test_tile_list_two_methods_and_mask(N, S, W, L, BM, BN):
    for causal in (False, True):
        a = oracle.tile_list_bruteforce(N, causal, S, W, L, BM, BN)
        b = oracle.tile_list_rows(N, causal, S, W, L, BM, BN)
        np.testing.assert_array_equal(a, b)
        # pin the records against a mask built from intervals, block by block
        m = interval_mask(N, S, W, L, causal)
        want = []
        for qb in range((N + BM - 1) // BM):
            for kb in range((N + BN - 1) // BN):
                blk = m[qb * BM:(qb + 1) * BM, kb * BN:(kb + 1) * BN]
                if blk.any():
                    want.append((qb, kb, int(blk.all())))
        np.testing.assert_array_equal(a, np.array(want, np.int32).reshape(-1, 3))


def test_tile_counts_large_n_consistent():
    # kept-pair total recovered from the row-interval tile list at 128K must be
    # at least the closed-form pair total, and every tile list is sorted
    N, S, W, L = 131072, 64, 2048, 256
    t = oracle.tile_list_rows(N, False, S, W, L)
    key = t[:, 0].astype(np.int64) * 10**6 + t[:, 1]
    assert np.all(np.diff(key) > 0)
    assert (t[:, 1] <= t[:, 0]).all()
    # per q-block: last-L blocks hold every causal tile
    nqb = N // 128
    per_qb = np.bincount(t[:, 0], minlength=nqb)
    assert per_qb[-1] == nqb and per_qb[-2] == nqb - 1
    # the middle blocks hold one sink tile + a band of ceil(W/BN)+1 tiles
    assert per_qb[500] == 1 + W // 128 + 1


# ----------------------------------------------------------------------------- attention


def sdpa_reference(q, k, v, Hq, Hkv, scale, mask):
    """torch scaled_dot_product_attention in float64 with kv heads repeated per group."""
    G = Hq // Hkv
    qt = torch.from_numpy(to_f64(q)).permute(0, 2, 1, 3)
    kt = torch.from_numpy(to_f64(k)).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(to_f64(v)).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=scale)
    return out.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("B,Hq,Hkv,N,D,S,W,L", [(2, 4, 2, 67, 16, 3, 9, 5), (1, 6, 3, 130, 32, 0, 17, 0),
                                                (1, 2, 2, 64, 8, 64, 1, 0), (1, 8, 1, 50, 64, 5, 5, 50)])
def test_attention_matches_library_routine(B, Hq, Hkv, N, D, S, W, L):
    q = rand_bf16((B, N, Hq, D), 1, 2.0)
    k = rand_bf16((B, N, Hkv, D), 2, 2.0)
    v = rand_bf16((B, N, Hkv, D), 3)
    scale = 1.0 / math.sqrt(D)
    for causal in (False, True):
        got = oracle.attention(q, k, v, B, Hq, Hkv, N, D, scale, causal, S, W, L)
        want = sdpa_reference(q, k, v, Hq, Hkv, scale, interval_mask(N, S, W, L, causal))
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_gqa_map_is_contiguous_groups():
    # head hq must read kv head hq // (Hq/Hkv): compare against explicit copies
    B, Hq, Hkv, N, D = 1, 6, 2, 40, 16
    q = rand_bf16((B, N, Hq, D), 4)
    k = rand_bf16((B, N, Hkv, D), 5)
    v = rand_bf16((B, N, Hkv, D), 6)
    kk = np.ascontiguousarray(np.repeat(k, 3, axis=2))
    vv = np.ascontiguousarray(np.repeat(v, 3, axis=2))
    a = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.25, False, 2, 7, 3)
    b = oracle.attention(q, kk, vv, B, Hq, Hq, N, D, 0.25, False, 2, 7, 3)
    np.testing.assert_array_equal(a, b)


def test_hand_worked_attention_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "hand_attention_n4.txt"))
            if l.strip() and not l.startswith("#")]
    N, D = 4, 2
    f = np.zeros((1, N, 1, D), np.float32)
    q, k, v = f.copy(), f.copy(), f.copy()
    q[0, :, 0, 0] = 1.0
    k[0, :, 0, 0] = np.arange(N)
    v[0, :, 0, 0] = np.arange(N)
    v[0, :, 0, 1] = 1.0
    q, k, v = (I.f32_to_bf16_bits(x) for x in (q, k, v))
    got = oracle.attention(q, k, v, 1, 1, 1, N, D, 1.0, False, 1, 1, 1)
    for row, kept, expr in rows:
        i = int(row)
        want = eval(expr, {"e": math.e})
        assert got[0, i, 0, 0] == pytest.approx(want, abs=1e-14)
        assert got[0, i, 0, 1] == pytest.approx(1.0, abs=1e-15)
        assert sorted(np.flatnonzero(oracle.mask_row(N, False, 1, 1, 1, i))) == \
            [int(x) for x in kept.split(",")]


@pytest.fixture(scope="module")
def mid_case():
    B, Hq, Hkv, N, D = 1, 4, 2, 300, 32
    q = rand_bf16((B, N, Hq, D), 7, 1.5)
    k = rand_bf16((B, N, Hkv, D), 8, 1.5)
    v = rand_bf16((B, N, Hkv, D), 9)
    return B, Hq, Hkv, N, D, q, k, v


def test_invariant_large_l_or_window_equals_causal(mid_case):
    B, Hq, Hkv, N, D, q, k, v = mid_case
    causal = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, True)
    for S, W, L in [(4, 10, N), (4, 10, N + 7), (100, 200, 0), (0, N, 0), (N, 1, 0)]:
        tri = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, False, S, W, L)
        np.testing.assert_array_equal(tri, causal)


def test_invariant_last_l_rows_are_causal_rows(mid_case):
    B, Hq, Hkv, N, D, q, k, v = mid_case
    S, W, L = 3, 20, 37
    causal = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, True)
    tri = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, False, S, W, L)
    np.testing.assert_array_equal(tri[:, N - L:], causal[:, N - L:])
    assert np.abs(tri[:, : N - L] - causal[:, : N - L]).max() > 1e-3  # the middle is really skipped


def test_invariant_rows_sum_to_one(mid_case):
    B, Hq, Hkv, N, D, q, k, v = mid_case
    _, rs = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, False, 3, 20, 37, with_rowsum=True)
    np.testing.assert_allclose(rs, 1.0, rtol=0, atol=1e-12)


def test_special_identity_window(mid_case):
    B, Hq, Hkv, N, D, q, k, v = mid_case
    out = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, False, 0, 1, 0)
    G = Hq // Hkv
    vv = np.repeat(to_f64(v), G, axis=2)
    np.testing.assert_array_equal(out, vv)


def test_special_zero_query_gives_mean_over_kept_set(mid_case):
    B, Hq, Hkv, N, D, _, k, v = mid_case
    S, W, L = 5, 31, 17
    q0 = np.zeros((B, N, Hq, D), np.uint16)
    out = oracle.attention(q0, k, v, B, Hq, Hkv, N, D, 0.2, False, S, W, L)
    vf = to_f64(v)
    pre = np.concatenate([np.zeros((B, 1, Hkv, D)), np.cumsum(vf, axis=1)], axis=1)
    G = Hq // Hkv
    for i in range(N):
        cnt = closed_form_count(i, N, S, W, L)
        if i >= N - L:
            tot = pre[:, i + 1]
        else:
            se, wb = min(S, i + 1), max(0, i - W + 1)
            tot = pre[:, se] + pre[:, i + 1] - pre[:, max(wb, se)]
        want = np.repeat(tot / cnt, G, axis=1)
        np.testing.assert_allclose(out[:, i], want, rtol=0, atol=1e-12)


def test_special_unit_values_give_unit_output(mid_case):
    B, Hq, Hkv, N, D, q, k, _ = mid_case
    ones = np.full((B, N, Hkv, D), 0x3F80, np.uint16)  # bf16 1.0
    out = oracle.attention(q, k, ones, B, Hq, Hkv, N, D, 0.2, False, 3, 20, 37)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-13)


def test_row_subset_equals_full_rows(mid_case):
    B, Hq, Hkv, N, D, q, k, v = mid_case
    full = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, False, 3, 20, 37)
    rows = [0, 5, 150, 262, 263, 299]
    sub = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, False, 3, 20, 37, rows=rows)
    np.testing.assert_array_equal(sub, full[:, rows])
