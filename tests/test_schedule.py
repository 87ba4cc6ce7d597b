"""The persistent work split (host export of the same code the launch uses):
every (q-block, q-head pair) item is processed exactly once, the longest
items come first in each CTA, and the per-CTA cost is balanced. With a
workspace the heavy items are cut into pieces whose tile ranges cover each
item's tile list exactly once."""
import numpy as np
import pytest

import long_context_prefill_trianglemix_b200 as tm
from long_context_prefill_trianglemix_b200 import build
from long_context_prefill_trianglemix_b200 import inputs as I


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build_lib()
    yield


CASES = [(wl.B, wl.Hq, wl.Hkv, wl.N, causal, wl.S, W, wl.L)
         for wl in I.WORKLOADS.values() for causal in (False, True)
         for W in ((wl.W,) + tuple(wl.windows))]
CASES += [(1, 2, 1, 1, False, 0, 1, 0), (3, 4, 1, 383, False, 1, 1, 1), (1, 14, 2, 777, False, 5, 200, 100),
          (2, 6, 2, 129, True, 0, 1, 0), (8, 32, 8, 4096, False, 64, 1024, 128)]


def rec_tiles(qb, h0, nv):
    """The (q-block, q head) Q tiles of a schedule record: a pair of heads of one
    q-block, or (bit 8 of the count) consecutive q-blocks of one head."""
    qpair, nq = nv >> 8, nv & 255
    return [(qb + k, h0) for k in range(nq)] if qpair else [(qb, h0 + k) for k in range(nq)]


def qblock_pairs(Hq, Hkv, causal):
    """Causal launches of odd groups pair two q-blocks of one head per item."""
    G = Hq // Hkv
    return causal and G % 2 == 1 and G > 1


def n_items_whole(B, Hq, Hkv, N, causal):
    G, nqb = Hq // Hkv, (N + 127) // 128
    if qblock_pairs(Hq, Hkv, causal):
        return (nqb + 1) // 2 * B * Hq
    return nqb * B * Hkv * ((G + 1) // 2)


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,S,W,L", CASES)
def test_every_item_exactly_once(B, Hq, Hkv, N, causal, S, W, L):
    rec = tm.tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, 148)
    nqb = (N + 127) // 128
    n_items = n_items_whole(B, Hq, Hkv, N, causal)
    assert len(rec) == n_items
    assert sorted(rec[:, 1].tolist()) == list(range(n_items))
    assert ((rec[:, 4] >> 8) == int(qblock_pairs(Hq, Hkv, causal))).all()
    # every (batch, q head, q-block) tile appears once
    tiles = set()
    for c, item, qb, h0, nv, t0, t1 in rec:
        assert t0 == 0
        for t in rec_tiles(qb, h0, nv):
            assert t not in tiles
            tiles.add(t)
    assert len(tiles) == nqb * B * Hq
    # the grid never exceeds the SM count or the item count
    assert rec[:, 0].max() < min(148, n_items)


@pytest.mark.parametrize("N,S,W,L", [(32768, 64, 1024, 128), (131072, 64, 2048, 256),
                                     (131072, 64, 512, 256), (65536, 64, 1024, 128)])
def test_triangle_split_is_balanced(N, S, W, L):
    rec = tm.tm_debug_schedule(1, 32, 8, N, False, S, W, L, 148)
    tiles = tm.tm_tile_list(N, False, S, W, L)
    per_qb = np.bincount(tiles[:, 0], minlength=(N + 127) // 128)
    cost = np.zeros(148)
    for c, item, qb, h0, nv, t0, t1 in rec:
        cost[c] += (per_qb[qb] + 3) * nv
    # within one normal item of the mean
    normal = (per_qb[:-3].max() + 3) * 2
    assert cost.max() - cost.mean() <= 1.5 * normal, (cost.max(), cost.mean(), normal)
    # a CTA's big items (the last-L q-blocks) come before its other items
    heavy = set(np.flatnonzero(per_qb >= 4 * normal).tolist())
    assert heavy, "the last-L q-blocks are big items"
    for c in range(148):
        qbs = rec[rec[:, 0] == c][:, 2].tolist()
        flags = [q in heavy for q in qbs]
        assert flags == sorted(flags, reverse=True), (c, qbs[:6])


@pytest.mark.parametrize("N,causal,W,L", [(32768, False, 1024, 128), (131072, False, 2048, 256),
                                          (131072, True, 1, 0), (32768, True, 1, 0)])
def test_concurrent_items_share_kv_tiles(N, causal, W, L):
    # Items are dealt in strided rounds: the 148 consecutive items of a round are
    # what the CTAs run at about the same time. In a triangle launch a round spans
    # a narrow band of q-blocks of every kv head. In a causal launch (chunked
    # group order) a round holds the q-blocks of one chunk of a single kv head,
    # so the K/V it reads is one head's (64 MB at 128K) and stays in L2; the
    # shortest q-blocks after the last full chunk run like the triangle's.
    rec = tm.tm_debug_schedule(1, 32, 8, N, causal, 64, W, L, 148)
    order = np.argsort(rec[:, 1])
    items, qbs, kvh = rec[order, 1], rec[order, 2], rec[order, 3] // 4
    for r0 in range(0, len(items) - 148, 148):
        band = qbs[r0:r0 + 148]
        full_chunks = (N // 128) // 74 * 74 * 16   # items of the full chunks
        if causal and r0 + 148 <= full_chunks:
            assert len(set(kvh[r0:r0 + 148].tolist())) == 1, r0
            assert band.max() - band.min() < 74, (r0, band.min(), band.max())
        else:
            assert band.max() - band.min() <= 10, (r0, band.min(), band.max())
    # each CTA's items increase; odd rounds run in reverse CTA order, so a CTA's
    # strides alternate between 2g - 1 - 2c and 2c + 1 (they sum to two rounds)
    for c in range(148):
        it = rec[rec[:, 0] == c][:, 1]
        d = np.diff(it)
        assert (d > 0).all(), (c, it[:6])
        main = d[-6:][d[-6:] < 2 * 148]   # normal items (big pieces have their own ids)
        assert set(main.tolist()) <= {2 * 148 - 1 - 2 * c, 2 * c + 1}, (c, main[:6])


@pytest.mark.parametrize("N,Hq,Hkv", [(131072, 32, 8), (65536, 32, 8), (32768, 32, 8),
                                      (131072, 4, 1), (65536, 8, 2), (131072, 28, 4),
                                      (65536, 28, 4), (131072, 7, 1)])
def test_causal_chunked_group_order_is_balanced(N, Hq, Hkv):
    rec = tm.tm_debug_schedule(1, Hq, Hkv, N, True, 0, 1, 0, 148)
    cost = np.zeros(148)
    for c, item, qb, h0, nv, t0, t1 in rec:
        last = max(q for q, _ in rec_tiles(qb, h0, nv))
        cost[c] += (last + 1 + 3) * (nv & 255)
    assert cost.max() / cost.mean() <= 1.01, cost.max() / cost.mean()


@pytest.mark.parametrize("N,Hq,Hkv", [(131072, 28, 4), (65536, 28, 4), (131072, 7, 1)])
def test_odd_group_causal_rounds_read_one_kv_head(N, Hq, Hkv):
    # Groups of 7 heads: items pair two q-blocks of one head, 7 per kv head and
    # slot; a turn of 21 slots is 147 items, and the grid is 147 CTAs, so every
    # round of the full chunks reads one kv head's K/V (64 MB at 128K, in L2)
    G = Hq // Hkv
    rec = tm.tm_debug_schedule(1, Hq, Hkv, N, True, 0, 1, 0, 148)
    grid = rec[:, 0].max() + 1
    assert grid == 148 // G * G
    order = np.argsort(rec[:, 1])
    kvh, qbs = rec[order, 3] // G, rec[order, 2]
    nslots = (N // 128 + 1) // 2
    full = nslots // (grid // G) * (grid // G) * G * Hkv   # items of the full chunks
    for r0 in range(0, full, grid):
        assert len(set(kvh[r0:r0 + grid].tolist())) == 1, r0
        assert qbs[r0:r0 + grid].max() - qbs[r0:r0 + grid].min() < 2 * (grid // G) + 1, r0


SPLIT_CASES = [(1, 4, 1, 131072, False, 64, 2048, 256), (1, 4, 1, 131072, False, 64, 512, 256),
               (1, 8, 2, 65536, False, 64, 1024, 128), (1, 32, 8, 131072, False, 64, 512, 256),
               (1, 4, 1, 131072, True, 0, 1, 0), (1, 2, 1, 32768, True, 0, 1, 0),
               (1, 4, 4, 512, False, 16, 64, 64), (2, 6, 2, 1000, False, 3, 100, 300),
               (1, 28, 4, 131072, False, 64, 1024, 128), (1, 7, 1, 65536, False, 64, 1024, 200),
               (2, 3, 1, 3129, True, 0, 1, 0), (1, 5, 1, 20000, True, 0, 1, 0)]


def cta_costs(rec, per_qb, n_ctas=148, overhead=3, split_overhead=1):
    cost = np.zeros(n_ctas)
    for c, item, qb, h0, nv, t0, t1 in rec:
        n_union = max(per_qb[q] for q, _ in rec_tiles(qb, h0, nv))
        piece = (t1 - t0) + overhead + (split_overhead if t1 - t0 < n_union else 0)
        cost[c] += piece * (nv & 255)
    return cost


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,S,W,L", SPLIT_CASES)
def test_split_pieces_cover_each_item_once(B, Hq, Hkv, N, causal, S, W, L):
    rec = tm.tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, 148, split=True)
    tiles = tm.tm_tile_list(N, causal, S, W, L)
    per_qb = np.bincount(tiles[:, 0], minlength=(N + 127) // 128)
    seen, end = {}, {}
    for c, item, qb, h0, nv, t0, t1 in rec:
        tiles = rec_tiles(qb, h0, nv)
        n_union = max(per_qb[q] for q, _ in tiles)   # the item's list covers its Q tiles' lists
        assert 0 <= t0 < t1 <= n_union
        for t in tiles:
            seen.setdefault(t, []).append((t0, t1))
            end[t] = n_union
    nqb = (N + 127) // 128
    assert len(seen) == nqb * B * Hq
    for (qb, h), ranges in seen.items():
        ranges.sort()
        assert ranges[0][0] == 0 and ranges[-1][1] == end[(qb, h)], (qb, h, ranges)
        for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
            assert a1 == b0, (qb, h, ranges)   # contiguous, no overlap
    # the item ids are a permutation
    assert sorted(rec[:, 1].tolist()) == list(range(len(rec)))
    # pieces of one heavy item run on different CTAs, all before normal work
    pieces = rec[(rec[:, 6] - rec[:, 5]) < per_qb[np.minimum(rec[:, 2] + (rec[:, 4] >> 8), nqb - 1)]]
    for key in {(int(q), int(h)) for _, _, q, h, _, _, _ in pieces}:
        ctas = pieces[(pieces[:, 2] == key[0]) & (pieces[:, 3] == key[1])][:, 0]
        assert len(set(ctas.tolist())) == len(ctas)


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,S,W,L", [c for c in SPLIT_CASES if c[3] >= 32768])
def test_split_balances_small_head_counts(B, Hq, Hkv, N, causal, S, W, L):
    tiles = tm.tm_tile_list(N, causal, S, W, L)
    per_qb = np.bincount(tiles[:, 0], minlength=(N + 127) // 128)
    whole = cta_costs(tm.tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, 148), per_qb)
    split = cta_costs(tm.tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, 148, split=True), per_qb)
    # never worse than the unsplit schedule, and within about a fifth of the mean
    assert split.max() <= whole.max() * 1.01
    assert split.max() <= 1.2 * split.mean() or split.max() <= whole.max() * 0.5 + split.mean(), (
        split.max(), split.mean(), whole.max())


def test_split_needed_only_when_an_item_exceeds_its_share():
    # Llama-3-8B at 128K with all 32 q heads: the last-L items fit in a CTA's share
    assert tm.tm_attn_workspace_size(1, 32, 8, 131072, 128, False, 64, 2048, 256, 148) == 0
    # a tensor-parallel shard (4 q heads, 1 kv head) has to cut them
    n = tm.tm_attn_workspace_size(1, 4, 1, 131072, 128, False, 64, 2048, 256, 148)
    assert n > 0
    rec = tm.tm_debug_schedule(1, 4, 1, 131072, False, 64, 2048, 256, 148, split=True)
    per_qb = np.bincount(tm.tm_tile_list(131072, False, 64, 2048, 256)[:, 0])
    n_pieces = int(((rec[:, 6] - rec[:, 5]) < per_qb[rec[:, 2]]).sum())
    ns = n_pieces // (2 * 2)          # 2 heavy q-blocks x 2 head pairs
    cnt_bytes = -(-2 * 2 * 8 * 4 // 256) * 256
    assert n == cnt_bytes + 2 * 2 * ns * 2 * (128 * 128 + 256) * 4
    # D = 64 records are half the size
    n64 = tm.tm_attn_workspace_size(1, 4, 1, 131072, 64, False, 64, 2048, 256, 148)
    assert n64 == cnt_bytes + 2 * 2 * ns * 2 * (128 * 64 + 256) * 4


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,W,L", [(1, 32, 8, 131072, False, 2048, 256),
                                                   (1, 32, 8, 32768, True, 1, 0),
                                                   (1, 28, 4, 131072, False, 1024, 128),
                                                   (2, 12, 4, 16384, False, 512, 64)])
def test_items_of_one_kv_head_and_q_block_are_adjacent(B, Hq, Hkv, N, causal, W, L):
    # The pairs of one kv head at one q-block read the same K/V tiles in the same
    # order; as consecutive items they go to neighbouring CTAs of the same round and
    # run in lockstep, so each tile comes from DRAM once for all of them.
    rec = tm.tm_debug_schedule(B, Hq, Hkv, N, causal, 64, W, L, 148)
    G = Hq // Hkv
    groups = {}
    for c, item, qb, h0, nv, t0, t1 in rec:
        groups.setdefault((qb, h0 // G), []).append(item)
    npairs = (G + 1) // 2
    for key, items in groups.items():
        assert len(items) == npairs
        assert max(items) - min(items) == npairs - 1, (key, sorted(items))


def union_tiles(N, causal, S, W, L, r0, r1):
    """Key blocks holding a kept key of any row in [r0, r1] (the union list of a
    q-block pair), from the pattern's per-row intervals: every causal key for
    causal rows and the last L rows, else the sinks [0, S) and the window
    [i - W + 1, i], whose ends grow with i."""
    if causal or r1 >= N - L:
        return r1 // 128 + 1
    blocks = set(range((min(S, r1 + 1) + 127) // 128))
    blocks.update(range(max(0, r0 - W + 1) // 128, r1 // 128 + 1))
    return len(blocks)


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,S,W,L", CASES[:12] + SPLIT_CASES[:4])
def test_pair_and_kv_rotation_keep_exact_coverage(B, Hq, Hkv, N, causal, S, W, L):
    # per-head band launches rotate the pair and kv-head digits per q-block and
    # (for non-causal patterns) pair two consecutive q-blocks of one head in an
    # item; every (q-block, head) must still be covered exactly once, and the
    # pieces of an item must cover its tile list (the union of its Q tiles')
    nqb = (N + 127) // 128
    for split in (False, True):
        rec = tm.tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, 148, split=split, mix_pairs=True)
        ranges = {}
        for c, item, qb, h0, nv, t0, t1 in rec:
            qpair, nq = nv >> 8, nv & 255
            assert qpair == (0 if causal else 1)
            tiles = [(qb + k, h0) for k in range(nq)] if qpair else [(qb, h0 + k) for k in range(nq)]
            ranges.setdefault(tuple(tiles), []).append((t0, t1))   # the pieces of one item
        seen = [t for tiles in ranges for t in tiles]
        assert len(seen) == len(set(seen)) == nqb * B * Hq
        for tiles, rg in ranges.items():
            rg.sort()
            qbs = sorted({t[0] for t in tiles})
            n_union = union_tiles(N, causal, S, W, L, qbs[0] * 128, min(N, (qbs[-1] + 1) * 128) - 1)
            assert rg[0][0] == 0 and rg[-1][1] == n_union, (tiles, rg, n_union)
            assert all(a1 == b0 for (_, a1), (b0, _) in zip(rg, rg[1:]))


@pytest.mark.parametrize("N,S,W,L", [(131072, 64, 4096, 256), (131072, 64, 4096, 128),
                                     (32768, 64, 4096, 128), (1000, 0, 300, 100)])
def test_qblock_pairs_waste_at_most_one_tile_per_q_tile(N, S, W, L):
    # a q-block pair's union list holds at most one tile more than each of its
    # two q-blocks' own lists (the neighbour's band edge or diagonal); the
    # q-block whose list is full causal (last-L rows) starts a pair
    per_qb = np.bincount(tm.tm_tile_list(N, False, S, W, L)[:, 0], minlength=(N + 127) // 128)
    rec = tm.tm_debug_schedule(1, 8, 2, N, False, S, W, L, 148, mix_pairs=True)
    for c, item, qb, h0, nv, t0, t1 in rec:
        nq = nv & 255
        for k in range(nq):
            assert t1 - per_qb[qb + k] <= 1, (qb, k, t1, per_qb[qb + k])


@pytest.mark.parametrize("W", [512, 2048, 4096, 8192, 16384, 32768])
def test_wide_windows_keep_last_rows_as_big_items(W):
    # The last-L q-blocks cost ~1024 tiles; with wide windows that is only a few
    # percent of a CTA's share, but as a normal item it would land on a handful
    # of CTAs; they count as big items once they cost twice the median q-block.
    N, L = 131072, 256
    per_qb = np.bincount(tm.tm_tile_list(N, False, 64, W, L)[:, 0], minlength=N // 128)
    for split in (False, True):
        rec = tm.tm_debug_schedule(1, 32, 8, N, False, 64, W, L, 148, split=split)
        cost = cta_costs(rec, per_qb)
        assert cost.max() <= 1.02 * cost.mean(), (W, split, cost.max() / cost.mean())


WINDOW_CASES = [  # B, Hq, Hkv, N, causal, S, W, L, chunk rows
    (1, 32, 8, 32768, False, 64, 1024, 128, 4096),
    (1, 32, 8, 32768, True, 0, 1, 0, 4096),
    (1, 32, 8, 131072, False, 64, 2048, 256, 8192),
    (2, 6, 2, 3000, False, 64, 300, 200, 512),
    (1, 28, 4, 5000, True, 0, 1, 0, 1024),
    (1, 14, 2, 777, False, 5, 200, 100, 128),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,S,W,L,chunk", WINDOW_CASES)
def test_row_chunk_windows_cover_each_item_once(B, Hq, Hkv, N, causal, S, W, L, chunk):
    """The host-buffer call runs one launch per row chunk over the q-blocks of
    that chunk; together the launches cover every (q-block, q head) once."""
    nqb = (N + 127) // 128
    seen = {}
    for r0 in range(0, N, chunk):
        lo, hi = r0 // 128, (min(N, r0 + chunk) + 127) // 128
        rec = tm.tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, 148, qb_lo=lo, qb_hi=hi)
        # (a window of the rows keeps head pairs: its q-blocks need not pair up)
        assert len(rec) == (hi - lo) * B * Hkv * ((Hq // Hkv + 1) // 2)
        assert rec[:, 2].min() >= lo and rec[:, 2].max() < hi
        # the longest q-blocks of the chunk come first in each CTA (for causal
        # and the triangle's last-L blocks: the highest q-blocks)
        for c in np.unique(rec[:, 0]):
            mine = rec[rec[:, 0] == c]
            if causal:
                assert mine[0, 2] == mine[:, 2].max()
        for c, item, qb, h0, nv, t0, t1 in rec:
            assert t0 == 0 and nv >> 8 == 0
            for t in rec_tiles(qb, h0, nv):
                assert t not in seen
                seen[t] = 1
    assert len(seen) == nqb * B * Hq


def test_window_arguments_rejected():
    import ctypes
    cnt = ctypes.c_longlong(0)
    L = tm.lib()
    for lo, hi in ((-1, 4), (4, 4), (5, 4), (0, 9)):   # N = 1000: 8 q-blocks
        assert L.tm_debug_schedule_window(1, 4, 2, 1000, 1, 0, 1, 0, 148, 0, lo, hi, None, 0,
                                          ctypes.byref(cnt)) == tm.TM_ERR_INVALID_ARG
    assert L.tm_debug_schedule_window(1, 4, 2, 1000, 1, 0, 1, 0, 148, 0, 3, -1, None, 0,
                                      ctypes.byref(cnt)) == tm.TM_OK
    assert cnt.value == 5 * 2 * 1


@pytest.mark.parametrize("N,L", [(131072, 256), (65536, 128), (32768, 128)])
def test_per_head_band_schedule_is_balanced(N, L):
    # the seeded per-head bands of the bench (windows 512..4096, sinks {0, 64}) on
    # the Llama-3-8B head layout: items are q-block pairs of one head; the heads
    # rotate across the CTAs, and the CTAs that hold a heavy (last-L) item sit
    # out rounds worth the heads' mean cost
    Hq, Hkv = 32, 8
    hS, hW = I.head_bands(Hq, 0)
    rec = tm.tm_debug_schedule_heads(1, Hq, Hkv, N, hS, hW, L, 148)
    cost = np.zeros(148)
    for c, item, qb, h0, nv, t0, t1 in rec:
        nq = nv & 255
        u = union_tiles(N, False, int(hS[h0]), int(hW[h0]), L, qb * 128, min(N, (qb + nq) * 128) - 1)
        cost[c] += (min(u, t1) - t0 + 3) * nq
    assert cost.max() / cost.mean() <= 1.08, cost.max() / cost.mean()


@pytest.mark.parametrize("seed", range(12))
def test_random_causal_odd_groups_cover_each_tile_once(seed):
    # random shapes of odd group size (q-block pairs of one head), with and without
    # the split workspace: every (q-block, q head) Q tile is covered exactly once,
    # and the pieces of an item cover its list (the later q-block's) without gaps
    rng = np.random.default_rng(seed)
    G = int(rng.choice([3, 5, 7, 9]))
    Hkv = int(rng.integers(1, 4))
    B = int(rng.integers(1, 3))
    N = int(rng.integers(1, 6000))
    Hq = G * Hkv
    nqb = (N + 127) // 128
    for split in (False, True):
        rec = tm.tm_debug_schedule(B, Hq, Hkv, N, True, 0, 1, 0, 148, split=split)
        ranges = {}
        for c, item, qb, h0, nv, t0, t1 in rec:
            tiles = tuple(rec_tiles(qb, h0, nv))
            assert nv >> 8 == (1 if G > 1 else 0) and 1 <= (nv & 255) <= 2
            ranges.setdefault(tiles, []).append((t0, t1))
        seen = [t for tiles in ranges for t in tiles]
        assert len(seen) == len(set(seen)) == nqb * B * Hq, (G, Hkv, B, N, split)
        for tiles, rg in ranges.items():
            rg.sort()
            last = max(q for q, _ in tiles)
            assert rg[0][0] == 0 and rg[-1][1] == last + 1, (tiles, rg)
            assert all(a1 == b0 for (_, a1), (b0, _) in zip(rg, rg[1:]))
