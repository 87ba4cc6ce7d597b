"""The persistent work split (host export of the same code the launch uses):
every (q-block, q-head pair) item is processed exactly once, the longest
items come first in each CTA, and the per-CTA cost is balanced."""
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


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,S,W,L", CASES)
def test_every_item_exactly_once(B, Hq, Hkv, N, causal, S, W, L):
    rec = tm.tm_debug_schedule(B, Hq, Hkv, N, causal, S, W, L, 148)
    G = Hq // Hkv
    nqb = (N + 127) // 128
    n_items = nqb * B * Hkv * ((G + 1) // 2)
    assert len(rec) == n_items
    assert sorted(rec[:, 1].tolist()) == list(range(n_items))
    # every (batch, q head, q-block) tile appears once
    tiles = set()
    for c, item, qb, h0, nv in rec:
        for h in range(h0, h0 + nv):
            assert (qb, h) not in tiles
            tiles.add((qb, h))
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
    for c, item, qb, h0, nv in rec:
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
    # Items are dealt in strided rounds: each round of 148 consecutive items (what
    # the CTAs run at about the same time) spans a narrow band of q-blocks of every
    # kv head, and each CTA's items are at least a round apart.
    rec = tm.tm_debug_schedule(1, 32, 8, N, causal, 64, W, L, 148)
    order = np.argsort(rec[:, 1])
    items, qbs = rec[order, 1], rec[order, 2]
    for r0 in range(0, len(items) - 148, 148):
        band = qbs[r0:r0 + 148]
        assert band.max() - band.min() <= 10, (r0, band.min(), band.max())
    for c in range(148):
        it = rec[rec[:, 0] == c][:, 1]
        d = np.diff(it)
        assert (d > 0).all() and (d >= 100).all(), (c, it[:6])
