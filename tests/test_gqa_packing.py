"""Does packing the q heads of a GQA group into one 128-row tile pay?

The idea: for the band part of the triangle,
put 32 consecutive query rows of each of the G = 4 q heads that share a kv
head into one M = 128 tile, so that one K/V tile feeds all four heads at once
and each 32-row slice visits only the key blocks its own rows keep. The saving
is the key blocks that a whole 128-row q-block visits but a 32-row slice of it
does not.

This counts that saving from the pattern alone (per-row kept intervals: the
sinks [0, S) and the window [i - W + 1, i], or every causal key for the last L
rows; TriangleMix blog post, section 介绍), for every workload's S, W, L. It
finds the saving exactly zero whenever W is a multiple of the 128-key block,
which every configured workload's window is: the band of every row of a
q-block then starts in the same key block, because i - W + 1 ranges over one
block as i ranges over the q-block, except for the block's last row, which
needs one block fewer, and every 32-row slice still holds a row that needs it.
For other windows the saving is at most three quarters of a key block per
q-block and head: 1.8 % of the visited work at W = 1100 and 1.2 % at W = 2000
(no saving at W = 1000), before any cost of the packing itself.
"""
import numpy as np
import pytest

BM = BN = 128


def kept_blocks(i0, i1, N, S, W, L):
    """Key blocks holding a kept key of any row in [i0, i1)."""
    blocks = set()
    for i in range(i0, min(i1, N)):
        if i >= N - L:
            lo_hi = [(0, i + 1)]
        else:
            lo_hi = [(0, min(S, i + 1)), (max(0, i - W + 1), i + 1)]
        for lo, hi in lo_hi:
            if hi > lo:
                blocks.update(range(lo // BN, (hi - 1) // BN + 1))
    return blocks


def mma_rows(N, S, W, L, slice_rows):
    """Visited (query row x key block) units per head when each tile holds
    `slice_rows` rows of one head (128 / slice_rows heads share a tile)."""
    total = 0
    for r0 in range(0, N, slice_rows):
        total += len(kept_blocks(r0, r0 + slice_rows, N, S, W, L)) * slice_rows
    return total


CASES = [  # N, S, W, L: the workloads' triangle parameters, on a shorter N
    (16384, 64, 1024, 128),   # Llama-3-8B 32K / 64K, Qwen2.5-7B 128K
    (16384, 64, 2048, 256),   # Llama-3-8B 128K
    (16384, 64, 512, 256),    # window sweep
    (16384, 64, 4096, 256),
]


@pytest.mark.parametrize("N,S,W,L", CASES)
def test_packing_saves_nothing_when_the_window_is_a_block_multiple(N, S, W, L):
    assert W % BN == 0
    assert mma_rows(N, S, W, L, 32) == mma_rows(N, S, W, L, BM)


@pytest.mark.parametrize("W", [1100, 2000])
def test_packing_saving_is_small_for_other_windows(W):
    N, S, L = 16384, 64, 256
    full, packed = mma_rows(N, S, W, L, BM), mma_rows(N, S, W, L, 32)
    assert packed < full
    nqb = N // BM
    # at most 3/4 of a key block of 128 rows per q-block (here under 2 % of the work)
    assert full - packed <= 0.75 * BM * nqb
    assert 1 - packed / full < 0.02
