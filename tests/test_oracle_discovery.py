"""Pins of the oracle's block pattern discovery (CPU only): the hand-worked
example in tests/golden/flashprefill_worked_example.txt, the uniform scores of
q = 0, the mean over probes of two known distributions, the probe-row
positions of a ragged block, and the selection's invariants."""
import math
import os
from fractions import Fraction

import numpy as np

import oracle
from long_context_prefill_trianglemix_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "flashprefill_worked_example.txt")


def bits(a):
    return I.f32_to_bf16_bits(np.asarray(a, np.float32))


def worked_inputs(N=8, BS=2):
    q = np.zeros((1, N, 1, 2), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, N, 1, 2), np.float32)
    k[0, :, 0, 0] = np.arange(N) // BS
    return bits(q), bits(k)


def test_worked_example_scores_and_selection():
    q, k = worked_inputs()
    sc = oracle.flashprefill_scores(q, k, 1, 1, 1, 8, 2, math.log(2.0), 1, BS=2)
    off, idx = oracle.flashprefill_select(sc, 0.5)
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        i_s, scores_s, kept_s = line.split()
        Ib = int(i_s)
        want = [float(Fraction(x)) for x in scores_s.split(",")]
        np.testing.assert_allclose(sc[0, Ib, :Ib + 1], want, rtol=0, atol=1e-14)
        assert (sc[0, Ib, Ib + 1:] == 0).all()
        assert idx[off[Ib]:off[Ib + 1]].tolist() == [int(x) for x in kept_s.split(",")]


def test_zero_queries_give_uniform_scores():
    B, Hq, Hkv, N, D = 2, 4, 2, 1000, 16
    q = np.zeros((B, N, Hq, D), np.uint16)
    k = bits(np.random.default_rng(1).standard_normal((B, N, Hkv, D)))
    sc = oracle.flashprefill_scores(q, k, B, Hq, Hkv, N, D, 0.25, 4)
    nb = sc.shape[1]
    for Ib in range(nb):
        np.testing.assert_allclose(sc[:, Ib, :Ib + 1], 1.0 / (Ib + 1), rtol=0, atol=1e-15)
    off, idx = oracle.flashprefill_select(sc, 1.0)  # ties: every block is a maximum
    assert np.diff(off).tolist() == [Ib + 1 for _ in range(B * Hkv) for Ib in range(nb)]


def test_mean_over_probes_and_heads():
    # two q heads on one kv head, one probe each: head 0 sees the worked example,
    # head 1 is zero (uniform); the score is the average of the two distributions
    N, BS = 8, 2
    q1, k = worked_inputs(N, BS)
    q = np.zeros((1, N, 2, 2), np.uint16)
    q[:, :, 0] = q1[:, :, 0]
    sc = oracle.flashprefill_scores(np.ascontiguousarray(q), k, 1, 2, 1, N, 2, math.log(2.0), 1,
                                    BS=BS)
    for Ib in range(4):
        J = np.arange(Ib + 1)
        want = 0.5 * (2.0 ** J / (2.0 ** (Ib + 1) - 1)) + 0.5 / (Ib + 1)
        np.testing.assert_allclose(sc[0, Ib, :Ib + 1], want, rtol=0, atol=1e-14)


def test_probe_rows_of_a_ragged_block():
    # N = 8 in blocks of 3: [0,3), [3,6), [6,8). With P = 2 the probes of a block
    # [r0, r1) are rows r0 + (r1 - r0) // 2 - 1 and r0 + 2 (r1 - r0) // 2 - 1:
    # 0 and 2, then 3 and 5, then (ragged) 6 and 7.
    N, BS = 8, 3
    k = np.zeros((1, N, 1, 2), np.float32)
    k[0, :, 0, 0] = np.arange(N) // BS
    probe_rows = {0: (0, 2), 1: (3, 5), 2: (6, 7)}
    q = np.full((1, N, 1, 2), 0.0, np.float32)
    q[..., 0] = -30.0                      # any row read by mistake would change the scores
    for rows in probe_rows.values():
        for r in rows:
            q[0, r, 0, 0] = 1.0
    sc = oracle.flashprefill_scores(bits(q), bits(k), 1, 1, 1, N, 2, math.log(2.0), 2, BS=BS)
    for Ib in range(3):
        J = np.arange(Ib + 1)
        np.testing.assert_allclose(sc[0, Ib, :Ib + 1], 2.0 ** J / (2.0 ** (Ib + 1) - 1), atol=1e-14)


def test_selection_invariants():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, N, D = 1, 4, 2, 2000, 32
    q = bits(rng.standard_normal((B, N, Hq, D)) * 2)
    k = bits(rng.standard_normal((B, N, Hkv, D)) * 2)
    sc = oracle.flashprefill_scores(q, k, B, Hq, Hkv, N, D, 0.5, 4)
    prev = None
    for alpha in (0.0, 0.2, 0.5, 0.8, 1.0):
        off, idx = oracle.flashprefill_select(sc, alpha)
        lists = [set(idx[off[r]:off[r + 1]].tolist()) for r in range(len(off) - 1)]
        nb = sc.shape[1]
        for r, s in enumerate(lists):
            Ib = r % nb
            assert int(np.argmax(sc[r // nb, Ib, :Ib + 1])) in s  # the best block is kept
            if alpha == 0.0:
                assert s == set(range(Ib + 1))
            if prev is not None:
                assert s <= prev[r]  # a higher alpha keeps a subset
        prev = lists
    # each score row is a probability distribution over the causal blocks
    for Ib in range(sc.shape[1]):
        np.testing.assert_allclose(sc[:, Ib, :Ib + 1].sum(-1), 1.0, atol=1e-12)


def test_block_shorter_than_the_probe_count_repeats_rows():
    # N = 3 in blocks of 128 with 8 probes: rows max(0, ((p + 1) * 3) // 8 - 1) =
    # 0, 0, 0, 0, 0, 1, 1, 2; all heads see one block, so the score is exactly 1
    q = bits(np.random.default_rng(4).standard_normal((1, 3, 2, 8)))
    k = bits(np.random.default_rng(5).standard_normal((1, 3, 1, 8)))
    sc = oracle.flashprefill_scores(q, k, 1, 2, 1, 3, 8, 0.3, 8)
    assert sc.shape == (1, 1, 1) and sc[0, 0, 0] == 1.0
