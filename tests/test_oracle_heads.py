"""Pins of the oracle's per-head bands (CPU only): each head's output equals
the (separately pinned) single-pattern oracle run with that head's sinks and
window on that head alone, equal bands reproduce the shared-band result
exactly, and a head with S = 0, W = 1, L = 0 returns v."""
import numpy as np
import pytest

import oracle
from long_context_prefill_trianglemix_b200 import inputs as I


def rand_bits(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return I.f32_to_bf16_bits((g.standard_normal(shape) * scale).astype(np.float32))


@pytest.mark.parametrize("B,Hq,Hkv,N,D,L", [(1, 4, 2, 300, 16, 20), (2, 6, 3, 257, 8, 0),
                                           (1, 7, 1, 200, 8, 199)])
def test_each_head_is_the_single_pattern_oracle(B, Hq, Hkv, N, D, L):
    rng = np.random.default_rng(N)
    Sh = rng.integers(0, 40, Hq)
    Wh = rng.integers(1, 120, Hq)
    q, k, v = rand_bits((B, N, Hq, D), 1, 2.0), rand_bits((B, N, Hkv, D), 2, 2.0), \
        rand_bits((B, N, Hkv, D), 3)
    got = oracle.attention_heads(q, k, v, B, Hq, Hkv, N, D, 0.3, Sh, Wh, L)
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        qh = np.ascontiguousarray(q[:, :, h:h + 1])
        kh, vh = np.ascontiguousarray(k[:, :, g:g + 1]), np.ascontiguousarray(v[:, :, g:g + 1])
        want = oracle.attention(qh, kh, vh, B, 1, 1, N, D, 0.3, False, int(Sh[h]), int(Wh[h]), L)
        np.testing.assert_array_equal(got[:, :, h:h + 1], want)


def test_equal_bands_are_the_shared_band():
    B, Hq, Hkv, N, D = 1, 8, 2, 400, 16
    q, k, v = rand_bits((B, N, Hq, D), 4), rand_bits((B, N, Hkv, D), 5), rand_bits((B, N, Hkv, D), 6)
    got = oracle.attention_heads(q, k, v, B, Hq, Hkv, N, D, 0.2, [7] * Hq, [50] * Hq, 30)
    want = oracle.attention(q, k, v, B, Hq, Hkv, N, D, 0.2, False, 7, 50, 30)
    np.testing.assert_array_equal(got, want)


def test_identity_head():
    B, Hq, Hkv, N, D = 1, 2, 2, 100, 8
    q, k, v = rand_bits((B, N, Hq, D), 7), rand_bits((B, N, Hkv, D), 8), rand_bits((B, N, Hkv, D), 9)
    got = oracle.attention_heads(q, k, v, B, Hq, Hkv, N, D, 0.2, [0, 5], [1, 9], 0)
    np.testing.assert_array_equal(got[:, :, 0], I.bf16_bits_to_f32(v[:, :, 0]).astype(np.float64))
