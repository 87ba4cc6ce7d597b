"""Helpers shared by the GPU tests: host<->device copies of bf16 bit arrays,
error statistics, and row samples. No attention arithmetic lives here."""
from __future__ import annotations

import numpy as np

from long_context_prefill_trianglemix_b200 import inputs as I

# bf16-output tolerance of the parity tests (max-abs, mean-abs over compared values)
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev(t) -> np.ndarray:
    """bf16 CUDA tensor -> float32 numpy array (exact)."""
    import torch
    bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return I.bf16_bits_to_f32(bits)


def err_stats(got: np.ndarray, want: np.ndarray):
    e = np.abs(got.astype(np.float64) - want.astype(np.float64))
    return float(e.max()), float(e.mean())


def assert_close(got, want, what=""):
    mx, mean = err_stats(got, want)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def sample_rows(N: int, L: int, seed: int, n_first=128, n_rand=256, n_last=None):
    """The last L rows (or n_last of them), the first rows, and seeded random rows."""
    rng = np.random.default_rng(seed)
    last = list(range(max(0, N - (L if n_last is None else min(L, n_last))), N))
    first = list(range(min(n_first, N)))
    rand = rng.choice(N, size=min(n_rand, N), replace=False).tolist()
    return sorted(set(last + first + rand))
