"""Failure detection on the GPU without a fault: the producer of one CTA is made
to withhold a Q tile (tm_debug_inject_stall), so that CTA's bounded wait runs
out. The launch must end by itself (about two seconds), report TM_ERR_TIMEOUT
through the device status word once, and leave the context usable: the next
call computes the right result."""
import math
import time

import numpy as np
import pytest

import oracle
import long_context_prefill_trianglemix_b200 as tm
from long_context_prefill_trianglemix_b200 import inputs as I
from gpu_util import assert_close, from_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_prefill_trianglemix_b200 import build
    build.build_lib()
    yield


def test_injected_stall_times_out_and_context_stays_usable():
    import torch
    B, Hq, Hkv, N, D, S, W, L = 1, 4, 2, 2048, 128, 16, 256, 64
    g = np.random.default_rng(91)
    q = I.f32_to_bf16_bits(g.standard_normal((B, N, Hq, D)).astype(np.float32))
    k = I.f32_to_bf16_bits(g.standard_normal((B, N, Hkv, D)).astype(np.float32))
    v = I.f32_to_bf16_bits(g.standard_normal((B, N, Hkv, D)).astype(np.float32))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    scale = 1.0 / math.sqrt(D)
    assert tm.tm_get_device_status() == tm.TM_OK
    o = torch.zeros_like(dq)
    t0 = time.perf_counter()
    tm.tm_debug_inject_stall(dq, dk, dv, o, B, Hq, Hkv, N, D, scale, S, W, L)
    assert tm.tm_get_device_status() == tm.TM_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert elapsed < 30.0, elapsed          # the bounded waits ended the launch
    assert tm.tm_get_device_status() == tm.TM_OK   # read once, then cleared
    # the context is usable: a normal call afterwards is correct
    o2 = torch.empty_like(dq)
    tm.tm_triangle_attn_fwd(dq, dk, dv, o2, B, Hq, Hkv, N, D, scale, S, W, L)
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    want = oracle.attention(q, k, v, B, Hq, Hkv, N, D, scale, False, S, W, L)
    assert_close(from_dev(o2), want, "after the injected stall")
