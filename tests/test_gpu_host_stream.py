"""tm_trianglemix_attn_fwd_host: the layer call on host buffers, streamed in
row chunks (copy-in, compute on the chunk's q-blocks, copy-out, overlapped).

Its output must be bit for bit that of tm_trianglemix_attn_fwd on the same
data in device memory: each q-block's arithmetic is the same, only which
launch and which CTA run it changes. Cases: the triangle and the causal
layer, ragged N with chunks that end inside the last q-block, D = 64, a
single chunk, the default chunk size, the 32K Llama shape, and a row sample
against the oracle. Argument checks without a GPU live in test_abi.py.
"""
import numpy as np
import pytest

import long_context_prefill_trianglemix_b200 as tm
from long_context_prefill_trianglemix_b200 import inputs as I
from gpu_util import assert_close, sample_rows

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


def pinned_bits(shape, seed, scale):
    import torch
    g = np.random.default_rng(seed)
    bits = I.f32_to_bf16_bits((g.standard_normal(shape) * scale).astype(np.float32))
    return torch.from_numpy(bits.view(np.int16)).pin_memory()


def run_both(B, Hq, Hkv, N, D, S, W, L, layer, tri_start, chunk, seed=7):
    """(host-streamed output, device-call output), both as int16 CPU tensors."""
    import torch
    hq = pinned_bits((B, N, Hq, D), seed, 2.0)
    hk = pinned_bits((B, N, Hkv, D), seed + 1, 2.0)
    hv = pinned_bits((B, N, Hkv, D), seed + 2, 1.0)
    ho = torch.full((B, N, Hq, D), -1, dtype=torch.int16).pin_memory()
    dq, dk, dv = (torch.empty(t.shape, dtype=torch.bfloat16, device="cuda") for t in (hq, hk, hv))
    do = torch.full((B, N, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    scale = 1.0 / np.sqrt(D)
    stream = torch.cuda.current_stream()
    tm.tm_trianglemix_attn_fwd_host(hq, hk, hv, ho, dq, dk, dv, do, B, Hq, Hkv, N, D, scale, S, W,
                                    L, layer, tri_start, chunk, stream)
    stream.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    # the device buffers now hold the inputs: the one-launch call on them
    ref = torch.empty_like(do)
    tm.tm_trianglemix_attn_fwd(dq, dk, dv, ref, B, Hq, Hkv, N, D, scale, S, W, L, layer, tri_start,
                               stream)
    stream.synchronize()
    assert torch.equal(dq.view(torch.int16).cpu(), hq)  # copied in unchanged
    return ho.clone(), ref.view(torch.int16).cpu(), (hq, hk, hv)


CASES = [  # B, Hq, Hkv, N, D, S, W, L, layer, tri_start, chunk rows
    (2, 6, 2, 3000, 128, 64, 300, 200, 1, 1, 512),     # triangle, ragged last chunk
    (2, 6, 2, 3000, 128, 64, 300, 200, 0, 1, 512),     # causal layer
    (1, 4, 2, 1000, 64, 3, 129, 37, 2, 0, 128),        # D = 64, one q-block per chunk
    (1, 8, 2, 2049, 128, 16, 64, 64, 1, 1, 4096),      # a single chunk
    (3, 4, 1, 383, 128, 1, 1, 1, 1, 1, 256),           # tiny window, several batches
    (1, 14, 2, 5000, 128, 5, 200, 100, 1, 1, 0),       # default chunk size (one chunk here)
]


@pytest.mark.parametrize("B,Hq,Hkv,N,D,S,W,L,layer,tri_start,chunk", CASES)
def test_host_stream_equals_device_call_bitwise(B, Hq, Hkv, N, D, S, W, L, layer, tri_start,
                                                chunk):
    import torch
    got, want, _ = run_both(B, Hq, Hkv, N, D, S, W, L, layer, tri_start, chunk)
    assert torch.equal(got, want)


def test_host_stream_llama_32k_bitwise_and_oracle_rows():
    import torch
    import oracle
    wl = I.WORKLOADS["llama3-8b-32k"]
    got, want, (hq, hk, hv) = run_both(wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.S, wl.W, wl.L, 1, 1,
                                       4096)
    assert torch.equal(got, want)
    rows = sample_rows(wl.N, wl.L, 5, 16, 48, n_last=16)
    q, k, v = (t.numpy().view(np.uint16) for t in (hq, hk, hv))
    ref = oracle.attention(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, 1.0 / np.sqrt(wl.D), False,
                           wl.S, wl.W, wl.L, rows=rows)
    out = I.bf16_bits_to_f32(got.numpy().view(np.uint16))[:, rows]
    assert_close(out, ref, "host-streamed 32K triangle, sampled rows")
