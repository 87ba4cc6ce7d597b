"""tm_trianglemix_attn_fwd_noalloc: the layer call with the split schedule on a
fixed device scratch array instead of a caller workspace, for callers that
cannot allocate device memory (a framework or pool that owns every device
byte, or a path where an allocation would synchronise the device).

On the GPU: two calls in a row give the same bits as the workspace entry
point (the scratch's arrival counters are cleared by every call, so the
second call does not see the first one's counts), for a triangle layer that
is split and a causal layer; a triangle call and a causal call with
different split layouts, enqueued back to back on one stream, each give the
workspace entry point's bits; a problem whose split needs more than the
scratch runs the unsplit schedule and gives the bits of the call without a
workspace. Without a GPU: the symbol is exported and bad arguments are
rejected before any CUDA call.
"""
import math

import numpy as np
import pytest

import long_context_prefill_trianglemix_b200 as tm
from long_context_prefill_trianglemix_b200 import build
from long_context_prefill_trianglemix_b200 import inputs as I


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build_lib()
    yield


def test_noalloc_rejects_bad_arguments_without_cuda():
    FAKE = 0x10000
    args = (FAKE, FAKE, FAKE, FAKE + 0x100000, 1, 4, 4, 64, 64, 0.1, 4, 8, 2)
    L = tm.lib()
    assert L.tm_trianglemix_attn_fwd_noalloc(*args, -1, 3, None) == tm.TM_ERR_INVALID_ARG
    assert L.tm_trianglemix_attn_fwd_noalloc(0, *args[1:], 5, 3, None) == tm.TM_ERR_INVALID_ARG
    bad_w = args[:11] + (0, 2)
    assert L.tm_trianglemix_attn_fwd_noalloc(*bad_w, 5, 3, None) == tm.TM_ERR_INVALID_ARG
    assert tm.TM_NOALLOC_SCRATCH_BYTES == 16 << 20


def _inputs(B, Hq, Hkv, N, D, seed):
    import torch
    g = np.random.default_rng(seed)

    def t(shape, scale):
        bits = I.f32_to_bf16_bits((g.standard_normal(shape) * scale).astype(np.float32))
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return t((B, N, Hq, D), 2.0), t((B, N, Hkv, D), 2.0), t((B, N, Hkv, D), 1.0)


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hkv,N,D,S,W,L", [(1, 4, 1, 32768, 128, 64, 1024, 128),
                                               (1, 2, 1, 4173, 128, 5, 100, 200),
                                               (1, 2, 1, 8192, 64, 16, 256, 300),
                                               (1, 3, 1, 4173, 128, 5, 100, 200)])
def test_noalloc_matches_workspace_entry_two_calls_in_a_row(B, Hq, Hkv, N, D, S, W, L):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    q, k, v = _inputs(B, Hq, Hkv, N, D, 41)
    scale = 1.0 / math.sqrt(D)
    assert 0 < tm.tm_attn_workspace_size(B, Hq, Hkv, N, D, False, S, W, L)
    compared = 0
    for layer in (1, 0):  # triangle (split), then causal (split or not, by shape)
        need = tm.tm_attn_workspace_size(B, Hq, Hkv, N, D, layer == 0, S, W, L)
        if need > tm.TM_NOALLOC_SCRATCH_BYTES:  # the unsplit fallback has its own test
            continue
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(q)
        tm.tm_trianglemix_attn_fwd_ws(q, k, v, ref, B, Hq, Hkv, N, D, scale, S, W, L, layer, 1,
                                      ws, need)
        outs = []
        for _ in range(2):
            o = torch.full_like(q, float("nan"))
            tm.tm_trianglemix_attn_fwd_noalloc(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L,
                                               layer, 1)
            outs.append(o)
        torch.cuda.synchronize()
        assert tm.tm_get_device_status() == tm.TM_OK
        for o in outs:
            assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), f"layer {layer}"
        compared += 1
    assert compared >= 1


@pytest.mark.gpu
def test_noalloc_different_splits_back_to_back_on_one_stream():
    """A triangle call and a causal call whose split schedules cut different
    items into different numbers of pieces, enqueued alternately on one stream
    with nothing in between: each call clears the counters its own layout
    uses, so none sees the previous call's counts."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, Hq, Hkv, N, D, S, W, L = 1, 2, 1, 8192, 64, 16, 256, 300
    need = [tm.tm_attn_workspace_size(B, Hq, Hkv, N, D, layer == 0, S, W, L) for layer in (0, 1)]
    assert 0 < need[1] < need[0] <= tm.TM_NOALLOC_SCRATCH_BYTES  # two different layouts
    q, k, v = _inputs(B, Hq, Hkv, N, D, 43)
    scale = 1.0 / math.sqrt(D)
    refs = []
    for layer in (0, 1):
        ws = torch.empty(need[layer], dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(q)
        tm.tm_trianglemix_attn_fwd_ws(q, k, v, ref, B, Hq, Hkv, N, D, scale, S, W, L, layer, 1,
                                      ws, need[layer])
        refs.append(ref)
    torch.cuda.synchronize()
    outs = []
    for layer in (1, 0, 1, 0):
        o = torch.full_like(q, float("nan"))
        tm.tm_trianglemix_attn_fwd_noalloc(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, layer, 1)
        outs.append((layer, o))
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    for layer, o in outs:
        assert torch.equal(o.view(torch.int16), refs[layer].view(torch.int16)), f"layer {layer}"


@pytest.mark.gpu
def test_noalloc_runs_unsplit_when_the_scratch_is_too_small():
    """A causal layer with two heads at 32K cuts so many long items that its
    split needs more than the scratch: the call runs the unsplit schedule,
    whose bits are those of the call without a workspace."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, Hq, Hkv, N, D = 1, 2, 1, 32768, 128
    need = tm.tm_attn_workspace_size(B, Hq, Hkv, N, D, True, 0, 1, 0)
    assert need > tm.TM_NOALLOC_SCRATCH_BYTES
    q, k, v = _inputs(B, Hq, Hkv, N, D, 47)
    scale = 1.0 / math.sqrt(D)
    ref = torch.empty_like(q)
    tm.tm_trianglemix_attn_fwd(q, k, v, ref, B, Hq, Hkv, N, D, scale, 0, 1, 0, 0, 1)
    outs = []
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        tm.tm_trianglemix_attn_fwd_noalloc(q, k, v, o, B, Hq, Hkv, N, D, scale, 0, 1, 0, 0, 1)
        outs.append(o)
    torch.cuda.synchronize()
    assert tm.tm_get_device_status() == tm.TM_OK
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
