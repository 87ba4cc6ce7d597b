"""Seeded synthetic q, k, v for the TriangleMix workloads.

This module draws numbers and nothing else: no masking, no softmax, no
attention arithmetic. Both the CUDA path and the CPU oracle are fed from it,
so they always see the same bf16 bytes.

The pages measure on model activations of Llama-3-8B / Qwen2.5-7B running
LongBench, RULER and Wikipedia text (TriangleMix blog post, sections 性能 and
缘由; 36kr interview, "Darstellung der Messergebnisse"). None of those are
available here; seeded tensors with the models' attention shapes stand in for
them. The value recipe per workload:

* plain:    q, k, v ~ N(0, 1) rounded to bf16.
* outliers: as plain, then for every kv head g four distinct channels are
            multiplied by 8 in k[..., g, :] and in every q head of g's group
            (the same channels in q and k, so they raise the logits).
* headscale: q and k heads each get their own factor ~ U[0.5, 2].
* planted:  as plain, then attention structure of the kind block-sparse
            methods find (FlashPrefill summary, section 2.1: vertical, slash
            and block patterns) is planted in the last channels of q and k:
            four sine/cosine channel pairs of position with long periods
            (8192 .. 65536 tokens), equal in q and k, so that q_i . k_j gains
            a sum of cos(w (i - j)) terms that favours nearby keys; and, per kv
            head, 16 seeded key blocks whose keys gain +3 in one more channel
            that every query of the group also carries (+3), so every later
            query attends to them.

Element values come from the C generator in ``tm_inputs.c`` (splitmix64 +
Box-Muller, bf16 round-to-nearest-even). Channel choices and head factors are
drawn here from the same splitmix64 finaliser so that they are identical on
every machine.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtm_inputs.so")
_lib = None

TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2
_M64 = (1 << 64) - 1


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: run `python -c 'import __graft_entry__ as g; g.build()'`")
        lib = ctypes.CDLL(_LIB_PATH)
        lib.tm_inputs_fill_bf16.restype = ctypes.c_int
        lib.tm_inputs_fill_bf16.argtypes = [
            ctypes.c_void_p, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
            ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.tm_inputs_normal_at.restype = ctypes.c_double
        lib.tm_inputs_normal_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.tm_inputs_stream_key.restype = ctypes.c_uint64
        lib.tm_inputs_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_int]
        _lib = lib
    return _lib


def _mix64(z: int) -> int:
    z = (z + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _uniform(seed: int, stream: int, n: int) -> float:
    """Uniform in [0, 1) from the splitmix64 stream (seed, stream), draw n."""
    key = _mix64(_mix64(seed) ^ _mix64(stream + 0x5151))
    return (_mix64((key + n) & _M64) >> 11) * (1.0 / (1 << 53))


def default_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def fill_bf16(out, B: int, N: int, H: int, D: int, seed: int, tensor_id: int,
              head_scale=None, chan_scale=None, nthreads: int | None = None):
    """Fill ``out`` (numpy uint16 array or raw host pointer int) for a [B, N, H, D] tensor."""
    lib = _load()
    if isinstance(out, np.ndarray):
        assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == B * N * H * D
        ptr = out.ctypes.data
    else:
        ptr = int(out)
    hs = None if head_scale is None else np.ascontiguousarray(head_scale, dtype=np.float32)
    cs = None if chan_scale is None else np.ascontiguousarray(chan_scale, dtype=np.float32)
    rc = lib.tm_inputs_fill_bf16(
        ctypes.c_void_p(ptr), B, N, H, D, ctypes.c_uint64(seed & _M64), tensor_id,
        None if hs is None else ctypes.c_void_p(hs.ctypes.data),
        None if cs is None else ctypes.c_void_p(cs.ctypes.data),
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("tm_inputs_fill_bf16: bad argument")
    return out


def normal_at(seed: int, tensor_id: int, n: int) -> float:
    """The unrounded normal sample behind flat element n (for generator self-tests)."""
    lib = _load()
    return lib.tm_inputs_normal_at(lib.tm_inputs_stream_key(seed & _M64, tensor_id), n)


@dataclass(frozen=True)
class Workload:
    """One attention workload: shapes, triangle parameters and value recipe."""
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    S: int
    W: int
    L: int
    layers: int = 1
    tri_start: int = 0
    recipe: str = "plain"          # plain | outliers | headscale
    seed_is_layer: bool = False
    windows: tuple = field(default=())

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    def seed(self, layer: int) -> int:
        return layer if self.seed_is_layer else 0


# The workloads: shapes of Llama-3-8B (32 q heads, 8 kv heads, head dim
# 128, 32 layers) and Qwen2.5-7B (28 q heads, 4 kv heads, 28 layers) with the
# layer splits the blog post reports (12 dense layers for Llama-3, 20 for
# Qwen2.5; section 性能) and triangle parameters S/W/L chosen per workload.
WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=4, N=512, D=64, S=16, W=64, L=64,
                     layers=2, tri_start=1),
    "llama3-8b-32k": Workload("llama3-8b-32k", B=1, Hq=32, Hkv=8, N=32768, D=128,
                              S=64, W=1024, L=128, layers=2, tri_start=1, recipe="outliers"),
    "llama3-8b-64k-32layer": Workload("llama3-8b-64k-32layer", B=1, Hq=32, Hkv=8, N=65536,
                                      D=128, S=64, W=1024, L=128, layers=32, tri_start=12,
                                      seed_is_layer=True),
    "llama3-8b-128k": Workload("llama3-8b-128k", B=1, Hq=32, Hkv=8, N=131072, D=128,
                               S=64, W=2048, L=256, layers=2, tri_start=1,
                               windows=(512, 1024, 2048, 4096)),
    "qwen2.5-7b-128k-28layer": Workload("qwen2.5-7b-128k-28layer", B=1, Hq=28, Hkv=4,
                                        N=131072, D=128, S=64, W=1024, L=128, layers=28,
                                        tri_start=20, recipe="headscale"),
    # One GPU's share of the same layers under tensor parallelism (heads split
    # over 8 and 4 GPUs): few heads per launch, so each last-L item is a large
    # fraction of the launch and is cut into pieces when a workspace is given.
    "llama3-8b-128k-tp8": Workload("llama3-8b-128k-tp8", B=1, Hq=4, Hkv=1, N=131072, D=128,
                                   S=64, W=2048, L=256, layers=2, tri_start=1),
    # The 128K Llama-3-8B shape with planted vertical and local attention
    # structure, the input of block pattern discovery.
    "llama3-8b-128k-planted": Workload("llama3-8b-128k-planted", B=1, Hq=32, Hkv=8, N=131072,
                                       D=128, S=64, W=2048, L=256, layers=2, tri_start=1,
                                       recipe="planted"),
    "qwen2.5-7b-128k-tp4": Workload("qwen2.5-7b-128k-tp4", B=1, Hq=7, Hkv=1, N=131072, D=128,
                                    S=64, W=1024, L=128, layers=28, tri_start=20,
                                    recipe="headscale"),
}


def outlier_channels(seed: int, Hkv: int, D: int, count: int = 4):
    """Per kv head, ``count`` distinct channels drawn without replacement."""
    chans = []
    for g in range(Hkv):
        picked, n = [], 0
        while len(picked) < count:
            c = int(_uniform(seed, 1000 + g, n) * D)
            n += 1
            if c not in picked:
                picked.append(c)
        chans.append(sorted(picked))
    return chans


def head_scales(seed: int, H: int, stream: int):
    return np.array([0.5 + 1.5 * _uniform(seed, stream, h) for h in range(H)], dtype=np.float32)


def scales_for(wl: Workload, layer: int = 0):
    """(head_scale, chan_scale) for q, k, v under the workload's recipe."""
    seed = wl.seed(layer)
    none = (None, None)
    if wl.recipe == "plain":
        return none, none, none
    if wl.recipe == "outliers":
        G = wl.Hq // wl.Hkv
        cq = np.ones((wl.Hq, wl.D), np.float32)
        ck = np.ones((wl.Hkv, wl.D), np.float32)
        for g, chans in enumerate(outlier_channels(seed, wl.Hkv, wl.D)):
            for c in chans:
                ck[g, c] = 8.0
                cq[g * G:(g + 1) * G, c] = 8.0
        return (None, cq.reshape(-1)), (None, ck.reshape(-1)), none
    if wl.recipe == "planted":
        return none, none, none
    if wl.recipe == "headscale":
        return (head_scales(seed, wl.Hq, 2000), None), (head_scales(seed, wl.Hkv, 2001), None), none
    raise ValueError(wl.recipe)


PLANT_PERIODS = (8192.0, 16384.0, 32768.0, 65536.0)
PLANT_AMP = 2.0
PLANT_VERTICAL_BLOCKS = 16
PLANT_VERTICAL_AMP = 3.0


def planted_vertical_blocks(seed: int, Hkv: int, nblocks: int):
    """Per kv head, the seeded key blocks of the planted recipe's vertical pattern."""
    return [sorted({int(_uniform(seed, 4000 + g, n) * nblocks)
                    for n in range(PLANT_VERTICAL_BLOCKS)}) for g in range(Hkv)]


def _plant(arr: np.ndarray, tensor_id: int, seed: int, G: int, BM: int = 128):
    """Add the planted structure to bf16 bits arr [B, N, H, D] in place (last
    2 * len(PLANT_PERIODS) + 1 channels; float32 sums rounded to bf16 RNE).
    Uses torch's CPU tensors only for their fast strided copies."""
    import torch
    B, N, H, D = arr.shape
    nc = 2 * len(PLANT_PERIODS) + 1
    sl = torch.from_numpy(arr.view(np.int16))[..., D - nc:]
    x = ((sl.to(torch.int32) & 0xFFFF) << 16).view(torch.float32)      # [B, N, H, nc]
    pos = np.arange(N, dtype=np.float64)
    add = np.zeros((N, nc), np.float32)
    for c, period in enumerate(PLANT_PERIODS):
        w = 2.0 * np.pi / period
        add[:, nc - 1 - 2 * c] = PLANT_AMP * np.cos(w * pos)           # channel D - 1 - 2c
        add[:, nc - 2 - 2 * c] = PLANT_AMP * np.sin(w * pos)           # channel D - 2 - 2c
    x += torch.from_numpy(add)[None, :, None, :]
    if tensor_id == TENSOR_Q:
        x[..., 0] += PLANT_VERTICAL_AMP                                 # channel D - nc
    elif tensor_id == TENSOR_K:
        for g, blocks in enumerate(planted_vertical_blocks(seed, H, (N + BM - 1) // BM)):
            for blk in blocks:
                x[:, blk * BM:(blk + 1) * BM, g, 0] += PLANT_VERTICAL_AMP
    sl.copy_(x.to(torch.bfloat16).view(torch.int16))


def make_qkv(wl: Workload, layer: int = 0, out=None, N: int | None = None, nthreads=None):
    """Return (q, k, v) as uint16 arrays of bf16 bits, shapes [B,N,Hq,D], [B,N,Hkv,D] x2.

    ``out`` may be a tuple of three preallocated uint16 arrays (e.g. views of
    pinned host tensors). ``N`` overrides the workload's sequence length.
    """
    N = wl.N if N is None else N
    seed = wl.seed(layer)
    (qh, qc), (kh, kc), (vh, vc) = scales_for(wl, layer)
    shapes = [(wl.B, N, wl.Hq, wl.D), (wl.B, N, wl.Hkv, wl.D), (wl.B, N, wl.Hkv, wl.D)]
    if out is None:
        out = tuple(np.empty(s, np.uint16) for s in shapes)
    for arr, shp, tid, hs, cs in zip(out, shapes, (TENSOR_Q, TENSOR_K, TENSOR_V),
                                    (qh, kh, vh), (qc, kc, vc)):
        fill_bf16(arr.reshape(-1), *shp[:2], shp[2], shp[3], seed, tid, hs, cs, nthreads)
        if wl.recipe == "planted" and tid != TENSOR_V:
            _plant(arr.reshape(shp), tid, seed, wl.Hq // wl.Hkv)
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float32 -> bf16 bits (NaN kept quiet). The 32-bit
    sum can wrap only for NaN bit patterns, which are handled separately."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16))
    r = r.astype(np.uint16)
    nan = (u & np.uint32(0x7F800000)) == np.uint32(0x7F800000)
    nan &= (u & np.uint32(0x007FFFFF)) != 0
    if nan.any():
        r[nan] = ((u[nan] >> np.uint32(16)) | np.uint32(0x40)).astype(np.uint16)
    return r


@dataclass(frozen=True)
class BlockIndexRecipe:
    """Structure of a synthetic block index (128 x 128 blocks) for the
    block-sparse shallow layers. The FlashPrefill summary (section 2.1) names
    the structures such indices hold: vertical (key blocks every query block
    attends to), slash (fixed distances below the diagonal) and scattered
    blocks; the first block (sinks) and the blocks next to the diagonal are
    kept by every such method. Counts are per (batch, kv head) for vertical
    and slash, per q-block for the local band; ``p_block`` is the chance that
    any other causal block is kept."""
    local: int = 8        # blocks qb-local+1 .. qb
    sink: int = 1         # blocks 0 .. sink-1
    vertical: int = 32    # seeded key blocks kept by every later q-block
    slash: int = 8        # seeded distances d: block qb - d
    p_block: float = 0.0  # independent chance of any remaining block


def make_block_index(B: int, Hkv: int, N: int, seed: int, recipe: BlockIndexRecipe = None,
                     BM: int = 128):
    """CSR block index: offsets int32 [B * Hkv * nqb + 1], indices int32 [nnz],
    each list strictly ascending within [0, qb]. Draws only index structure."""
    recipe = recipe or BlockIndexRecipe()
    nqb = (N + BM - 1) // BM
    lists = []
    for b in range(B):
        for g in range(Hkv):
            stream = 3000 + 64 * (b * Hkv + g)
            vert = {int(_uniform(seed, stream, n) * nqb) for n in range(recipe.vertical)}
            dist = {1 + int(_uniform(seed, stream + 1, n) * max(1, nqb - 1))
                    for n in range(recipe.slash)}
            rnd_key = _mix64(_mix64(seed) ^ _mix64(stream + 2))
            for qb in range(nqb):
                kb = set(range(max(0, qb - recipe.local + 1), qb + 1))
                kb |= set(range(min(recipe.sink, qb + 1)))
                kb |= {c for c in vert if c <= qb}
                kb |= {qb - d for d in dist if d <= qb}
                if recipe.p_block > 0:
                    rng = np.random.default_rng((rnd_key + qb) & _M64)
                    extra = np.flatnonzero(rng.random(qb + 1) < recipe.p_block)
                    kb |= set(extra.tolist())
                lists.append(sorted(kb))
    offsets = np.zeros(len(lists) + 1, np.int32)
    offsets[1:] = np.cumsum([len(x) for x in lists])
    indices = np.fromiter((c for x in lists for c in x), dtype=np.int32, count=int(offsets[-1]))
    return offsets, indices


def full_causal_index(B: int, Hkv: int, N: int, BM: int = 128):
    """CSR index listing every causal block (block-sparse = causal attention)."""
    nqb = (N + BM - 1) // BM
    per = [list(range(qb + 1)) for qb in range(nqb)] * (B * Hkv)
    offsets = np.zeros(len(per) + 1, np.int32)
    offsets[1:] = np.cumsum([len(x) for x in per])
    return offsets, np.fromiter((c for x in per for c in x), np.int32, count=int(offsets[-1]))


def head_bands(Hq: int, seed: int, w_min: int = 512, w_max: int = 4096, sinks=(0, 64)):
    """Seeded per-head (S_h, W_h): windows log-uniform in [w_min, w_max], sinks
    drawn from ``sinks`` (a calibrated policy stands in for nothing here; this
    only spreads the bands the way per-head calibration would)."""
    S = np.array([sinks[int(_uniform(seed, 5000, h) * len(sinks)) % len(sinks)]
                  for h in range(Hq)], np.int32)
    lo, hi = np.log(w_min), np.log(w_max)
    W = np.array([int(round(np.exp(lo + (hi - lo) * _uniform(seed, 5001, h)))) for h in range(Hq)],
                 np.int32)
    return S, W
