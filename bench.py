#!/usr/bin/env python
"""Benchmark of TriangleMix prefill attention on B200.

One step = one pass of the TriangleMix layer schedule over one batch of
synthetic inputs of the named workload: the triangle layer (layer index =
tri_start) and the dense causal layer just below it (tri_start - 1), both
through ``tm_trianglemix_attn_fwd``. The headline metric is the triangle
kernel's throughput counting only the FLOPs of the tiles it visits (4*BM*BN*D
per kept 128x128 tile per q head); the causal kernel's time gives the speedup.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With N > 1 (under torchrun) every rank runs an independent replica: the path
shards by (batch, kv-head group) with no exchange, so there is no data-path
collective; only the timing is reduced (max over ranks).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_prefill_trianglemix_b200 import inputs as I  # noqa: E402

METRIC = "triangle-attn prefill TFLOP/s (kept tiles) at 128K; speedup vs own causal"
UNIT = "TFLOP/s"
BM = BN = 128
# Per-launch DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the
# triangle launch of the default workload (llama3-8b-128k, W=2048) from a
# one-launch ncu capture of a process that allocates only that layer, keyed by
# the hash of the build inputs it was taken on; reported only while the
# sources still match (else null).
TRAFFIC: dict = {"8379aa4f698f7c4d": 2263159296 + 1049690880}


def _code_only(text: str) -> str:
    """Source text without // and /* */ comments (and # comments in Python),
    whitespace runs collapsed: a change to comments or layout does not change
    the kernel."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_sources() -> list:
    """The files kernel_source_hash covers."""
    pkg = os.path.join(ROOT, "long_context_prefill_trianglemix_b200")
    paths = [p for p in sorted(glob.glob(os.path.join(pkg, "csrc", "*")))
             if not p.endswith(".py")]
    paths += sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))
    paths.append(os.path.join(pkg, "build.py"))
    return paths


def kernel_source_hash() -> str:
    """Hash of everything that decides what a launch does: every library
    source (kernels, the C-ABI file with the layer dispatch and the schedule
    choice), the public header (tile shape) and the build script (compile
    flags), as code."""
    h = hashlib.sha256()
    for p in kernel_sources():
        with open(p, encoding="utf-8") as f:
            text = f.read()
        if p.endswith(".py"):
            text = re.sub(r"#[^\n]*", " ", text)
        h.update(os.path.basename(p).encode())
        h.update(_code_only(text).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"burst": float(d["bf16_tflops"]), "sustained": float(d["bf16_tflops_sustained"]),
                "hbm": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"burst": 1590.0, "sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


def workload_config(wl, W, n_ranks) -> dict:
    """The `config` object of both arms' JSON lines (same workload, same keys)."""
    q_gb = wl.B * wl.N * wl.Hq * wl.D * 2 / 1e9
    return {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "N": wl.N, "D": wl.D,
            "S": wl.S, "W": W, "L": wl.L, "tri_start": wl.tri_start,
            "step": "triangle layer + causal layer via tm_trianglemix_attn_fwd_ws",
            "l2": "inputs larger than L2 (q alone is %.2f GB)" % q_gb,
            "parallelism": "replicas" if n_ranks > 1 else "single"}


def tile_flop(wl, causal, W=None) -> float:
    import long_context_prefill_trianglemix_b200 as tm
    tiles = tm.tm_kept_tiles(wl.N, causal, wl.S, wl.W if W is None else W, wl.L)
    return float(tiles) * wl.B * wl.Hq * 4.0 * BM * BN * wl.D


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="tm_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        busy = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)]
        return {"sm_mhz": statistics.median(busy or sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(wl, W, n_rows: int, seed: int, host, target_s: float = 0.0):
    """Time the fp64 oracle on a row sample of the triangle layer; returns
    (seconds, tile-FLOP equivalent of the sample, cores, description).
    With target_s > 0 the sample grows (doubling the rows) until one timed
    call lasts about target_s seconds; only that last call is reported."""
    import numpy as np

    import oracle
    q, k, v = host
    # the kept-tile credit comes from the oracle's own tile list, so this leg
    # (and the reference arm) loads no part of the CUDA library
    tiles = oracle.tile_list_rows(wl.N, False, wl.S, W, wl.L)
    per_qb = np.bincount(tiles[:, 0], minlength=(wl.N + BM - 1) // BM)
    cores = oracle.hardware_threads()
    while True:
        rng = np.random.default_rng(seed)
        rows = sorted(rng.choice(wl.N, size=min(n_rows, wl.N), replace=False).tolist())
        t0 = time.perf_counter()
        oracle.attention(q, k, v, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale, False, wl.S, W,
                         wl.L, rows=rows, nthreads=cores)
        dt = time.perf_counter() - t0
        if target_s <= 0 or dt >= 0.5 * target_s or n_rows >= wl.N:
            break
        n_rows = int(n_rows * min(64.0, max(2.0, target_s / max(dt, 1e-3))))
    # each sampled row stands for its share (1/BM) of its q-block's kept tiles
    equiv = float(sum(per_qb[r // BM] for r in rows)) * BN * 4.0 * wl.D * wl.Hq * wl.B
    desc = (f"{len(rows)} seeded random query rows x all {wl.Hq} q heads of the triangle layer "
            f"(W={W}), {cores} threads; credited with their share of the kept-tile FLOPs")
    return dt, equiv, cores, desc


# ----------------------------------------------------------------------------- arms

def reduce_over_ranks(values, device="cpu"):
    """Max over ranks of per-rank timings (ms). The replicas share no data: this
    reduction of the timings is the only collective of a multi-GPU run."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(n_ranks, steps, flop_per_step, max_ms_total):
    """Throughput of N replicas: all ranks' work over the slowest rank's time."""
    return n_ranks * steps * flop_per_step / (max_ms_total * 1e-3) / 1e12


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args):
    ws, rank, _ = dist_setup()
    if rank != 0:
        return 0
    wl = I.WORKLOADS[args.workload]
    W = args.window or wl.W
    host = I.make_qkv(wl)
    for s in range(args.warmup):
        oracle_sample(wl, W, args.ref_rows, 1000 + s, host)
    tot_t, tot_f = 0.0, 0.0
    desc, cores = "", 1
    for s in range(args.steps):
        dt, equiv, cores, desc = oracle_sample(wl, W, args.ref_rows, s, host)
        tot_t += dt
        tot_f += equiv
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl, W, ws),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def algorithmic_bytes(wl) -> float:
    """Minimum HBM bytes of one layer: q, k, v read once and o written once (bf16)."""
    return 2.0 * wl.B * wl.N * wl.D * (2 * wl.Hq + 2 * wl.Hkv)


def timed_calls(stream, calls, steps):
    """Run each of `calls` once per step, timing every call with CUDA events on
    `stream`; returns per-call lists of milliseconds."""
    import torch
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in calls] for _ in range(steps)]
    for s in range(steps):
        for c, fn in enumerate(calls):
            ev[s][c][0].record(stream)
            fn()
            ev[s][c][1].record(stream)
    torch.cuda.synchronize()
    return [[ev[s][c][0].elapsed_time(ev[s][c][1]) for s in range(steps)]
            for c in range(len(calls))]


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import long_context_prefill_trianglemix_b200 as tm

    ws, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wl = I.WORKLOADS[args.workload]
    W = args.window or wl.W
    if wl.layers > 2 and args.legs == "all":
        rc = run_model(args, wl, W, ws, rank)
        if ws > 1:
            dist.barrier()
            dist.destroy_process_group()
        return rc
    tri_layer, causal_layer = wl.tri_start, max(wl.tri_start - 1, 0)
    assert wl.tri_start >= 1

    # pinned host inputs (filled in place by the seeded generator), then device copies
    shp_q, shp_kv = (wl.B, wl.N, wl.Hq, wl.D), (wl.B, wl.N, wl.Hkv, wl.D)
    hq = torch.empty(shp_q, dtype=torch.int16, pin_memory=True)
    hk = torch.empty(shp_kv, dtype=torch.int16, pin_memory=True)
    hv = torch.empty(shp_kv, dtype=torch.int16, pin_memory=True)
    host_np = tuple(t.numpy().view(np.uint16) for t in (hq, hk, hv))
    I.make_qkv(wl, tri_layer, out=host_np)
    dq, dk, dv = (t.cuda().view(torch.bfloat16) for t in (hq, hk, hv))
    do = torch.empty_like(dq)
    stream = torch.cuda.current_stream()

    # workspace for the split schedule (allocated once, outside the timed region;
    # 0 bytes when no item needs cutting, as for all 32 heads of Llama-3-8B)
    ws_bytes = 0
    if args.split == "auto":
        ws_bytes = max(tm.tm_attn_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, causal, wl.S, W,
                                                 wl.L) for causal in (False, True))
    wsbuf = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda") if ws_bytes else None

    def layer_call(layer, q=dq, k=dk, v=dv, o=do):
        tm.tm_trianglemix_attn_fwd_ws(q, k, v, o, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                                      wl.S, W, wl.L, layer, wl.tri_start, wsbuf, ws_bytes, stream)

    tri_f, causal_f = tile_flop(wl, False, W), tile_flop(wl, True)
    step = [lambda: layer_call(tri_layer)]
    if args.legs != "triangle":
        step.append(lambda: layer_call(causal_layer))

    for _ in range(args.warmup):
        for fn in step:
            fn()
    torch.cuda.synchronize()
    if tm.tm_get_device_status(stream) != tm.TM_OK:
        raise RuntimeError("device status not ok after warm-up")

    sampler = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    launches0 = tm.tm_debug_launch_count()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(step) + 1)]
          for _ in range(args.steps)]
    for s in range(args.steps):
        ev[s][0].record(stream)
        for c, fn in enumerate(step):
            fn()
            ev[s][c + 1].record(stream)
    torch.cuda.synchronize()
    launches = tm.tm_debug_launch_count() - launches0
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop()
    status = tm.tm_get_device_status(stream)
    tri_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(args.steps)]
    cau_ms = ([ev[s][1].elapsed_time(ev[s][2]) for s in range(args.steps)]
              if len(step) > 1 else [float("nan")])
    total_ms = ev[0][0].elapsed_time(ev[-1][-1])
    tri_sum = sum(tri_ms)

    extra = {}
    e2e_ms = float("nan")
    if args.legs == "all":
        # end to end through the host-buffer call: pinned host q, k, v in, the
        # triangle layer, pinned host o out, streamed in row chunks (the library
        # overlaps copy-in, compute and copy-out); `stream` completes after the
        # last copy-out, so its events bracket all of it
        ho = torch.empty(shp_q, dtype=torch.int16, pin_memory=True)

        def host_call():
            tm.tm_trianglemix_attn_fwd_host(hq, hk, hv, ho, dq, dk, dv, do, wl.B, wl.Hq, wl.Hkv,
                                            wl.N, wl.D, wl.scale, wl.S, W, wl.L, tri_layer,
                                            wl.tri_start, 0, stream)

        host_call()  # warm-up (the library creates its copy streams on first use)
        e2e_steps = max(3, args.steps)
        e2e_ms = sum(timed_calls(stream, [host_call], e2e_steps)[0]) / e2e_steps
        extra = other_legs(args, wl, W, tm, dq, dk, dv, do, stream, sum(cau_ms) / len(cau_ms),
                           tri_layer)

    total_ms, tri_sum, e2e_ms = reduce_over_ranks([total_ms, tri_sum, e2e_ms], device="cuda")

    peaks = load_peaks()
    tri_avg = tri_sum / args.steps
    achieved = tri_f / (tri_avg * 1e-3) / 1e12
    value = whole_job_tflops(ws, args.steps, tri_f, tri_sum)
    hbm_gbs = algorithmic_bytes(wl) / (tri_avg * 1e-3) / 1e9
    causal_avg = sum(cau_ms) / len(cau_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, W, ws),
        "split_workspace_bytes": ws_bytes,
        "legs": args.legs,
        "triangle_ms": tri_avg,
        "triangle_ms_p10_p90": [float(np.percentile(tri_ms, 10)), float(np.percentile(tri_ms, 90))],
        "causal_ms": causal_avg,
        "causal_tflops": causal_f / (causal_avg * 1e-3) / 1e12,
        "speedup_vs_causal": causal_avg / tri_avg,
        "kept_tile_tflop": tri_f / 1e12,
        "kept_pair_tflops": (tm.tm_triangle_kept_pairs(wl.N, wl.S, W, wl.L) * wl.B * wl.Hq * 4.0
                             * wl.D) / (tri_avg * 1e-3) / 1e12,
        "triangle_hbm": {"algorithmic_bytes": algorithmic_bytes(wl), "gbs": hbm_gbs,
                         "frac_of_measured_hbm": hbm_gbs / peaks["hbm"],
                         "what": "q, k, v read once and o written once, over the triangle "
                                 "launch's time (the kernel is tensor-bound; this is context)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["sustained"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["sustained"],
                     "peak_kind": f"bf16 dense, {peaks['source']} sustained (kernel runs inside "
                                  "a long step after the causal layer)",
                     "frac_of_burst": achieved / peaks["burst"],
                     "traffic": TRAFFIC.get(kernel_source_hash()) if wl.name == "llama3-8b-128k"
                     and W == 2048 else None},
        "gpu_launches": launches,
        "clocks": clocks,
        "device_status": tm.status_string(status),
    }
    if args.legs == "all":
        line["e2e"] = {
            "value": whole_job_tflops(ws, 1, tri_f, e2e_ms), "unit": UNIT,
            "h2d_bytes_per_step": int((dq.numel() + dk.numel() + dv.numel()) * 2),
            "d2h_bytes_per_step": int(do.numel() * 2),
            "what": "tm_trianglemix_attn_fwd_host: pinned host q,k,v -> device, triangle "
                    "layer, output -> pinned host, streamed in 8192-row chunks; mean of %d calls"
                    % max(3, args.steps)}
        line.update(extra)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        dt, equiv, cores, desc = oracle_sample(wl, W, args.cpu_rows, 7, host_np, target_s=10.0)
        line["cpu_baseline"] = {"value": equiv / dt / 1e12, "unit": UNIT, "cores": cores,
                                "kind": "oracle", "sample": desc, "seconds": dt}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == tm.TM_OK else 1


def other_legs(args, wl, W, tm, dq, dk, dv, do, stream, causal_ms, tri_layer):
    """The legs next to the headline step, each timed on its own after it: the
    block-sparse shallow layer on a seeded index, per-head bands, and block
    pattern discovery feeding block-sparse attention."""
    import dataclasses

    import numpy as np
    import torch

    # block-sparse shallow layer (a seeded vertical / slash / local block index,
    # 128x128 blocks)
    bs_off, bs_idx = I.make_block_index(wl.B, wl.Hkv, wl.N, 0)
    d_off = torch.from_numpy(bs_off).cuda()
    d_idx = torch.from_numpy(bs_idx).cuda()

    def sparse_call():
        tm.tm_block_sparse_attn_fwd(dq, dk, dv, do, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                                    d_off, d_idx, len(bs_idx), stream)

    for _ in range(args.warmup):
        sparse_call()
    bs_ms = float(np.mean(timed_calls(stream, [sparse_call], args.steps)[0]))
    bs_f = float(len(bs_idx)) * (wl.Hq // wl.Hkv) * 4.0 * BM * BN * wl.D

    # per-head bands (seeded windows 512..4096 and sinks {0, 64} per q head) on the
    # same inputs; useful FLOPs count each head's own tiles
    hS, hW = I.head_bands(wl.Hq, 0)
    head_tiles = sum(tm.tm_kept_tiles(wl.N, False, int(hS[h]), int(hW[h]), wl.L)
                     for h in range(wl.Hq)) * wl.B
    hb_ws_n = tm.tm_attn_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, False, int(hS.max()),
                                        int(hW.max()), wl.L)
    hb_ws = torch.empty(max(hb_ws_n, 16), dtype=torch.uint8, device="cuda")

    def heads_call():
        tm.tm_triangle_attn_fwd_heads(dq, dk, dv, do, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                                      hS, hW, wl.L, hb_ws, hb_ws_n, stream)

    for _ in range(args.warmup):
        heads_call()
    hb_ms = float(np.mean(timed_calls(stream, [heads_call], args.steps)[0]))

    # block pattern discovery (probes per block, alpha) producing an index on the
    # GPU, then block-sparse attention over it. Seeded N(0,1) tensors have no
    # attention structure to find, so this leg runs on the same shapes with the
    # planted recipe (local and vertical structure).
    pwl = dataclasses.replace(wl, recipe="planted")
    pq, pk, _ = I.make_qkv(pwl, tri_layer)
    dq_p = torch.from_numpy(pq.view(np.int16)).cuda().view(torch.bfloat16)
    dk_p = torch.from_numpy(pk.view(np.int16)).cuda().view(torch.bfloat16)
    del pq, pk
    nqb = (wl.N + BM - 1) // BM
    disc_ws_n = tm.tm_flashprefill_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, args.probes)
    disc_ws = torch.empty(disc_ws_n, dtype=torch.uint8, device="cuda")
    cap = tm.tm_flashprefill_index_capacity(wl.B, wl.Hkv, wl.N)
    f_off = torch.empty(wl.B * wl.Hkv * nqb + 1, dtype=torch.int32, device="cuda")
    f_idx = torch.empty(cap, dtype=torch.int32, device="cuda")

    def discover_call():
        tm.tm_flashprefill_block_index(dq_p, dk_p, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.scale,
                                       args.alpha, args.probes, disc_ws, disc_ws_n, f_off, f_idx,
                                       cap, None, stream)

    def discovered_sparse_call():
        tm.tm_block_sparse_attn_fwd(dq_p, dk_p, dv, do, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D,
                                    wl.scale, f_off, f_idx, cap, stream)

    for _ in range(args.warmup):
        discover_call()
        discovered_sparse_call()
    disc_t, dsa_t = timed_calls(stream, [discover_call, discovered_sparse_call], args.steps)
    disc_ms, dsa_ms = float(np.mean(disc_t)), float(np.mean(dsa_t))
    f_nnz = int(f_off[-1].item())
    bs_ms, disc_ms, dsa_ms, hb_ms = reduce_over_ranks([bs_ms, disc_ms, dsa_ms, hb_ms],
                                                      device="cuda")
    return {
        "block_sparse": {
            "what": "tm_block_sparse_attn_fwd, seeded block index (local 8, sink 1, vertical 32, "
                    "slash 8 blocks per list), timed separately after the steps",
            "ms": bs_ms,
            "tflops_kept_tiles": bs_f / (bs_ms * 1e-3) / 1e12,
            "kept_tiles": int(len(bs_idx)) * (wl.Hq // wl.Hkv),
            "density_vs_causal": len(bs_idx) / (wl.B * wl.Hkv * nqb * (nqb + 1) / 2),
            "speedup_vs_causal": causal_ms / bs_ms,
        },
        "head_bands": {
            "what": "tm_triangle_attn_fwd_heads, seeded per-head windows 512..4096 (log-uniform) "
                    "and sinks {0, 64}, L shared; items pair two q-blocks of one head",
            "ms": hb_ms,
            "tflops_own_tiles": head_tiles * 4.0 * BM * BN * wl.D / (hb_ms * 1e-3) / 1e12,
            "own_tiles": int(head_tiles),
            "speedup_vs_causal": causal_ms / hb_ms,
        },
        "discovery": {
            "what": "tm_flashprefill_block_index (pooled keys, %d probe rows per block and q "
                    "head, alpha %.2f) then tm_block_sparse_attn_fwd over the index it wrote; "
                    "q and k of the planted recipe (local and vertical structure)"
                    % (args.probes, args.alpha),
            "speedup_vs_causal": causal_ms / dsa_ms,
            "discover_ms": disc_ms,
            "attention_ms": dsa_ms,
            "density_vs_causal": f_nnz / (wl.B * wl.Hkv * nqb * (nqb + 1) / 2),
            "attention_tflops_kept_tiles": f_nnz * (wl.Hq // wl.Hkv) * 4.0 * BM * BN * wl.D
                                           / (dsa_ms * 1e-3) / 1e12,
        },
    }


def run_model(args, wl, W, ws, rank):
    """All layers of a multi-layer workload, each with its own seeded inputs
    (seed = layer), resident on the device. One step is one pass of the
    TriangleMix schedule over every layer (causal below tri_start, triangle
    from it); a second pass with every layer causal gives the dense total.
    Totals are sums of the per-layer median times."""
    import numpy as np
    import torch

    import long_context_prefill_trianglemix_b200 as tm

    shp_q, shp_kv = (wl.B, wl.N, wl.Hq, wl.D), (wl.B, wl.N, wl.Hkv, wl.D)
    hq = torch.empty(shp_q, dtype=torch.int16, pin_memory=True)
    hk = torch.empty(shp_kv, dtype=torch.int16, pin_memory=True)
    hv = torch.empty(shp_kv, dtype=torch.int16, pin_memory=True)
    host_np = tuple(t.numpy().view(np.uint16) for t in (hq, hk, hv))
    dev = []
    for layer in range(wl.layers):
        I.make_qkv(wl, layer, out=host_np)
        dev.append(tuple(t.cuda().view(torch.bfloat16) for t in (hq, hk, hv)))
    do = torch.empty_like(dev[0][0])
    stream = torch.cuda.current_stream()
    ws_bytes = 0
    if args.split == "auto":
        ws_bytes = max(tm.tm_attn_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, causal, wl.S, W,
                                                 wl.L) for causal in (False, True))
    wsbuf = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda") if ws_bytes else None

    def call(layer, tri_start):
        q, k, v = dev[layer]
        return lambda: tm.tm_trianglemix_attn_fwd_ws(q, k, v, do, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D,
                                                     wl.scale, wl.S, W, wl.L, layer, tri_start,
                                                     wsbuf, ws_bytes, stream)

    mix = [call(layer, wl.tri_start) for layer in range(wl.layers)]
    dense = [call(layer, wl.layers) for layer in range(wl.layers)]  # every layer causal
    for _ in range(args.warmup):
        for fn in mix + dense:
            fn()
    torch.cuda.synchronize()
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    launches0 = tm.tm_debug_launch_count()
    t_mix = timed_calls(stream, mix, args.steps)
    t_dense = timed_calls(stream, dense, args.steps)
    launches = tm.tm_debug_launch_count() - launches0
    clocks = sampler.stop()
    status = tm.tm_get_device_status(stream)
    med_mix = [float(np.median(t)) for t in t_mix]
    med_dense = [float(np.median(t)) for t in t_dense]
    tri_layers = list(range(wl.tri_start, wl.layers))
    tri_f = tile_flop(wl, False, W)
    tri_ms = sum(med_mix[layer] for layer in tri_layers)
    vals = reduce_over_ranks([tri_ms, sum(med_mix), sum(med_dense)], device="cuda")
    tri_ms, mix_total, dense_total = vals
    peaks = load_peaks()
    achieved = tri_f * len(tri_layers) / (tri_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": ws * achieved, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mix_total,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(wl, W, ws),
        "model": {
            "what": "every layer with its own seeded inputs (seed = layer); totals are sums of "
                    "per-layer medians over the steps",
            "layers": wl.layers, "tri_start": wl.tri_start,
            "trianglemix_total_ms": mix_total,
            "all_causal_total_ms": dense_total,
            "attention_time_saved": 1.0 - mix_total / dense_total,
            "speedup_vs_all_causal": dense_total / mix_total,
            "causal_layers_ms": sum(med_mix[:wl.tri_start]),
            "triangle_layers_ms": tri_ms,
            "per_layer_ms": med_mix,
            "per_layer_all_causal_ms": med_dense,
        },
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["sustained"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["sustained"],
                     "peak_kind": f"bf16 dense, {peaks['source']} sustained",
                     "frac_of_burst": achieved / peaks["burst"], "traffic": None},
        "gpu_launches": launches,
        "clocks": clocks,
        "device_status": tm.status_string(status),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if status == tm.TM_OK else 1


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="llama3-8b-128k", choices=sorted(I.WORKLOADS))
    ap.add_argument("--window", type=int, default=0, help="override W of the workload")
    ap.add_argument("--cpu-rows", type=int, default=256, help="first oracle sample for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=2048, help="oracle rows per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--probes", type=int, default=4, help="discovery probe rows per block")
    ap.add_argument("--alpha", type=float, default=0.3, help="discovery threshold factor")
    ap.add_argument("--split", choices=("auto", "off"), default="auto",
                    help="auto: give the launch the workspace that lets it cut long items")
    ap.add_argument("--legs", choices=("all", "step", "triangle"), default="all",
                    help="all: the step plus the e2e, block-sparse, per-head and discovery legs "
                         "(multi-layer workloads: the whole model); step: the triangle + causal "
                         "step only; triangle: the triangle layer only (for profiling)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps, always
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
