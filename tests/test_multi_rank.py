"""Multi-GPU runs are replicas: the (batch, kv-head group) units shard with no
exchange, so the only collective is the max-over-ranks reduction of timings.
These tests run that path with two gloo ranks on the CPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r pretends its replica took (10 + r) ms for the whole run and 3 + 2r ms e2e
        total, tri, e2e = bench.reduce_over_ranks([100.0 + rank, 10.0 + rank, 3.0 + 2 * rank])
        value = bench.whole_job_tflops(world, 5, 2e12, tri)
        out.put((rank, total, tri, e2e, value))
    finally:
        dist.destroy_process_group()


def test_timings_reduce_to_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, total, tri, e2e, value in res:
        assert (total, tri, e2e) == (101.0, 11.0, 5.0)
        # two replicas x five steps x 2 TFLOP each over the slowest 11 ms
        assert value == pytest.approx(2 * 5 * 2e12 / 11e-3 / 1e12)


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks([1.5, 2.5]) == [1.5, 2.5]


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3", "--ref-rows", "4"],
                       capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    if rank == 0:
        line = json.loads(lines[-1])
        assert line["impl"] == "reference" and line["n_gpus"] == 2
        assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
        assert line["unit"] == "TFLOP/s" and line["value"] > 0
    else:
        assert lines == []
