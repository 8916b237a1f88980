"""The N > 1 path of bench.py on CPU: world_size-2 gloo ranks (replicas, no data-path
collective; the only collectives are the timing reductions)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slowest = bench.max_over_ranks(10.0 + 3.0 * rank, dist, "cpu")
        q.put((rank, slowest, bench.job_ms_per_layer(slowest, steps=5, world=world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_timing_reduction_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    # both ranks see the slowest rank's time; the job rate counts the layers of both ranks
    assert [g[1] for g in got] == [13.0, 13.0]
    assert [g[2] for g in got] == [pytest.approx(1.3), pytest.approx(1.3)]


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.job_ms_per_layer(20.0, steps=10, world=1) == 2.0


def _reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny", "--steps", "1", "--warmup", "0", "--ref-budget", "0.2"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_on_rank0_only():
    r1 = _reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _reference(0, 2)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "ms/layer"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
