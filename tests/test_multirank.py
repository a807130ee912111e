"""The multi-GPU path of the benchmark on CPU: replicas only (every (batch, head) is
independent, so each rank runs the whole workload and no data-path collective exists);
what crosses ranks is the barrier around the timed region and the max over ranks of the
time. These run as world-size-2 gloo process groups."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_body(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        slowest = bench.max_over_ranks(1.0 + rank, world)   # rank 1 is the slow one
        value = bench.replica_value(2e12, slowest, world)
        bench.barrier(world)
        out.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_value_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_body, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time, and the job value counts both replicas
    assert [r[1] for r in res] == [2.0, 2.0]
    assert all(abs(r[2] - 2 * 2e12 / 2e-3 / 1e12) < 1e-9 for r in res)


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference` launched as 2 ranks: rank 0 alone runs the oracle and
    prints one JSON line; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_pisa",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
