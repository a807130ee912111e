"""Head sharding on the host: the partition of the flattened (batch * heads) index over
ranks, the per-rank data (the same bytes the whole run holds), the whole-job value under
strong scaling and the optional all-gather of O, the last two as world-size-2 gloo groups."""
import dataclasses
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from piecewise_attention_diffusion_b200 import synth  # noqa: E402
from piecewise_attention_diffusion_b200.shard import gather_heads, head_range, shard_of  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7, 8])
@pytest.mark.parametrize("n_heads", [0, 1, 2, 5, 24, 40, 128])
def test_head_range_covers_every_head_once(n_heads, world):
    ranges = [head_range(n_heads, world, r) for r in range(world)]
    # contiguous, in rank order, from 0 to n_heads
    assert ranges[0][0] == 0 and ranges[-1][1] == n_heads
    assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
    sizes = [b - a for a, b in ranges]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
    # larger ranges first, so rank 0 holds the largest
    assert sizes == sorted(sizes, reverse=True)
    assert sum(sizes) == n_heads


@pytest.mark.parametrize("args", [(-1, 2, 0), (4, 0, 0), (4, 2, 2), (4, 2, -1)])
def test_head_range_rejects_bad_arguments(args):
    with pytest.raises(ValueError):
        head_range(*args)


def test_shard_of_takes_flattened_heads_across_batch_entries():
    x = torch.arange(2 * 3 * 4 * 5, dtype=torch.float32).reshape(2, 3, 4, 5)
    for world in (1, 2, 4, 6):
        parts = [shard_of(x, world, r) for r in range(world)]
        assert all(p.dim() == 4 and p.shape[0] == 1 for p in parts)
        assert torch.equal(torch.cat([p[0] for p in parts]), x.reshape(6, 4, 5))


@pytest.mark.parametrize("name,batch,heads,world", [("tiny_pisa", 1, 2, 2),
                                                    ("image_pisa", 2, 3, 4)])
def test_shard_data_is_the_whole_runs_bytes(name, batch, heads, world):
    """A rank generates only its heads; they are the bytes of those heads in the whole
    workload (the generator seeds each flattened head on its own)."""
    w = dataclasses.replace(synth.workloads()[name], batch=batch, heads=heads)
    if w.seq_len > 1024:
        w = dataclasses.replace(w, seq_len=1024, grid=(32, 32))
    full = [x.reshape(batch * heads, w.seq_len, w.head_dim) for x in synth.make_qkv(w)]
    for r in range(world):
        h0, h1 = head_range(batch * heads, world, r)
        part = synth.make_qkv(w, heads=range(h0, h1))
        for a, b in zip(part, full):
            assert torch.equal(a, b[h0:h1])


def test_shard_workload_of_the_bench():
    import bench
    w = synth.workloads()["video_pisa"]
    seen = []
    for r in range(3):
        wr, (h0, h1) = bench.shard_workload(w, 3, r)
        assert wr.batch == 1 and wr.heads == h1 - h0 and wr.seq_len == w.seq_len
        seen += list(range(h0, h1))
    assert seen == list(range(40))
    with pytest.raises(SystemExit):
        bench.shard_workload(synth.workloads()["tiny_pisa"], 3, 0)


# ------------------------------------------------------------------ gloo ranks
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
        n_heads, L, d = 5, 3, 2
        full = torch.arange(n_heads * L * d, dtype=torch.float32).reshape(1, n_heads, L, d)
        mine = shard_of(full, world, rank)
        got = gather_heads(mine.clone(), n_heads, world, rank)
        ok_gather = torch.equal(got, full[0])
        # rank r ran (r + 1) TFLOP in its slowest-rank time of 2 ms
        slowest = bench.max_over_ranks(1.0 + rank, world)
        strong = bench.job_value((rank + 1) * 1e12, slowest, world, "heads")
        weak = bench.job_value(1e12, slowest, world, "replicas")
        bench.barrier(world)
        out.put((rank, ok_gather, tuple(mine.shape), strong, weak))
    finally:
        dist.destroy_process_group()


def test_gather_heads_and_job_value_gloo():
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
    # 5 heads over 2 ranks: 3 and 2; every rank holds the whole O after the gather
    assert [r[2] for r in res] == [(1, 3, 3, 2), (1, 2, 3, 2)]
    assert all(r[1] for r in res)
    # strong scaling adds the ranks' work (1 + 2 TFLOP in 2 ms); replicas count N copies
    assert all(abs(r[3] - 3e12 / 2e-3 / 1e12) < 1e-6 for r in res)
    assert all(abs(r[4] - 2 * 1e12 / 2e-3 / 1e12) < 1e-6 for r in res)


def test_gather_heads_single_rank_is_a_reshape():
    x = torch.randn(1, 4, 3, 2)
    assert torch.equal(gather_heads(x, 4, 1, 0), x[0])
    with pytest.raises(ValueError):
        gather_heads(x, 5, 1, 0)
