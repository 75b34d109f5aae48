"""The N > 1 host path of the benchmark on CPU (gloo, 2 ranks): each rank runs
its own replica of the workload (different seeds, no data exchange), the
step time is the maximum over ranks, and the job throughput counts both
ranks' work."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    import workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        step = 1e-3 * (1 + rank)              # rank 1 is slower
        slowest = bench.max_over_ranks(step, world)
        bench.sync_all(world)
        d = wl.make_config(2, seed=rank)      # replicas: seeded per rank
        digest = float(d.q.float().sum())
        got = [None] * world
        dist.all_gather_object(got, digest)
        value = bench.job_throughput(bench.decode_bytes(d.seq_lens.tolist(), d.Q), slowest, world, 1e9)
        q.put((rank, slowest, got, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, slowest, digests, value in out:
        assert slowest == pytest.approx(2e-3)
        assert digests[0] != digests[1]       # each rank has its own batch
    # both ranks report the same whole-job value
    assert out[0][3] == pytest.approx(out[1][3])
