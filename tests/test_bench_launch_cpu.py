"""The benchmark's N-rank launch on CPU: `--gpus N` without a launcher starts
N ranks through torchrun on 127.0.0.1, a world size other than N is refused,
and ranks started that way (gloo here) find their rank from the launcher's
environment, take the slowest rank's step time and report one whole-job value
from rank 0."""
import json
import os
import socket
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import datetime, json, os, sys
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
import workloads as wl
world, rank, local = bench.check_world(2, os.environ)
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
step = 1e-3 * (1 + rank)                      # rank 1 is the slower replica
slowest = bench.max_over_ranks(step, world)
d = wl.make_config(2, seed=rank)              # each replica has its own batch
value = bench.job_throughput(bench.decode_bytes(d.seq_lens.tolist(), d.Q), slowest, world, 1e9)
if rank == 0:
    print("RESULT " + json.dumps({{"world": world, "slowest": slowest, "value": value}}), flush=True)
dist.destroy_process_group()
"""


def _port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_launch_command_runs_n_ranks_on_localhost():
    cmd = bench.launch_command(["--gpus", "4", "--steps", "7"], 4, 29555)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd and "--master-port=29555" in cmd
    assert cmd[-5].endswith("bench.py") and cmd[-4:] == ["--gpus", "4", "--steps", "7"]


def test_world_size_must_match_gpus():
    assert bench.check_world(1, {}) == (1, 0, 0)
    assert bench.check_world(2, {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}) == (2, 1, 1)
    with pytest.raises(SystemExit):
        bench.check_world(8, {"WORLD_SIZE": "1"})
    with pytest.raises(SystemExit):
        bench.check_world(1, {"WORLD_SIZE": "2"})


def test_two_replica_ranks_through_torchrun(tmp_path):
    script = tmp_path / "rank.py"
    script.write_text(RANK_SCRIPT.format(root=ROOT))
    cmd = bench.launch_command([], 2, _port(), script=str(script))
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("RESULT ")]
    assert len(lines) == 1                    # only rank 0 reports
    res = json.loads(lines[0][len("RESULT "):])
    assert res["world"] == 2 and res["slowest"] == pytest.approx(2e-3)
    one = bench.decode_bytes(__import__("workloads").make_config(2, seed=0).seq_lens.tolist(), 1)
    assert res["value"] == pytest.approx(one * 2 / 2e-3 / 1e9)


@pytest.mark.parametrize("args", [["--config", "4"], ["--config", "5"], ["--config", "2", "--page-size", "196"],
                                  ["--config", "4", "--f16"]])
def test_reference_arm_runs_on_the_host(args):
    """`bench.py --impl reference` times the oracle on the host cores (no GPU)
    and prints one JSON line with the workload's name, unit and a positive
    value, for the prefill workloads and the page-size / fp16 variants too."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", *args], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    if "--page-size" in args:
        assert line["config"]["workload"].endswith("_ps196")
    if "--f16" in args:
        assert line["config"]["workload"].endswith("_f16")
