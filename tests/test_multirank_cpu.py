"""Multi-rank host logic of bench.py on CPU: two `gloo` ranks in child
processes (the path shards into independent replicas, so the only exchange
is the timing reduction).  Checked: every rank sees the element-wise maximum
of the ranks' device times, the whole-job rate divides all ranks' units by
that slowest time, one process alone is the identity, and under torchrun the
reference arm runs on rank 0 only (other ranks print nothing)."""
import json
import os
import socket
import subprocess
import sys
from argparse import Namespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

WORKER = r"""
import json, os, sys
from datetime import timedelta
sys.path.insert(0, os.environ["REPO_ROOT"])
import torch, torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
try:
    times = [10.0 + rank, 3.0 * (world - rank), 0.25]
    got = bench.max_over_ranks(times, torch.device("cpu"))
    print(json.dumps({"rank": rank, "got": got, "rate": bench.whole_job_rate(world, 50, got[0])}))
finally:
    dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_share_the_slowest_time():
    port, world = _free_port(), 2
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), REPO_ROOT=ROOT)
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=180)
        finally:
            if p.poll() is None:
                p.kill()
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(o["rank"] for o in outs) == [0, 1]
    for o in outs:
        assert o["got"] == [11.0, 6.0, 0.25]  # max over ranks, element by element
        assert o["rate"] == pytest.approx(world * 50 / 11.0e-3)


def test_one_process_is_the_identity():
    import torch
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]
    assert bench.whole_job_rate(1, 10, 20.0) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    args = Namespace(warmup=3, steps=2, gpus=2, impl="reference")
    assert bench.reference_arm(args, 1, 2) is None
    assert capsys.readouterr().out == ""
