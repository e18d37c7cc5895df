"""The multi-GPU bench path on the host: two `gloo` ranks on the CPU.

A multi-GPU run is replicas only (every rank encodes its own batch; the
forward has no exchange step); the only collectives are the barriers and the
max over ranks of the timed region.  These tests run that host logic with
world_size 2 over gloo and check what rank 0 would report.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from jepa_video_encoder_b200 import synth  # noqa: E402

LOCAL_MS = (12.5, 17.25)  # each rank's timed region


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        torch.distributed.barrier()
        total = bench.max_over_ranks(LOCAL_MS[rank], world)
        rate = bench.whole_job_rate(4 * 3137, world, 10, total)
        torch.distributed.barrier()
        q.put((rank, total, rate))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max(LOCAL_MS)
    for rank, total, rate in got:
        assert total == slowest  # every rank agrees on the slowest rank's time
        assert rate == pytest.approx(2 * 4 * 3137 * 10 / (slowest / 1000.0), rel=1e-12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(100, 1, 4, 2000.0) == pytest.approx(200.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    """Under torchrun the oracle arm runs on rank 0; the other ranks exit at
    once with status 0 and print nothing."""
    class Args:
        steps, warmup = 3, 1
    cfg = synth.WORKLOADS["lewm_vit_ti14_224_b1"]
    assert bench.run_reference(Args(), cfg, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
