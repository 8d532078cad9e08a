"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): the time of a
step is the max over ranks, the rate counts every rank's batch (weak scaling),
and only rank 0 prints the reference arm's line."""
import io
import os
import socket
import contextlib

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 5.5][rank]
        out[rank] = bench.max_over_ranks(ms, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == 5.5 and out[1] == 5.5


def test_weak_scaling_rate_counts_every_rank():
    one = bench.whole_job_rate(1, 10, 1000.0, 20.0)
    two = bench.whole_job_rate(2, 10, 1000.0, 20.0)
    assert two == 2 * one
    assert one == pytest.approx(10 * 1000.0 / 0.020)


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(1.25, torch.device("cpu")) == 1.25


def test_reference_arm_prints_on_rank_zero_only():
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0",
                             "--cpu-seconds", "1", "--workload", "tiny_f32_b1h1_t64_d16"])
    from recurrent_decode_la_b200 import inputs
    wl = inputs.WORKLOADS[args.workload]
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args, wl, world=2, rank=1) == 0
    assert buf.getvalue() == ""
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args, wl, world=2, rank=0) == 0
    import json
    line = json.loads(buf.getvalue().strip())
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
