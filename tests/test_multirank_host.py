"""The N > 1 launch path of bench.py on CPU: world_size-2 gloo ranks.

The layer shards into independent replicas, one per GPU, with no collective
on the data path; the only cross-rank steps are the barrier around the timed
region and the max-over-ranks reduction of the time.  These tests run that
host logic on CPU ranks (gloo, 127.0.0.1) and check that the reference arm
runs on rank 0 only.
"""
from __future__ import annotations

import contextlib
import io
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank "measured" a different time for its replica: every rank
        # gets the slowest, and the line is built from it
        t = bench.max_over_ranks(0.010 * (rank + 1), dist, device="cpu")
        dist.barrier()
        args = type("A", (), {"workload": "qkv", "steps": 10, "warmup": 3})()
        m = {"seconds": t, "ops_per_step": synth.QKV.ops, "warmup": 3,
             "config": bench.workload_config(synth.QKV), "launches_per_step": 2}
        line = bench.build_line(args, m, dist.get_world_size())
        # the reference arm prints on rank 0 only; other ranks exit quietly
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            if rank != 0:
                bench.run_reference(args)
        out.put((rank, t, buf.getvalue(), line))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_only_rank0_reports():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import synth
    for rank, t, printed, line in res:
        assert t == pytest.approx(0.020)
        if rank != 0:
            assert printed == ""
        # whole-job value: both replicas' operations over the slowest time
        assert line["n_gpus"] == 2 and line["scaling"] == "weak"
        assert line["value"] == pytest.approx(2 * synth.QKV.ops * 10 / 0.020 / 1e12, rel=1e-3)
        assert line["ms_per_step"] == pytest.approx(2.0)
        assert line["gpu_launches"] == 20
        assert line["config"] == res[0][3]["config"]


def test_both_arms_report_the_same_config():
    import bench
    import synth
    cfg = bench.workload_config(synth.QKV)
    assert cfg["M"] == 4352 and cfg["K"] == 3072 and cfg["N"] == 9216
    assert "gpu" not in cfg and "kernel_variant" not in cfg   # nothing that differs per arm


def test_gpus_flag_relaunches_under_torchrun():
    import bench
    cmd = bench.launcher_argv(4, 29555, ["--gpus", "4", "--steps", "5"])
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "--master-port=29555" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"] and cmd[-5].endswith("bench.py")


def test_job_rate_counts_every_replica():
    import bench
    # 2 replicas x 10 steps x 1e12 ops in 0.5 s (max over ranks) = 40e12 ops/s
    assert bench.job_rate(1e12, 10, 0.5, 2) == pytest.approx(40e12)
    assert bench.job_rate(1e12, 10, 0.5, 1) == pytest.approx(20e12)
