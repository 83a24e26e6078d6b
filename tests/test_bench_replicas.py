"""The multi-GPU path of bench.py is N independent replicas (the layer forward does not shard):
each rank times its own steps, the job takes the slowest rank's time, and the value is the
tokens all ranks processed over that time.  Checked here with two gloo ranks on the CPU; the
reference arm runs on rank 0 only."""
import io
import os
import socket
import contextlib

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(torch, dist, times[rank], device="cpu")
        out[rank] = (ms, bench.job_tokens_per_s(world, 4096, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        times = [0.50, 0.75]
        mp.start_processes(_rank_main, args=(2, _free_port(), times, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    ms, value = res[0]
    assert ms == 0.75
    assert value == pytest.approx(2 * 4096 / 0.75e-3)


def test_job_throughput_is_weak_scaling():
    one = bench.job_tokens_per_s(1, 4096, 0.5)
    assert bench.job_tokens_per_s(8, 4096, 0.5) == pytest.approx(8 * one)


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        steps, warmup, gpus = 1, 3, 2
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(Args(), 1) is None
    assert buf.getvalue() == ""


def test_overlap_efficiency_formula():
    # 8 layers, copies slower than compute: ideal = copy + 7 * copy + compute
    assert bench.overlap_efficiency(60.0, 5.0, 8, 60 * 8 + 5) == pytest.approx(1.0)
    assert bench.overlap_efficiency(60.0, 5.0, 8, 2 * (60 * 8 + 5)) == pytest.approx(0.5)
    # compute-bound layers: ideal = copy + 7 * compute + compute
    assert bench.overlap_efficiency(2.0, 10.0, 8, 2.0 + 80.0) == pytest.approx(1.0)


def test_failed_auxiliary_measurement_is_reported_not_fatal(capsys):
    """A decode / other-workload / stack measurement that raises leaves an error entry in the
    line; the headline still prints."""
    import bench

    def boom():
        raise RuntimeError("device check failed")

    assert bench.guarded("decode", lambda: {"T1": 1.0}) == {"T1": 1.0}
    out = bench.guarded("decode", boom)
    assert out == {"error": "RuntimeError: device check failed"}
    assert "decode failed" in capsys.readouterr().err
