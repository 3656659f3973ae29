"""Host logic of the multi-rank benchmark, run as two gloo ranks on CPU.

Each rank runs its own replica of the layer on its own batch (row split, weak
scaling): the only cross-rank steps are the barriers around the timed loop and
the maximum of the per-rank step times. These tests drive the same helpers
bench.py uses under torchrun, over gloo instead of NCCL."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, step_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench

    w, r, local = bench.dist_setup(world, timeout_s=60)
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    slowest = bench.max_over_ranks(w, step_ms[rank])
    out[rank] = slowest
    bench.barrier(w)
    dist.destroy_process_group()


@pytest.mark.parametrize("step_ms", [(0.125, 0.25), (0.5, 0.0625)])
def test_step_time_is_the_slowest_rank(step_ms):
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), step_ms, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1] == max(step_ms)


def test_whole_job_throughput_counts_every_rank():
    import bench

    flops = 2.0 * 4608 * 3072 * 9216
    one = bench.whole_job_tflops(1, flops, 0.1)
    assert abs(one - flops / 1e-4 / 1e12) < 1e-9
    # weak scaling: N ranks each doing one step in the same time is N times the work
    assert abs(bench.whole_job_tflops(4, flops, 0.1) - 4 * one) < 1e-9
    # the slowest rank sets the time
    assert bench.whole_job_tflops(2, flops, 0.2) == pytest.approx(one)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, ref_rows = 1, 3, 1

    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""


def test_trimmed_mean_drops_both_tails():
    import bench

    xs = [1.0] * 8 + [100.0, -50.0]
    assert bench.trimmed_mean(xs, 0.1) == 1.0
    assert bench.trimmed_mean([2.0, 4.0], 0.1) == 3.0          # too few samples to trim
    ticks = [89.088] * 6 + [90.112] * 4                         # event times on a 1.024 us grid
    assert abs(bench.trimmed_mean(ticks, 0.1) - (5 * 89.088 + 3 * 90.112) / 8) < 1e-9
