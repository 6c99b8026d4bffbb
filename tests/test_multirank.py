"""The N > 1 benchmark path on CPU: two gloo ranks exercise the barrier and the max-over-ranks
aggregation that bench.py uses with NCCL on GPUs (the attention path itself shards with no
collective: each rank runs an independent batch)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench._barrier(world)
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        ms, tflops = bench.whole_job_rate(local_ms, 1e12, world, device="cpu")
        out[rank] = (ms, tflops)
        bench._barrier(world)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_aggregate_max_time_and_total_work():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms, tflops = out[rank]
        assert ms == 15.0                        # the slowest rank's time
        assert abs(tflops - 2 * 1e12 / 15e-3 / 1e12) < 1e-9  # both ranks' work over that time


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        gpus, steps, warmup = 2, 1, 3

    from attn_workloads import WORKLOADS

    assert bench.run_reference(A(), WORKLOADS[2], 2, 1) is None


def test_single_rank_needs_no_process_group():
    assert bench.whole_job_rate(4.0, 2e9, 1, device="cpu") == (4.0, 2e9 / 4e-3 / 1e12)
