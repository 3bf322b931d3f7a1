"""Host logic of the multi-GPU bench path, run as world_size-2 gloo ranks on CPU.

The hot path shards by independent (batch, head) work per rank with no data
exchange, so the only multi-rank logic is the timing aggregation: every rank
takes the max of the per-rank times and reports every rank's work over it.
"""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 30.0][rank]
        total = bench.max_over_ranks(local_ms, torch.device("cpu"), True)
        value = bench.job_tflops(world, 2.0e12, 5, total)
        out[rank] = (total, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    # both ranks see the slowest rank's time and the same whole-job value
    assert out[0] == out[1]
    total, value = out[0]
    assert total == 30.0
    assert value == pytest.approx(world * 2.0e12 * 5 / 30.0e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.25, torch.device("cpu"), False) == 7.25
    assert bench.job_tflops(1, 1.0e12, 4, 2.0) == pytest.approx(2000.0)


def test_reference_arm_other_ranks_do_nothing(capsys):
    class A:
        oracle_rows, warmup, steps, bits, lq = 4, 0, 1, 4, 8
    assert bench.run_reference(A, None, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
