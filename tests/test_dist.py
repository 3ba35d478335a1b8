"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The scan has no exchange step on one node's data-parallel axis, so N ranks run
N independent replicas; what the ranks share is the timing reduction (max over
ranks) and the whole-job throughput.  These run without a GPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + rank, world, "cpu")
        out[rank] = (ms, bench.throughput(1000, world, 5, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_timing_is_max_over_ranks_and_throughput_counts_all_replicas():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 11.0
    assert res[0][1] == res[1][1] == pytest.approx(1000 * 2 * 5 / 11e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.throughput(10, 1, 2, 1.0) == pytest.approx(20000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import argparse
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(gpus=2, steps=1, warmup=0, impl="reference", workload="tiny_fp32", batch=None,
                              no_e2e=True, no_cpu_baseline=True)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
