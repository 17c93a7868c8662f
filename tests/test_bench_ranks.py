"""The multi-rank path of bench.py on CPU (gloo, world size 2): every rank is
an independent replica of the decode step, the job's time is the slowest
rank's, and the value is microseconds per token over all ranks' tokens.  The
reference arm's other ranks exit without work."""
import argparse
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
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # rank r reports its own times; every rank must see the maximum
        got = bench.max_over_ranks([4.0 + rank, 5.0 + 2 * rank, 3.0 - rank], world, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_gloo_world_2():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == [5.0, 7.0, 3.0]


def test_job_value_counts_every_replica():
    # 2 replicas of BATCH tokens each in 4.3 ms: 4.3 ms / (2 BATCH) tokens
    assert bench.job_us_per_token(4.3, 2) == pytest.approx(4.3e3 / (2 * bench.BATCH))
    assert bench.job_us_per_token(4.3, 1) == pytest.approx(4.3e3 / bench.BATCH)
    assert bench.max_over_ranks([1.5, 2.5], 1, None) == [1.5, 2.5]


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    called = []
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: called.append(1) or (1.0, 1.0, 1))
    args = argparse.Namespace(steps=1, warmup=0, gpus=2, impl="reference", case=None)
    assert bench.run_reference(args, rank=1, world=2) is None
    assert not called
