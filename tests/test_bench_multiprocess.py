"""The benchmark's multi-process logic on CPU with two gloo ranks: the time
reported is the slowest rank's (element-wise max over ranks, the same on
every rank), the value counts every rank's tokens, each replica draws its
own batch, and the reference arm does its work on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def free_port() -> int:
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        times = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 7.0], world, "cpu")
        out[rank] = times
    finally:
        dist.destroy_process_group()


def test_times_are_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(worker, args=(2, free_port(), out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    assert res[0] == res[1] == [11.0, 5.0, 7.0]


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks([1.5, 2.0], 1) == [1.5, 2.0]


def test_whole_job_value_counts_every_rank():
    # 200,704 tokens per rank, 2 ranks, 50 us per step
    assert bench.whole_job_tokens_per_s(200704, 2, 0.05) == pytest.approx(200704 * 2 / 50e-6)


def test_replicas_draw_different_batches():
    import bra_inputs as bi
    shape, seed = bi.WORKLOADS["tiny"]
    a = bi.make_inputs(shape, bench.rank_seed(seed, 0)).q_store
    b = bi.make_inputs(shape, bench.rank_seed(seed, 1)).q_store
    assert not (a == b).all()


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
