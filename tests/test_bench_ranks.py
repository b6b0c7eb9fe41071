"""The multi-rank host logic of bench.py on CPU: two gloo ranks, each with
its own (different) timing, agree on the slowest rank's time and on the
whole-job throughput; the reference arm leaves every rank but 0 at once."""

import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        local_ms = [12.5, 40.0][rank]
        m = b.max_over_ranks(local_ms, torch, dist, world, "cpu")
        v = b.job_throughput(50, 100, m, world)
        out[rank] = (m, v)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        m, v = out[r]
        assert m == 40.0
        assert v == pytest.approx(world * 50 * 100 / 0.040)


def test_one_rank_is_the_identity():
    b = _bench()
    assert b.max_over_ranks(7.25, torch, dist, 1, "cpu") == 7.25
    assert b.job_throughput(64, 10, 2.0, 1) == pytest.approx(64 * 10 / 0.002)


def test_reference_arm_skips_ranks_other_than_zero(monkeypatch):
    b = _bench()
    monkeypatch.setenv("RANK", "1")

    class Args:
        config, steps, warmup, gpus = "tiny_adarms", 3, 3, 2
    assert b.run_reference(Args()) == 0
