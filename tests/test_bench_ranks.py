"""The multi-rank timing path of bench.py on CPU: gloo, world size 2.

Each rank times its own replica; the job's device time is the maximum over
ranks and the throughput counts every rank's tokens.  Run here on gloo ranks
(the GPU launch uses the same functions over NCCL).
"""
import importlib.util
import os
import socket
from pathlib import Path

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", ROOT / "bench.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        ms = b.max_over_ranks(times[rank], world)
        out[rank] = (ms, b.job_tok_s(ms, 10, world))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    times = [123.0, 250.0]
    mp.start_processes(_rank, args=(world, port, times, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        ms, tok = out[r]
        assert ms == 250.0
        assert tok == pytest.approx(world * 10 / 0.25)


def test_single_rank_is_identity():
    b = _bench()
    assert b.max_over_ranks(7.5, 1) == 7.5
    assert b.job_tok_s(500.0, 20, 1) == pytest.approx(40.0)
