"""The multi-rank plumbing of bench.py on CPU: two gloo ranks run its
barrier and its max-over-ranks reduction, the two collective steps every
rank of `bench.py --gpus N` takes around the timed region."""

from __future__ import annotations

import importlib.util
import os
import socket
from pathlib import Path

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = importlib.util.spec_from_file_location("bench_module", ROOT / "bench.py")
        bench = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(bench)
        bench.barrier(world)
        # rank r "measured" (r + 1) * 1.5 ms: everyone must report the slowest
        got = bench.max_over_ranks(world, (rank + 1) * 1.5, device="cpu")
        bench.barrier(world)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        assert dict(out) == {0: 3.0, 1: 3.0}


def test_single_rank_is_the_identity():
    spec = importlib.util.spec_from_file_location("bench_module", ROOT / "bench.py")
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    assert bench.max_over_ranks(1, 2.5) == 2.5
    bench.barrier(1)   # no process group needed
    assert torch.tensor([1.0]).item() == 1.0
