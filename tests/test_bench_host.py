"""Host logic of bench.py: argument defaults, per-rank workloads and the max-over-ranks
reduction of the multi-GPU path, run as two gloo ranks on CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_defaults_finish_quickly():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and 1 <= a.steps <= 10
    assert a.impl == "ours" and a.workload == "mlp_down"


def test_rank_seeds_are_distinct_and_rank0_is_the_workload_seed():
    seeds = [bench.rank_seed("mlp_down", r) for r in range(8)]
    assert seeds[0] == 2 and len(set(seeds)) == 8


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max(1.5 + rank, "cpu")
        bench.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert res == [(0, 2.5), (1, 2.5)]


def test_reduce_max_single_process_is_identity():
    assert bench.reduce_max(3.25, "cpu") == 3.25
