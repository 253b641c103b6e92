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


def test_sweep_bytes_and_roofline():
    """Sweep bytes of the 2048 x 6144 bf16 layer at 3 bits, groups of 128: W 25.2 MB, the upper
    triangle of U 75.5 MB, codes 4.7 MB, scales and zero-points 0.49 MB; the GEMM share is
    subtracted from the stage time."""
    from types import SimpleNamespace
    W = torch.empty(2048, 6144, dtype=torch.bfloat16)
    layer = SimpleNamespace(m=2048, n=6144, W=W, bits=3, group_size=128)
    b = bench.sweep_bytes(layer)
    assert b == 2048 * 6144 * 2 + 4 * 6144 * 6145 // 2 + 2048 * 6144 * 3 // 8 + 2048 * 48 * 5
    assert abs(b / 1e6 - 105.9) < 0.1
    r = bench.sweep_roofline(layer, 2.0, {"sweep_tc": {"ms": 1.25}, "factor_tc": {"ms": 4.0},
                                          "peak_tc": 229.0})
    assert abs(r["achieved_gbs"] - b / 2e-3 / 1e9) < 1e-9
    assert r["gemm_ms"] == 1.25 and abs(r["column_loop_ms"] - 0.75) < 1e-12
    assert 0 < r["frac"] < 1
    assert "gemm_ms" not in bench.sweep_roofline(layer, 2.0, None)


def _layer_digest(rank):
    """The rank's own layer (weak scaling: an independent layer per rank) through the oracle:
    (number of weights, code digest, the layer's first weight)."""
    import hashlib
    import numpy as np
    import datagen
    import oracle
    L = datagen.tiny(device="cpu", seed=bench.rank_seed("tiny", rank))
    res = oracle.gptq_layer(L.W.double().numpy(), L.X.double().numpy(), L.bits, L.group_size,
                            L.lambda_rel)
    codes = np.ascontiguousarray(res["codes"].astype(np.int64))
    return L.m * L.n, hashlib.sha256(codes.tobytes()).hexdigest(), float(L.W[0, 0])


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = _layer_digest(rank)
        every = [None] * world
        dist.all_gather_object(every, mine)
        q.put((rank, every))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_quantize_their_own_layers():
    """The multi-GPU path shards by layer: each rank quantizes the independent layer its seed
    names, with no data exchange. Two gloo ranks gather what they computed; each rank's result
    equals a standalone run of its seed, the two layers differ, and the whole-job unit count is
    the sum over ranks (bench.py reports world x m x n weights per step)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got[0] == got[1]                      # both ranks hold the same gathered view
    every = got[0]
    alone = [_layer_digest(r) for r in range(2)]
    assert every == alone                        # rank r computed exactly seed r's layer
    assert every[0][1] != every[1][1] and every[0][2] != every[1][2]
    assert sum(e[0] for e in every) == 2 * 256 * 256
