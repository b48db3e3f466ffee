"""The multi-rank host logic of bench.py on CPU: two gloo ranks, independent sequences,
the step time reduced as the max over ranks, whole-job throughput."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = bench.shard_plan(rank, world, 4096, 512)
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms)
        seeds = [None] * world
        dist.all_gather_object(seeds, plan["seed"])
        from sparse_attention_17_b200 import inputs as G
        d = G.mla_prefill_gauss(T=64, seed=plan["seed"], k=16)
        sig = float(d["kv"].float().sum())
        sigs = [None] * world
        dist.all_gather_object(sigs, sig)
        out[rank] = (ms, tuple(seeds), tuple(sigs),
                     bench.aggregate_tokens_per_s(plan["tokens"], world, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0          # max over ranks
    assert res[0][1] == (0, 1)                      # each rank its own sequence
    assert res[0][2][0] != res[0][2][1]             # ... with different inputs
    assert res[0][3] == pytest.approx(2 * 4096 / 0.015)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    with pytest.raises(ValueError):
        bench.shard_plan(2, 2, 10, 1)
