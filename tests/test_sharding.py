"""Query-row sharding of one prefill over several ranks, host side: the zig-zag blocks
cover every query row once and balance the causal work; the all-gather of token shards
rebuilds the full key and latent arrays on every rank (two gloo ranks on CPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_17_b200 import sharding as SH


@pytest.mark.parametrize("T,world", [(65536, 1), (65536, 2), (65536, 8), (1000, 3), (7, 4)])
def test_zigzag_blocks_cover_rows_once(T, world):
    seen = torch.zeros(T, dtype=torch.int32)
    for r in range(world):
        for q0, rows in SH.zigzag_blocks(T, world, r):
            assert rows > 0 and q0 % 16 == 0
            seen[q0:q0 + rows] += 1
    assert bool((seen == 1).all())


@pytest.mark.parametrize("world", [2, 4, 8])
def test_zigzag_balances_causal_work(world):
    T, k = 65536, 2048
    work = [SH.pair_counts(SH.zigzag_blocks(T, world, r), k) for r in range(world)]
    scored = [w[0] for w in work]
    attended = [w[1] for w in work]
    assert sum(scored) == T * (T + 1) // 2
    assert max(scored) / min(scored) < 1.01
    # attention: rows before k attend fewer keys, so the rank holding block 0 has less
    # to do; the slowest rank stays within 2 % of the average
    assert max(attended) / (sum(attended) / world) < 1.02


def test_token_shard():
    assert SH.token_shard(65536, 4, 3) == (49152, 16384)
    with pytest.raises(ValueError):
        SH.token_shard(10, 4, 0)
    with pytest.raises(ValueError):
        SH.zigzag_blocks(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T = 96
        full_ref = torch.arange(T * 5, dtype=torch.float32).view(T, 5)
        s0, n = SH.token_shard(T, world, rank)
        local = full_ref[s0:s0 + n].clone()
        full = torch.empty_like(full_ref)
        SH.all_gather_rows(local, full)
        out[rank] = bool(torch.equal(full, full_ref))
    finally:
        dist.destroy_process_group()


def test_all_gather_rows_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res == {0: True, 1: True}


def _oracle_rank_worker(rank, world, port, T, k, out):
    """One rank of the row-sharded prefill with the CPU oracle as the compute: all-gather
    the token shards of k_idx and the latent cache, then indices and attention for the
    rank's zig-zag query blocks only."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as O
        from sparse_attention_17_b200 import inputs as G
        d = G.mla_prefill_int(T=T, k=k, seed=5)
        s0, n = SH.token_shard(T, world, rank)
        k_full = torch.empty_like(d["k_idx"])
        kv_full = torch.empty_like(d["kv"])
        SH.all_gather_rows(d["k_idx"][s0:s0 + n].contiguous(), k_full)
        SH.all_gather_rows(d["kv"][s0:s0 + n].contiguous(), kv_full)
        mine = []
        for q0, rows in SH.zigzag_blocks(T, world, rank):
            idx = O.prefill_indices(d["q_idx"], k_full, d["w"], k, q_begin=q0, rows=rows)
            o, lse = O.sparse_mla_prefill(d["q"][q0:q0 + rows], kv_full, idx, G.SCALE_MLA)
            mine.append((q0, rows, idx, o, lse))
        allr = [None] * world
        dist.all_gather_object(allr, mine)
        if rank == 0:
            out["blocks"] = [b for r in allr for b in r]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,world", [(256, 2), (240, 3)])
def test_row_sharded_oracle_prefill_equals_unsharded(T, world):
    """Sharding is exact: ranks that all-gather the key and latent shards and compute only
    their zig-zag blocks reproduce the unsharded indices and outputs bit for bit."""
    from oracle import oracle as O
    from sparse_attention_17_b200 import inputs as G
    k = 64
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_oracle_rank_worker, args=(world, port, T, k, out), nprocs=world, join=True)
        blocks = out["blocks"]
    d = G.mla_prefill_int(T=T, k=k, seed=5)
    ref_idx = O.prefill_indices(d["q_idx"], d["k_idx"], d["w"], k)
    ref_out, ref_lse = O.sparse_mla_prefill(d["q"], d["kv"], ref_idx, G.SCALE_MLA)
    seen = torch.zeros(T, dtype=torch.int32)
    for q0, rows, idx, o, lse in blocks:
        seen[q0:q0 + rows] += 1
        assert (idx == ref_idx[q0:q0 + rows]).all()
        assert (o == ref_out[q0:q0 + rows]).all() and (lse == ref_lse[q0:q0 + rows]).all()
    assert bool((seen == 1).all())
