"""Query-row sharding of one prefill on the GPU, with N ranks emulated one after another on
a single device: each emulated rank rebuilds the full key and latent arrays from the ranks'
token shards (what the all-gather delivers) and runs sharding.prefill_rank_rows -- the code
the row-sharded benchmark runs -- for its zig-zag blocks.  Together the ranks must write
every row once, with the oracle's indices (integer indexer inputs: exact) and outputs
within the bf16 gate on sampled rows, and bit-identical to the unsharded single call."""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from sparse_attention_17_b200 import sharding as SH
from oracle import oracle as O
from parity import check_close_bf16, check_indices_exact

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.check_device_errors()
    yield
    assert dsa.check_device_errors() == 0


@pytest.mark.parametrize("world", [2, 4])
def test_emulated_ranks_reproduce_the_unsharded_prefill(world):
    T, k = 4096, 2048
    d = G.mla_prefill_int(T=T, k=k, seed=3)
    x = {n: d[n].cuda() for n in ("q_idx", "k_idx", "w", "q", "kv")}
    ld = (T + 3) // 4 * 4
    scores = torch.empty((768, ld), device="cuda")  # windows cut inside the blocks too
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    out = torch.zeros((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    shards = [SH.token_shard(T, world, r) for r in range(world)]
    covered = torch.zeros(T, dtype=torch.int32)
    for r in range(world):
        # the all-gather's result: every rank's token shard, in rank order
        k_full = torch.cat([x["k_idx"][s:s + n] for s, n in shards])
        kv_full = torch.cat([x["kv"][s:s + n] for s, n in shards])
        blocks = SH.zigzag_blocks(T, world, r)
        for q0, rows in blocks:
            covered[q0:q0 + rows] += 1
        SH.prefill_rank_rows(dsa, x["q_idx"], k_full, x["w"], x["q"], kv_full, blocks, k,
                             scores, idx, out, G.SCALE_MLA)
    torch.cuda.synchronize()
    assert bool((covered == 1).all())
    ref_idx = O.prefill_indices(d["q_idx"], d["k_idx"], d["w"], k)
    check_indices_exact(idx, ref_idx, f"{world} emulated ranks: indices")
    rows = np.r_[0:16, 2040:2060, 1000:1010, 3000:3010, T - 16:T]
    ref, _ = O.sparse_mla_prefill(d["q"][rows], d["kv"], ref_idx[rows], G.SCALE_MLA)
    check_close_bf16(out[torch.from_numpy(rows).cuda()], ref, f"{world} emulated ranks: attention")
    # unsharded: one call over all rows; the sharded rows must match it bit for bit
    idx1 = torch.empty((T, k), dtype=torch.int32, device="cuda")
    out1 = torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dsa.layer_stack_workspace_size(T) // 4, device="cuda")
    dsa.layer_stack("F", [x], idx1, ws, k, G.SCALE_MLA, [out1])
    torch.cuda.synchronize()
    assert torch.equal(idx, idx1)
    assert torch.equal(out.view(torch.int16), out1.view(torch.int16))
