"""Query-row sharding of one long prefill over several GPUs (host-side plumbing).

Query rows of a DSA prefill are independent once every rank holds the full indexer keys
and latent cache: a query selects among, and attends to, keys of the whole prefix.  So
a T-token prefill splits over N ranks as
  1. each rank produces the keys and latent rows of its own contiguous token shard
     (T / N rows);
  2. one all-gather of those rows (k_idx: 128 B per token, latent: 1152 B per token) into
     every rank's own memory;
  3. each rank runs the single-GPU path (indexer + top-k + sparse MLA) for its query rows.
The causal triangle makes late rows dearer than early ones, so the query rows are dealt
in zig-zag blocks: 2N equal blocks, rank r taking blocks r and 2N-1-r, which gives every
rank nearly the same number of (query, key) pairs.  Outputs stay sharded by query block.
"""
from __future__ import annotations


def zigzag_blocks(T: int, world: int, rank: int, align: int = 16) -> list[tuple[int, int]]:
    """Query-row blocks (start, rows) of `rank`: blocks r and 2*world-1-r of 2*world
    blocks of ceil(T / 2world) rows rounded up to `align` (the last ones may be short or
    empty; empty blocks are dropped)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    if T < 0:
        raise ValueError("T must be >= 0")
    nb = 2 * world
    bs = -(-T // nb)
    bs = -(-bs // align) * align if bs else 0
    out = []
    for b in (rank, nb - 1 - rank):
        q0 = b * bs
        rows = min(bs, T - q0)
        if rows > 0:
            out.append((q0, rows))
    return out


def token_shard(T: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous token rows (start, rows) whose keys and latent rows `rank` produces and
    contributes to the all-gather; T must be a multiple of world (equal shards)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    if T % world:
        raise ValueError("T must be a multiple of the number of ranks")
    n = T // world
    return rank * n, n


def pair_counts(blocks: list[tuple[int, int]], k: int) -> tuple[int, int]:
    """(causal (query, key) pairs scored by the indexer, keys attended) of query blocks."""
    scored = sum((q0 + 1 + q0 + rows) * rows // 2 for q0, rows in blocks)
    attended = 0
    for q0, rows in blocks:
        for t in range(q0, q0 + rows):
            attended += min(t + 1, k)
    return scored, attended


def all_gather_rows(local, full, group=None) -> None:
    """full <- the concatenation over ranks of each rank's `local` token shard (equal
    shards, rank order), through torch.distributed (NCCL on GPUs, gloo on CPU)."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        full.copy_(local)
        return
    dist.all_gather_into_tensor(full, local.contiguous(), group=group)


def prefill_rank_rows(lib, q_idx, k_full, w, q, kv_full, blocks, k: int, scores, idx, out,
                      scale: float) -> None:
    """Step 3 for one rank: indexer + top-k per window of its query blocks into the index
    buffer, then sparse MLA for those rows, through the library's C ABI (`lib` is the
    sparse_attention_17_b200 module).  k_full / kv_full hold every token (after the
    all-gather); q_idx, w, q, idx [T, k] and out [T, 16, 512] are indexed by token, and
    only the rows of `blocks` are read or written; scores is a [window, ld] workspace."""
    rw = scores.shape[0]
    for q0, rows in blocks:
        for w0 in range(q0, q0 + rows, rw):
            wr = min(rw, q0 + rows - w0)
            lib.indexer_scores(q_idx, k_full, w, scores, w0, wr)
            lib.topk_select(scores, k, idx[w0:w0 + wr], q_begin=w0, rows=wr)
        lib.sparse_mla_fwd(q[q0:q0 + rows], kv_full, idx[q0:q0 + rows], out[q0:q0 + rows],
                           scale)
