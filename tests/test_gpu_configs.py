"""GPU parity at the full sizes of the five workloads, run through the same entry points
and launch configuration the benchmark uses (windowed indexer + top-k, then sparse MLA),
checked against the CPU oracle on every output it can afford and on sampled rows
elsewhere.

  tiny fp32    T=3072, k=512                     indices (all rows) bit-exact, outputs all rows
  MLA int      T=8192, k=2048                    indices (all rows) bit-exact, sampled outputs
  IndexCache   27 layers FSS x 9, T=16384, k=2048  launch counts, S layers reuse F indices
                                                 bit for bit, sampled rows of several layers
  MLA gauss    T=65536, k=2048                   sampled rows, near-tie rule, outputs
  decode       64 x 32768 paged, k=2048          indices (all rows) bit-exact, all outputs
"""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import (check_close_bf16, check_close_f32, check_indices_exact,
                    check_indices_near_ties, check_lse)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.check_device_errors()
    yield
    assert dsa.check_device_errors() == 0


def _cuda(d, names):
    return {n: d[n].cuda() for n in names}


def _prefill_gpu(x, T, k, window_rows=0, lse=False):
    """The benchmark's prefill step: dsa_layer_stack with a single F layer."""
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    l = torch.empty((T, 16), device="cuda") if lse else None
    ws = torch.empty(dsa.layer_stack_workspace_size(T, window_rows) // 4, device="cuda")
    dsa.layer_stack("F", [x], idx, ws, k, G.SCALE_MLA, [out], [l] if lse else None)
    torch.cuda.synchronize()
    return idx, out, l


def _sample_rows(T, k, seed=0, n_random=100):
    r = np.random.default_rng(seed)
    rows = set(range(min(64, T)))
    rows |= set(range(max(0, k - 8), min(T, k + 12)))
    rows |= set(int(v) for v in r.integers(0, T, n_random))
    rows |= set(range(max(0, T - 64), T))
    return np.array(sorted(rows))


def test_tiny_fp32_full_path():
    d = G.tiny_fp32(T=3072)
    T, k = 3072, 512
    x = _cuda(d, ("q_idx", "k_idx", "w", "q", "k", "v"))
    sc = torch.empty((T, T), device="cuda")
    dsa.indexer_scores(x["q_idx"], x["k_idx"], x["w"], sc)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    dsa.topk_select(sc, k, idx)
    out = torch.empty((T, 4, 32), device="cuda")
    lse = torch.empty((T, 4), device="cuda")
    dsa.sparse_mla_fwd(x["q"], x["k"], idx, out, d["scale"], lse=lse, v=x["v"])
    ref_idx = O.prefill_indices(d["q_idx"], d["k_idx"], d["w"], k)
    check_indices_exact(idx, ref_idx, "tiny fp32 indices")
    ref, ref_lse = O.sparse_mha(d["q"], d["k"], d["v"], ref_idx, d["scale"])
    check_close_f32(out, ref, "tiny fp32 attention")
    check_lse(lse, ref_lse, "tiny fp32 lse", tol=1e-4)


@pytest.mark.parametrize("T", [8192, 2057])
def test_mla_prefill_integer_indexer(T):
    """T=8192 is the integer-indexer prefill workload; 2057 is the 'sparse forward longer
    than top-k 2048' length of the DSV2-Lite-IndexCache card's validation list."""
    k = 2048
    d = G.mla_prefill_int(T=T, k=k)
    x = _cuda(d, ("q_idx", "k_idx", "w", "q", "kv"))
    idx, out, lse = _prefill_gpu(x, T, k, lse=True)
    ref_idx = O.prefill_indices(d["q_idx"], d["k_idx"], d["w"], k)
    check_indices_exact(idx, ref_idx, f"T={T} indices")
    rows = _sample_rows(T, k)
    ref, ref_lse = O.sparse_mla_prefill(d["q"][rows], d["kv"], ref_idx[rows], G.SCALE_MLA)
    check_close_bf16(out[torch.from_numpy(rows).cuda()], ref, f"T={T} attention")
    check_lse(lse[torch.from_numpy(rows).cuda()], ref_lse, f"T={T} lse")


def test_mla_prefill_gaussian_T65536_sampled():
    T, k = 65536, 2048
    d = G.mla_prefill_gauss(T=T, k=k)
    x = _cuda(d, ("q_idx", "k_idx", "w", "q", "kv"))
    idx, out, _ = _prefill_gpu(x, T, k)
    rows = _sample_rows(T, k, seed=4, n_random=60)
    g_idx = idx[torch.from_numpy(rows).cuda()].cpu().numpy()
    ref_idx = np.empty_like(g_idx)
    scores = []
    for i, t in enumerate(rows):
        sc = O.indexer_scores_prefill(d["q_idx"], d["k_idx"], d["w"], int(t), 1, int(t) + 1)
        ref_idx[i] = O.topk(sc, [int(t) + 1], k)[0]
        scores.append(sc[0])
    swaps = check_indices_near_ties(g_idx, ref_idx, scores, [int(t) + 1 for t in rows],
                                    "T=65536 indices")
    assert swaps <= len(rows)  # near-ties are rare with Gaussian scores
    # attention checked with the GPU's own indices (they may swap near-ties)
    ref, _ = O.sparse_mla_prefill(d["q"][rows], d["kv"], g_idx, G.SCALE_MLA)
    check_close_bf16(out[torch.from_numpy(rows).cuda()], ref, "T=65536 attention")


def test_index_cache_stack_fss_x9():
    T, k, pattern = 16384, 2048, "FSS" * 9
    st = G.layer_stack(T=T, pattern=pattern, k=k)
    layers = [_cuda(L, [n for n in ("q", "kv", "q_idx", "k_idx", "w") if n in L])
              for L in st["layers"]]
    outs = [torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda") for _ in layers]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.layer_stack_workspace_size(T) // 4, device="cuda")
    nwin = -(-T // (dsa.layer_stack_workspace_size(T) // (4 * T)))
    dsa.reset_launch_counts()
    dsa.layer_stack(pattern, layers, idx, ws, k, G.SCALE_MLA, outs)
    torch.cuda.synchronize()
    # IndexCache: indexer and top-k run only in the 9 F layers; attention in all 27
    assert dsa.launch_count(0) == 9 * nwin
    assert dsa.launch_count(1) == 9 * nwin
    assert dsa.launch_count(2) == 27
    # the buffer now holds the last F layer's (layer 24) indices: exact on every row
    rows = _sample_rows(T, k, seed=7, n_random=40)
    L24 = st["layers"][24]
    g_idx = idx.cpu().numpy()
    check_indices_exact(g_idx, O.prefill_indices(L24["q_idx"], L24["k_idx"], L24["w"], k),
                        "layer 24 indices, all rows")
    # every F layer l: a separate dsa_indexer_scores + dsa_topk_select of its inputs, fed to
    # separate attention calls of layers l, l+1, l+2, reproduces the stack's outputs bit
    # for bit (the S layers used exactly the F layer's indices, and nothing else)
    ld = (T + 3) // 4 * 4
    sc = torch.empty((4096, ld), device="cuda")
    for f in range(0, 27, 3):
        idx_f = torch.empty((T, k), dtype=torch.int32, device="cuda")
        for q0 in range(0, T, 4096):
            dsa.indexer_scores(layers[f]["q_idx"], layers[f]["k_idx"], layers[f]["w"], sc, q0,
                               4096)
            dsa.topk_select(sc, k, idx_f[q0:q0 + 4096], q_begin=q0, rows=4096)
        for l in (f, f + 1, f + 2):
            ref_out = torch.empty_like(outs[l])
            dsa.sparse_mla_fwd(layers[l]["q"], layers[l]["kv"], idx_f, ref_out, G.SCALE_MLA)
            torch.cuda.synchronize()
            assert torch.equal(ref_out.view(torch.int16), outs[l].view(torch.int16)), l
        if f == 24:
            assert torch.equal(idx_f, idx)
    # sampled rows of F and S layers against the oracle (F layer 0 -> layers 0, 1, 2)
    L0 = st["layers"][0]
    ref_idx0 = np.stack([O.prefill_indices(L0["q_idx"], L0["k_idx"], L0["w"], k,
                                           q_begin=int(t), rows=1)[0] for t in rows])
    for l in (0, 2, 24, 26):
        ref_i = ref_idx0 if l < 3 else np.stack([g_idx[t] for t in rows])
        ref, _ = O.sparse_mla_prefill(st["layers"][l]["q"][rows], st["layers"][l]["kv"], ref_i,
                                      G.SCALE_MLA)
        check_close_bf16(outs[l][torch.from_numpy(rows).cuda()], ref, f"stack layer {l}")


def test_decode_full():
    B, L, k = 64, 32768, 2048
    d = G.mla_decode(B=B, L=L, k=k)
    x = _cuda(d, ("q_idx", "w", "k_idx_pool", "q", "kv_pool", "page_table", "seq_lens"))
    sc = torch.empty((B, L), device="cuda")
    dsa.indexer_scores(x["q_idx"], x["k_idx_pool"], x["w"], sc, page_table=x["page_table"],
                       seq_lens=x["seq_lens"])
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    dsa.topk_select(sc, k, idx, row_len=x["seq_lens"], max_len=L)
    out = torch.empty((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 16), device="cuda")
    ws = torch.empty(dsa.sparse_mla_workspace_size(B, k, decode=True) // 4 + 4, device="cuda")
    dsa.sparse_mla_fwd(x["q"], x["kv_pool"], idx, out, G.SCALE_MLA, lse=lse,
                       page_table=x["page_table"], seq_lens=x["seq_lens"], workspace=ws)
    torch.cuda.synchronize()
    ref_sc = O.indexer_scores_decode(d["q_idx"], d["k_idx_pool"], d["w"], d["page_table"],
                                     d["seq_lens"])
    ref_idx = O.topk(ref_sc, d["seq_lens"].numpy(), k)
    check_indices_exact(idx, ref_idx, "decode indices")
    ref, ref_lse = O.sparse_mla_decode(d["q"], d["kv_pool"], d["page_table"], ref_idx,
                                       G.SCALE_MLA)
    check_close_bf16(out, ref, "decode attention")
    check_lse(lse, ref_lse, "decode lse")
