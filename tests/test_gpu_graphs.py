"""The library's calls inside CUDA graphs (the pages' serving stacks run the model under
full CUDA graphs): every call is asynchronous on the caller's stream, allocates nothing
and never synchronises, so a captured sequence of calls must replay to bit-identical
results -- also after new inputs are copied into the captured buffers."""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
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


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm-up outside the capture (first-use attributes, lazy loading)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def test_layer_stack_graph_replay_bit_exact():
    T, k, pattern = 4096, 2048, "FSS" * 3
    st = G.layer_stack(T=T, pattern=pattern, k=k)
    layers = [{n: v.cuda() for n, v in L.items()} for L in st["layers"]]
    ws = torch.empty(dsa.layer_stack_workspace_size(T, 1024) // 4, device="cuda")

    def eager(lays):
        outs = [torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda") for _ in lays]
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        dsa.layer_stack(pattern, lays, idx, ws, k, G.SCALE_MLA, outs)
        torch.cuda.synchronize()
        return outs, idx

    ref_outs, ref_idx = eager(layers)
    outs = [torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda") for _ in layers]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    g = _capture(lambda: dsa.layer_stack(pattern, layers, idx, ws, k, G.SCALE_MLA, outs))
    for o in outs:
        o.zero_()
    idx.fill_(-5)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx)
    for a, b in zip(outs, ref_outs):
        assert torch.equal(_bits(a), _bits(b))
    # new inputs in the captured buffers: the replay follows them
    st2 = G.layer_stack(T=T, pattern=pattern, k=k, mla_seed_base=3000, indexer_seed_base=4000)
    for L, L2 in zip(layers, st2["layers"]):
        for n in L:
            L[n].copy_(L2[n])
    ref2_outs, ref2_idx = eager(layers)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx, ref2_idx) and not torch.equal(ref2_idx, ref_idx)
    for a, b in zip(outs, ref2_outs):
        assert torch.equal(_bits(a), _bits(b))
    # the replay against the oracle: the last F layer's indices on every row, and sampled
    # rows of an F and an S layer computed from the oracle's indices
    L6 = st2["layers"][6]
    ref_i6 = O.prefill_indices(L6["q_idx"], L6["k_idx"], L6["w"], k)
    check_indices_exact(idx, ref_i6, "graph replay: layer 6 indices")
    rows = np.r_[0:8, 2040:2056, T - 8:T]
    for l in (6, 8):
        ref, _ = O.sparse_mla_prefill(st2["layers"][l]["q"][rows], st2["layers"][l]["kv"],
                                      ref_i6[rows], G.SCALE_MLA)
        check_close_bf16(outs[l][torch.from_numpy(rows).cuda()], ref, f"graph replay layer {l}")


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_step_graph_replay_bit_exact(fp8):
    """Decode indexer + top-k + sparse MLA (split keys, merge) captured as one graph."""
    B, L, k = 8, 5000, 2048
    d = (G.mla_decode_fp8 if fp8 else G.mla_decode)(B=B, L=L, k=k)
    x = {n: d[n].cuda() for n in ("q_idx", "w", "k_idx_pool", "q", "kv_pool", "page_table",
                                   "seq_lens")}
    scores = torch.empty((B, (L + 3) // 4 * 4), device="cuda")
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dsa.sparse_mla_workspace_size(B, k, decode=True) // 4 + 4, device="cuda")

    def step():
        dsa.indexer_scores(x["q_idx"], x["k_idx_pool"], x["w"], scores,
                           page_table=x["page_table"], seq_lens=x["seq_lens"])
        dsa.topk_select(scores, k, idx, row_len=x["seq_lens"], max_len=L)
        if fp8:
            dsa.sparse_mla_fp8_fwd(x["q"], x["kv_pool"], d["kv_scale"], idx, out, G.SCALE_MLA,
                                   page_table=x["page_table"], seq_lens=x["seq_lens"],
                                   workspace=ws)
        else:
            dsa.sparse_mla_fwd(x["q"], x["kv_pool"], idx, out, G.SCALE_MLA,
                               page_table=x["page_table"], seq_lens=x["seq_lens"], workspace=ws)

    step()
    torch.cuda.synchronize()
    ref_idx, ref_out = idx.clone(), out.clone()
    g = _capture(step)
    idx.fill_(-3)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(_bits(out), _bits(ref_out))
    # the replay against the oracle: exact indices and the attention within the gate
    o_sc = O.indexer_scores_decode(d["q_idx"], d["k_idx_pool"], d["w"], d["page_table"],
                                   d["seq_lens"])
    o_idx = O.topk(o_sc, d["seq_lens"].numpy(), k)
    check_indices_exact(idx, o_idx, "decode graph replay indices")
    if fp8:
        o_out, o_lse = O.sparse_mla_fp8_decode(d["q"], d["kv_pool"], d["kv_scale"],
                                               d["page_table"], o_idx, G.SCALE_MLA)
    else:
        o_out, o_lse = O.sparse_mla_decode(d["q"], d["kv_pool"], d["page_table"], o_idx,
                                           G.SCALE_MLA)
    check_close_bf16(out, o_out, "decode graph replay attention")
