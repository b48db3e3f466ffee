"""dsa_layer_stack with F/S patterns other than FSS x n, against the oracle's IndexCache
loop (vLLM docs, IndexCache, "How It Works": an F layer computes and stores the top-k
indices, an S layer reuses those of the nearest preceding F layer).

Patterns: the 61-layer index_topk_pattern printed in the docs' "Configuration Examples"
(tests/golden), index_topk_freq = 4 over 9 layers ("Configuration Reference"), all-F, and
one F followed by a long run of S layers.  At T = 1100, k = 512, with 256-row index
windows: every F layer's indices are exact on every row (integer indexer inputs), every
layer's output is within the bf16 gate on sampled rows, and the indexer and top-k launch
only for F layers."""
import json
import os

import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import check_close_bf16, check_indices_exact

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _pattern(name):
    if name == "printed61":
        with open(os.path.join(GOLD, "index_topk_pattern_61.json")) as f:
            return json.load(f)["pattern"]
    if name == "freq4x9":
        return dsa.pattern_from_freq(4, 9)
    if name == "FFF":
        return "FFF"
    return "F" + "S" * 11


@pytest.fixture(autouse=True)
def _clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.check_device_errors()
    yield
    assert dsa.check_device_errors() == 0


@pytest.mark.parametrize("name", ["printed61", "freq4x9", "FFF", "long_S"])
def test_layer_stack_pattern_against_oracle(name):
    pattern = _pattern(name)
    if name == "freq4x9":
        assert pattern == O.pattern_from_freq(4, 9) == "FSSSFSSSF"
    T, k, rw = 1100, 512, 256
    st = G.layer_stack(T=T, pattern=pattern, k=k)
    layers = [{n: v.cuda() for n, v in L.items()} for L in st["layers"]]
    outs = [torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda") for _ in layers]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.layer_stack_workspace_size(T, rw) // 4, device="cuda")
    nwin = -(-T // rw)
    dsa.reset_launch_counts()
    dsa.layer_stack(pattern, layers, idx, ws, k, G.SCALE_MLA, outs)
    torch.cuda.synchronize()
    nF = pattern.count("F")
    assert dsa.launch_count(dsa.KERNEL_INDEXER) == nF * nwin
    assert dsa.launch_count(dsa.KERNEL_TOPK) == nF * nwin
    assert dsa.launch_count(dsa.KERNEL_ATTENTION) == len(pattern)
    rows = np.r_[0:8, 505:520, 700:704, T - 8:T]
    rows_t = torch.from_numpy(rows).cuda()
    cur = None
    for l, ch in enumerate(pattern):
        L = st["layers"][l]
        if ch == "F":
            cur = O.prefill_indices(L["q_idx"], L["k_idx"], L["w"], k)
            # F layer l+1..: the GPU's buffer for this layer is checked through the next
            # layers' outputs; the buffer itself ends with the last F layer's indices
        ref, _ = O.sparse_mla_prefill(L["q"][rows], L["kv"], cur[rows], G.SCALE_MLA)
        check_close_bf16(outs[l][rows_t], ref, f"{name} layer {l} ({ch})")
    check_indices_exact(idx, cur, f"{name}: index buffer after the last F layer")


def test_each_f_layer_indices_exact_in_a_mixed_pattern():
    """Every F layer's indices, on every row: the stack run layer by layer (prefixes of
    the pattern), each time comparing the buffer with that F layer's oracle indices."""
    pattern = "FSFFSSF"
    T, k = 1100, 512
    st = G.layer_stack(T=T, pattern=pattern, k=k)
    layers = [{n: v.cuda() for n, v in L.items()} for L in st["layers"]]
    ws = torch.empty(dsa.layer_stack_workspace_size(T, 512) // 4, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    for l, ch in enumerate(pattern):
        if ch != "F":
            continue
        outs = [torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
                for _ in range(l + 1)]
        dsa.layer_stack(pattern[:l + 1], layers[:l + 1], idx, ws, k, G.SCALE_MLA, outs)
        torch.cuda.synchronize()
        L = st["layers"][l]
        check_indices_exact(idx, O.prefill_indices(L["q_idx"], L["k_idx"], L["w"], k),
                            f"F layer {l}")
