"""The whole prefill path (indexer -> top-k -> sparse MLA, through dsa_layer_stack with one
'F' layer) at the edge sizes of the test plan: sequence lengths around the 64- and
128-row tiles, around k = 2048 (including the 2057-token forward the IndexCache card
reports) and a ragged 4099; top-512 and top-2048.  Integer indexer inputs: indices
bit-exact against the oracle, attention within the bf16 gate."""
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


@pytest.mark.parametrize("k", [512, 2048])
@pytest.mark.parametrize("T", [1, 63, 64, 127, 128, 129, 2047, 2048, 2049, 2057, 4099])
def test_prefill_path_edge_sizes(T, k):
    d = G.mla_prefill_int(T=T, k=k, seed=T + k)
    cuda = {n: d[n].cuda() for n in ("q_idx", "k_idx", "w", "q", "kv")}
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dsa.layer_stack_workspace_size(T) // 4 + 4, device="cuda")
    dsa.layer_stack("F", [cuda], idx, ws, k, G.SCALE_MLA, [out])
    torch.cuda.synchronize()
    ref_idx = O.prefill_indices(d["q_idx"], d["k_idx"], d["w"], k)
    check_indices_exact(idx, ref_idx, f"T={T} k={k}")
    rows = np.unique(np.r_[0:min(T, 40), max(0, T - 40):T,
                           np.random.default_rng(T).integers(0, T, 40)])
    ref, _ = O.sparse_mla_prefill(d["q"][rows], d["kv"], ref_idx[rows], G.SCALE_MLA)
    check_close_bf16(out[torch.from_numpy(rows).cuda()], ref, f"T={T} k={k}")
