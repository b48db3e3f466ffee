"""GPU parity of dsa_index_varlen: a batch of independent prefill sequences packed along
the token axis (unequal lengths, empty and one-token sequences, gaps standing for left
padding), bit for bit against the oracle on integer indexer inputs, then the sparse MLA
of the whole packed batch with those indices against the oracle."""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import check_close_bf16, check_indices_exact, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.check_device_errors()
    yield
    assert dsa.check_device_errors() == 0


def _run(d, starts, lens, k, window_rows):
    N = d["q_idx"].shape[0]
    idx = torch.full((N, k), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.index_varlen_workspace_size(max(lens), window_rows) // 4 + 64,
                     device="cuda")
    dsa.index_varlen(dev(d["q_idx"]), dev(d["k_idx"]), dev(d["w"]), starts, lens, k, idx, ws)
    torch.cuda.synchronize()
    ref = O.prefill_indices_varlen(d["q_idx"], d["k_idx"], d["w"], starts, lens, k, fill=-7)
    check_indices_exact(idx, ref, "varlen indices")
    return idx, ref


@pytest.mark.parametrize("window_rows", [0, 700])
def test_packed_batch_exact(window_rows):
    lens = [3000, 1, 2048, 2049, 0, 5000, 700, 16]
    gaps = [0, 5, 0, 37, 3, 0, 11, 2]
    starts, pos = [], 0
    for g, L in zip(gaps, lens):
        pos += g
        starts.append(pos)
        pos += L
    N = pos + 9
    d = G.indexer_int(N, 31)
    _run(d, starts, lens, 2048, window_rows)


def test_left_padded_batch_then_attention():
    """B=3 rows of T=2600 tokens, left-padded by 0 / 100 / 1999 tokens: sequence b is
    rows b*T + pad_b .. (b+1)*T - 1.  The sparse MLA of the packed batch then reads the
    packed indices directly."""
    B, T, k = 3, 2600, 2048
    pads = [0, 100, 1999]
    starts = [b * T + p for b, p in enumerate(pads)]
    lens = [T - p for p in pads]
    N = B * T
    d = G.indexer_int(N, 32)
    d.update(G.mla_layer(N, 33))
    idx, ref = _run(d, starts, lens, k, 0)
    out = torch.zeros((N, 16, 512), dtype=torch.bfloat16, device="cuda")
    dsa.sparse_mla_fwd(dev(d["q"]), dev(d["kv"]), idx.clamp(min=-1), out, G.SCALE_MLA)
    rows = np.concatenate([np.arange(s, s + L) for s, L in zip(starts, lens)])
    sample = rows[np.random.default_rng(3).choice(len(rows), 300, replace=False)]
    sample = np.sort(np.r_[sample, starts, [s + L - 1 for s, L in zip(starts, lens)]])
    ref_out, _ = O.sparse_mla_prefill(d["q"][sample], d["kv"], ref[sample], G.SCALE_MLA)
    check_close_bf16(out[torch.from_numpy(sample).cuda()], ref_out, "varlen attention")
