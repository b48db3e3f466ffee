"""The largest sizes the C ABI accepts, end to end on the GPU against the oracle: decode
rows of 262144 keys (the top-k limit) through a 4096-entry page table, integer indexer
inputs so that every score is exact, then the top-2048 of those rows; and top-k rows of
262144 scores with massive ties and with distinct Gaussian values."""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import check_indices_exact, dev

pytestmark = pytest.mark.gpu

MAX_LEN = 262144


@pytest.fixture(autouse=True)
def _clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.check_device_errors()
    yield
    assert dsa.check_device_errors() == 0


def test_decode_indexer_and_topk_at_max_length():
    lens = [MAX_LEN, 200003]
    B, k = len(lens), 2048
    d = G.mla_decode(B=B, L=MAX_LEN, seed=77, seq_lens=lens)
    sc = torch.full((B, MAX_LEN), float("nan"), device="cuda")
    dsa.indexer_scores(dev(d["q_idx"]), dev(d["k_idx_pool"]), dev(d["w"]), sc,
                       page_table=dev(d["page_table"]), seq_lens=dev(d["seq_lens"]))
    ref = O.indexer_scores_decode(d["q_idx"], d["k_idx_pool"], d["w"], d["page_table"],
                                  d["seq_lens"], S=MAX_LEN)
    g = sc.cpu().numpy().astype(np.float64)
    for b, n in enumerate(lens):
        assert np.array_equal(g[b, :n], ref[b, :n]), b
    idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    dsa.topk_select(sc, k, idx, row_len=dev(d["seq_lens"]), max_len=MAX_LEN)
    check_indices_exact(idx, O.topk(ref, np.array(lens), k), "max-length decode rows")


@pytest.mark.parametrize("kind", ["ties", "gauss"])
def test_topk_rows_at_max_length(kind):
    r = np.random.default_rng(5 if kind == "ties" else 6)
    rows, k = 3, 2048
    if kind == "ties":
        sc = r.integers(0, 7, (rows, MAX_LEN)).astype(np.float32)
    else:
        sc = r.normal(size=(rows, MAX_LEN)).astype(np.float32)
    n_valid = [MAX_LEN, MAX_LEN - 1, 131077]
    idx = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    dsa.topk_select(torch.from_numpy(sc).cuda(), k, idx,
                    row_len=torch.tensor(n_valid, dtype=torch.int32, device="cuda"),
                    max_len=MAX_LEN)
    check_indices_exact(idx, O.topk(sc.astype(np.float64), n_valid, k), f"max-length {kind}")
