"""GPU tests of dsa_index_select (indexer + top-k without dense score rows).

Its result must be identical to dsa_indexer_scores followed by dsa_topk_select on the same
rows: both take the same tensor-core scores and the same selection rule, so the indices
are compared bit for bit -- on integer inputs (massive ties), on Gaussian inputs with rows
long enough to use the sampled thresholds, across several windows, and on rows built so
that the sampled threshold misleads and the dense fallback has to settle them.  One case
is also checked against the CPU oracle directly.
"""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import check_indices_exact

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.check_device_errors()
    yield
    assert dsa.check_device_errors() == 0


def _dense(q_idx, k_idx, w, k, q_begin, rows):
    S = k_idx.shape[0]
    ld = (S + 3) // 4 * 4
    sc = torch.empty((rows, ld), device="cuda")
    idx = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    dsa.indexer_scores(q_idx, k_idx, w, sc, q_begin, rows)
    dsa.topk_select(sc, k, idx, q_begin=q_begin, rows=rows)
    return idx


def _fused(q_idx, k_idx, w, k, q_begin, rows, window=None):
    S = k_idx.shape[0]
    ws_bytes = dsa.index_select_workspace_size(window or rows, S)
    ws = torch.empty(ws_bytes // 4 + 64, dtype=torch.float32, device="cuda")
    off = (-ws.data_ptr()) % 256 // 4  # 256-byte aligned view
    ws = ws[off:off + ws_bytes // 4]
    idx = torch.full((rows, k), -9, dtype=torch.int32, device="cuda")
    dsa.index_select(q_idx, k_idx, w, idx, k, ws, q_begin=q_begin, rows=rows)
    torch.cuda.synchronize()
    return idx


def _cuda(d):
    return d["q_idx"].cuda(), d["k_idx"].cuda(), d["w"].cuda()


@pytest.mark.parametrize("T,q_begin,rows", [(8192, 0, 8192), (3000, 1000, 2000)])
def test_integer_rows_without_sampling(T, q_begin, rows):
    """Rows of at most 8192 keys: every key is a candidate."""
    q_idx, k_idx, w = _cuda(G.indexer_int(T, 5))
    k = 2048
    a = _fused(q_idx, k_idx, w, k, q_begin, rows)
    b = _dense(q_idx, k_idx, w, k, q_begin, rows)
    assert torch.equal(a, b)


def test_integer_rows_with_sampling_and_windows():
    """T=16384 integer inputs (ties everywhere): rows past 8192 keys use the sampled
    thresholds and the tie bitmaps; four windows."""
    T, k = 16384, 2048
    q_idx, k_idx, w = _cuda(G.indexer_int(T, 6))
    a = _fused(q_idx, k_idx, w, k, 0, T, window=4096)
    b = _dense(q_idx, k_idx, w, k, 0, T)
    assert torch.equal(a, b)


@pytest.mark.parametrize("k", [2048, 512])
def test_gaussian_rows_with_sampling(k):
    T = 24576
    q_idx, k_idx, w = _cuda(G.indexer_gauss(T, 7))
    q_begin, rows = 8000, T - 8000
    a = _fused(q_idx, k_idx, w, k, q_begin, rows, window=2048)
    b = _dense(q_idx, k_idx, w, k, q_begin, rows)
    assert torch.equal(a, b)


def test_misleading_sample_falls_back_to_dense():
    """Keys of the sampled tiles (one 128-key tile in 16) score far above the others, so
    each row's threshold lands among them and too few keys pass it: those rows must come
    out of the dense fallback, identical to the dense path."""
    T, k = 20480, 2048
    d = G.indexer_gauss(T, 8)
    s = torch.arange(T)
    sampled = (s // 128) % 16 == 0
    d["k_idx"][sampled] = (d["k_idx"][sampled].float() * 4).to(torch.bfloat16)
    q_idx, k_idx, w = _cuda(d)
    a = _fused(q_idx, k_idx, w, k, 0, T, window=4096)
    b = _dense(q_idx, k_idx, w, k, 0, T)
    assert torch.equal(a, b)


def test_misleading_sample_in_narrow_windows():
    """The same planted keys with 64-row windows: each window's fallback top-k is a launch
    of few rows, which takes the cluster path (two CTAs per row) with a row mask."""
    T, k = 12288, 2048
    d = G.indexer_gauss(T, 10)
    s = torch.arange(T)
    sampled = (s // 128) % 16 == 0
    d["k_idx"][sampled] = (d["k_idx"][sampled].float() * 4).to(torch.bfloat16)
    q_idx, k_idx, w = _cuda(d)
    q_begin, rows = T - 256, 256
    a = _fused(q_idx, k_idx, w, k, q_begin, rows, window=64)
    b = _dense(q_idx, k_idx, w, k, q_begin, rows)
    assert torch.equal(a, b)


def test_against_oracle_sampled_rows():
    """T=12000 integer inputs, rows past the no-sample bound checked against the oracle."""
    T, k = 12000, 2048
    d = G.indexer_int(T, 9)
    q_idx, k_idx, w = _cuda(d)
    a = _fused(q_idx, k_idx, w, k, 0, T).cpu().numpy()
    for t in (8192, 9000, 11999):
        ref = O.prefill_indices(d["q_idx"], d["k_idx"], d["w"], k, q_begin=t, rows=1)
        check_indices_exact(a[t:t + 1], ref, f"row {t}")
