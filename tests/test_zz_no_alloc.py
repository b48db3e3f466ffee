"""The allocation-free decode entry point (dsa_sparse_mla_decode_noalloc).

Callers that cannot allocate device memory where they decode (a fixed memory pool, an
allocation-free serving loop) use this entry point: it keeps the per-split partials in a
library-owned device array instead of a caller workspace.  This file checks, through the
C ABI, two calls in a row -- on different inputs, so the second reuses the array the
first wrote -- against the workspace-based dsa_sparse_mla_fwd decode path (bit for bit:
both run the same kernels with the same split count) and against the CPU oracle, and a
batch of 300 sequences, where the array holds fewer splits per sequence than the
workspace path takes, against both within the bf16 tolerance.  It is collected last so
that a failure here does not hide the other tests' results.
"""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import _lib
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import check_close_bf16, check_lse

pytestmark = pytest.mark.gpu


def _case(seed, lens, k):
    d = G.mla_decode(B=len(lens), L=max(lens), seed=seed, seq_lens=lens)
    r = np.random.default_rng(seed)
    idx = np.full((len(lens), k), -1, dtype=np.int32)
    for b, n in enumerate(lens):
        m = min(n, k)
        idx[b, :m] = np.sort(r.choice(n, m, replace=False))
    host = {n: d[n] for n in ("q", "kv_pool", "page_table", "seq_lens")}
    host["idx"] = idx
    return host


def _many_sequences_case(seed, B, k):
    """B sequences of 2049..3000 tokens over a shared pool of 2B pages: each page table is
    a random draw of pool pages (sequences may share pages; the kernels only read them)."""
    d = G.mla_decode(B=B, L=128, seed=seed)  # q [B,16,576] and a pool of 2B 64-token pages
    r = np.random.default_rng(seed)
    lens = r.integers(2049, 3001, B)
    max_pages = (int(lens.max()) + 63) // 64
    pt = r.integers(0, d["kv_pool"].shape[0], (B, max_pages)).astype(np.int32)
    idx = np.full((B, k), -1, dtype=np.int32)
    for b, n in enumerate(lens):
        idx[b] = np.sort(r.choice(int(n), k, replace=False))
    return {"q": d["q"], "kv_pool": d["kv_pool"], "page_table": torch.from_numpy(pt),
            "seq_lens": torch.from_numpy(lens.astype(np.int32)), "idx": idx}


def _cuda(host):
    c = {n: host[n].cuda() for n in ("q", "kv_pool", "page_table", "seq_lens")}
    c["idx"] = torch.from_numpy(host["idx"]).cuda()
    return c


def _noalloc(lib, c, out, lse):
    q, kv, pt = c["q"], c["kv_pool"], c["page_table"]
    st = lib.dsa_sparse_mla_decode_noalloc(
        q.shape[0], 16, 576, 512, G.SCALE_MLA, q.data_ptr(), kv.data_ptr(),
        kv.shape[0] * kv.shape[1], pt.data_ptr(), pt.shape[1], kv.shape[1],
        c["seq_lens"].data_ptr(), c["idx"].data_ptr(), c["idx"].shape[1], c["idx"].shape[1],
        out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == _lib.DSA_OK, (lib.dsa_status_string(st), lib.dsa_last_error())


def _with_workspace(c):
    B, k = c["q"].shape[0], c["idx"].shape[1]
    ws = torch.empty(dsa.sparse_mla_workspace_size(B, k, decode=True) // 4 + 4, device="cuda")
    out = torch.empty((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 16), device="cuda")
    dsa.sparse_mla_fwd(c["q"], c["kv_pool"], c["idx"], out, G.SCALE_MLA, lse=lse,
                       page_table=c["page_table"], seq_lens=c["seq_lens"], workspace=ws)
    return out, lse


def _oracle(host):
    return O.sparse_mla_decode(host["q"], host["kv_pool"], host["page_table"], host["idx"],
                               G.SCALE_MLA)


def _run_noalloc(lib, c):
    B = c["q"].shape[0]
    out = torch.full((B, 16, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, 16), float("nan"), device="cuda")
    _noalloc(lib, c, out, lse)
    return out, lse


def test_noalloc_decode_matches_workspace_path_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = dsa.load()
    cases = [_case(21, [3000, 1500, 2048, 5000, 64, 2049], 2048),
             _case(22, [700, 9000, 4100], 512)]
    for host in cases:  # two calls in a row; the second reuses the array the first wrote
        c = _cuda(host)
        out, lse = _run_noalloc(lib, c)
        ref_out, ref_lse = _with_workspace(c)
        torch.cuda.synchronize()
        # same kernels, same split count: identical bits
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(lse, ref_lse)
        o_ref, o_lse = _oracle(host)
        check_close_bf16(out, o_ref, "no-alloc decode vs oracle")
        check_lse(lse, o_lse, "no-alloc decode lse vs oracle")
    assert dsa.check_device_errors() == 0


def test_noalloc_decode_many_sequences_fewer_splits():
    """300 sequences need more (sequence, split) units than the array holds at the
    workspace path's split count, so the entry point takes fewer splits per sequence: the
    result moves within rounding, and both paths stay within the gate of the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = dsa.load()
    host = _many_sequences_case(23, 300, 2048)
    c = _cuda(host)
    out, lse = _run_noalloc(lib, c)
    ref_out, ref_lse = _with_workspace(c)
    torch.cuda.synchronize()
    ws_units = dsa.sparse_mla_workspace_size(300, 2048, decode=True) // (16 * 513 * 4)
    assert ws_units > 511  # the workspace path splits more than the array allows
    check_close_bf16(out, ref_out.float().cpu().numpy(), "capped no-alloc vs workspace")
    check_lse(lse, ref_lse.cpu().numpy(), "capped no-alloc lse vs workspace")
    o_ref, o_lse = _oracle(host)
    check_close_bf16(out, o_ref, "capped no-alloc vs oracle")
    check_lse(lse, o_lse, "capped no-alloc lse vs oracle")
    check_close_bf16(ref_out, o_ref, "workspace decode vs oracle")
    assert dsa.check_device_errors() == 0


def test_noalloc_rejects_too_many_sequences_before_launch():
    lib = dsa.load()
    st = lib.dsa_sparse_mla_decode_noalloc(512, 16, 576, 512, 0.1, 16, 16, 64, 16, 1, 64, 16,
                                           16, 64, 64, 16, 16, None)
    assert st == _lib.DSA_ERR_UNSUPPORTED
    assert b"at most 511 sequences" in lib.dsa_last_error()
    # a later successful argument check clears the message
    st = lib.dsa_sparse_mla_decode_noalloc(0, 16, 576, 512, 0.1, 16, 16, 64, 16, 1, 64, 16,
                                           16, 64, 64, 16, 16, None)
    assert st == _lib.DSA_OK and lib.dsa_last_error() == b""
