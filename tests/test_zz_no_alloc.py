"""The allocation-free decode entry point (dsa_sparse_mla_decode_noalloc).

Callers that cannot allocate device memory where they decode (a fixed memory pool, an
allocation-free serving loop) use this entry point: it keeps the per-split partials in a
library-owned device array instead of a caller workspace.  This file checks, through the
C ABI, that two calls in a row -- on different inputs, so the second reuses the array
the first wrote -- agree with the workspace-based dsa_sparse_mla_fwd decode path within
the bf16 tolerance the other tests use.  It is collected last so that a failure here
does not hide the other tests' results.
"""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import _lib
from sparse_attention_17_b200 import inputs as G
from parity import check_close_bf16, check_lse

pytestmark = pytest.mark.gpu


def _case(seed, lens, k):
    d = G.mla_decode(B=len(lens), L=max(lens), seed=seed, seq_lens=lens)
    r = np.random.default_rng(seed)
    idx = np.full((len(lens), k), -1, dtype=np.int32)
    for b, n in enumerate(lens):
        m = min(n, k)
        idx[b, :m] = np.sort(r.choice(n, m, replace=False))
    cu = {n: d[n].cuda() for n in ("q", "kv_pool", "page_table", "seq_lens")}
    cu["idx"] = torch.from_numpy(idx).cuda()
    return cu


def _noalloc(lib, c, out, lse):
    q, kv, pt = c["q"], c["kv_pool"], c["page_table"]
    st = lib.dsa_sparse_mla_decode_noalloc(
        q.shape[0], 16, 576, 512, G.SCALE_MLA, q.data_ptr(), kv.data_ptr(),
        kv.shape[0] * kv.shape[1], pt.data_ptr(), pt.shape[1], kv.shape[1],
        c["seq_lens"].data_ptr(), c["idx"].data_ptr(), c["idx"].shape[1], c["idx"].shape[1],
        out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == _lib.DSA_OK, lib.dsa_status_string(st)


def _with_workspace(c):
    B, k = c["q"].shape[0], c["idx"].shape[1]
    ws = torch.empty(dsa.sparse_mla_workspace_size(B, k, decode=True) // 4 + 4, device="cuda")
    out = torch.empty((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 16), device="cuda")
    dsa.sparse_mla_fwd(c["q"], c["kv_pool"], c["idx"], out, G.SCALE_MLA, lse=lse,
                       page_table=c["page_table"], seq_lens=c["seq_lens"], workspace=ws)
    return out, lse


def test_noalloc_decode_matches_workspace_path_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = dsa.load()
    cases = [_case(21, [3000, 1500, 2048, 5000, 64, 2049], 2048),
             _case(22, [700, 9000, 4100], 512)]
    for c in cases:  # two calls in a row; the second reuses the array the first wrote
        B = c["q"].shape[0]
        out = torch.full((B, 16, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 16), float("nan"), device="cuda")
        _noalloc(lib, c, out, lse)
        ref_out, ref_lse = _with_workspace(c)
        torch.cuda.synchronize()
        check_close_bf16(out, ref_out.float().cpu().numpy(), "no-alloc decode vs workspace")
        check_lse(lse, ref_lse.cpu().numpy(), "no-alloc decode lse")
    assert dsa.check_device_errors() == 0


def test_noalloc_rejects_too_many_sequences_before_launch():
    lib = dsa.load()
    st = lib.dsa_sparse_mla_decode_noalloc(512, 16, 576, 512, 0.1, 16, 16, 64, 16, 1, 64, 16,
                                           16, 64, 64, 16, 16, None)
    assert st == _lib.DSA_ERR_UNSUPPORTED
