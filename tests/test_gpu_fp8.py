"""GPU parity of the fp8 (E4M3) latent cache.

* dsa_latent_quantize_fp8 against the oracle's encoder, bit for bit (the quotient is the
  fp32 IEEE division on both sides, then round-to-nearest-even with finite saturation);
  the inputs include exact midpoints between codes, saturating and underflowing values,
  signed zeros and a length that is not a multiple of the kernel's 8-element step.
* dsa_sparse_mla_fp8_fwd (prefill and paged decode) against the oracle's attention over
  kv_scale * E4M3(code), with the same bf16 output gate as the bf16 path: the products of
  f16-widened codes and the f16 query are exact in fp32, the probabilities are rounded to
  f16 (finer than the bf16 of the bf16 path) and the output to bf16.
"""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import check_close_bf16, check_lse, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.check_device_errors()
    yield
    assert dsa.check_device_errors() == 0


def _special_bf16(kv_scale):
    pos = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    vals = np.concatenate([mids, -mids, pos, [0.0, -0.0, 448.0, 464.0, 480.0, 512.0, -1024.0,
                                              2.0 ** 20, 2.0 ** -12, -(2.0 ** -11), 2.0 ** -10]])
    # scale into the cache's range; keep only values that bf16 holds exactly
    x = torch.tensor(vals * kv_scale, dtype=torch.float64)
    b = x.to(torch.bfloat16)
    return b[b.double() == x]


@pytest.mark.parametrize("kv_scale", [2.0 ** -7, 0.0123, 1.0])
def test_latent_quantize_bit_exact(kv_scale):
    g = torch.Generator().manual_seed(5)
    n = 576 * 173 + 5
    c = (torch.randn(n, generator=g) * 0.5).to(torch.bfloat16)
    sp = _special_bf16(kv_scale)
    c[:sp.numel()] = sp
    dst = torch.full((n,), 0xAA, dtype=torch.uint8, device="cuda")
    dsa.latent_quantize_fp8(dev(c), kv_scale, dst)
    ref = O.latent_quantize_fp8(c, kv_scale)
    got = dst.cpu().numpy()
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (bad[:8], c[bad[:8]], got[bad[:8]], ref[bad[:8]])


def _causal_random_idx(T, k, seed):
    r = np.random.default_rng(seed)
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = min(t + 1, k)
        idx[t, :n] = np.sort(r.choice(t + 1, n, replace=False))
    return idx


@pytest.mark.parametrize("T,k", [(200, 2048), (2600, 2048), (1100, 512), (70, 64)])
def test_sparse_mla_fp8_prefill(T, k):
    d = G.mla_layer_fp8(T, seed=T)
    idx = _causal_random_idx(T, k, T)
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, 16), device="cuda")
    dsa.sparse_mla_fp8_fwd(dev(d["q"]), dev(d["kv"]), d["kv_scale"], dev(torch.from_numpy(idx)),
                           out, G.SCALE_MLA, lse=lse)
    ref, ref_lse = O.sparse_mla_fp8_prefill(d["q"], d["kv"], d["kv_scale"], idx, G.SCALE_MLA)
    check_close_bf16(out, ref, f"fp8 mla prefill T={T}")
    check_lse(lse, ref_lse, "fp8 mla prefill")


def test_sparse_mla_fp8_prefill_large_logits_and_odd_scale():
    """q x 8 (logits spread over tens of units: the lazy rescale) and a kv_scale that is
    not a power of two."""
    T, k = 700, 512
    d = G.mla_layer_fp8(T, seed=12, kv_scale=0.0123)
    q = (d["q"].float() * 8).to(torch.bfloat16)
    idx = _causal_random_idx(T, k, 12)
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, 16), device="cuda")
    dsa.sparse_mla_fp8_fwd(dev(q), dev(d["kv"]), 0.0123, dev(torch.from_numpy(idx)), out,
                           G.SCALE_MLA, lse=lse)
    ref, ref_lse = O.sparse_mla_fp8_prefill(q, d["kv"], 0.0123, idx, G.SCALE_MLA)
    g = out.float().cpu().numpy()
    assert np.all(np.abs(g - ref) <= 2e-2 + 1e-2 * np.abs(ref))
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 1e-2
    check_lse(lse, ref_lse, "fp8 rescale", tol=2e-2)


def test_quantize_then_attend():
    """bf16 latent rows -> dsa_latent_quantize_fp8 -> dsa_sparse_mla_fp8_fwd equals the
    oracle's attention over the oracle's own codes of the same rows."""
    T, k = 1500, 2048
    d = G.mla_layer(T, seed=21)
    s = 2.0 ** -7
    codes = torch.empty((T, 576), dtype=torch.uint8, device="cuda")
    dsa.latent_quantize_fp8(dev(d["kv"]), s, codes)
    ref_codes = O.latent_quantize_fp8(d["kv"], s)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    idx = _causal_random_idx(T, k, 21)
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    dsa.sparse_mla_fp8_fwd(dev(d["q"]), codes, s, dev(torch.from_numpy(idx)), out, G.SCALE_MLA)
    ref, _ = O.sparse_mla_fp8_prefill(d["q"], ref_codes, s, idx, G.SCALE_MLA)
    check_close_bf16(out, ref, "quantize then attend")


@pytest.mark.parametrize("lens,k", [([3000, 1500, 2048, 5000], 2048), ([40, 7000], 512)])
def test_sparse_mla_fp8_decode(lens, k):
    B, L = len(lens), max(lens)
    d = G.mla_decode_fp8(B=B, L=L, seed=len(lens), seq_lens=lens)
    r = np.random.default_rng(1)
    idx = np.full((B, k), -1, dtype=np.int32)
    for b, n in enumerate(lens):
        m = min(n, k)
        idx[b, :m] = np.sort(r.choice(n, m, replace=False))
    ws = torch.empty(dsa.sparse_mla_workspace_size(B, k, decode=True) // 4 + 4, device="cuda")
    out = torch.empty((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 16), device="cuda")
    dsa.sparse_mla_fp8_fwd(dev(d["q"]), dev(d["kv_pool"]), d["kv_scale"],
                           dev(torch.from_numpy(idx)), out, G.SCALE_MLA, lse=lse,
                           page_table=dev(d["page_table"]), seq_lens=dev(d["seq_lens"]),
                           workspace=ws)
    ref, ref_lse = O.sparse_mla_fp8_decode(d["q"], d["kv_pool"], d["kv_scale"], d["page_table"],
                                           idx, G.SCALE_MLA)
    check_close_bf16(out, ref, "fp8 mla decode")
    check_lse(lse, ref_lse, "fp8 mla decode")


def test_sparse_mla_fp8_decode_full_size():
    """The decode workload at full size (64 sequences x 32768 keys over 64-token pages,
    top-2048 selected per sequence), every output row against the oracle."""
    B, L, k = 64, 32768, 2048
    d = G.mla_decode_fp8(B=B, L=L, seed=0)
    r = np.random.default_rng(2)
    idx = np.stack([np.sort(r.choice(L, k, replace=False)) for _ in range(B)]).astype(np.int32)
    ws = torch.empty(dsa.sparse_mla_workspace_size(B, k, decode=True) // 4 + 4, device="cuda")
    out = torch.empty((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 16), device="cuda")
    dsa.sparse_mla_fp8_fwd(dev(d["q"]), dev(d["kv_pool"]), d["kv_scale"],
                           dev(torch.from_numpy(idx)), out, G.SCALE_MLA, lse=lse,
                           page_table=dev(d["page_table"]), seq_lens=dev(d["seq_lens"]),
                           workspace=ws)
    ref, ref_lse = O.sparse_mla_fp8_decode(d["q"], d["kv_pool"], d["kv_scale"], d["page_table"],
                                           idx, G.SCALE_MLA)
    check_close_bf16(out, ref, "fp8 decode full")
    check_lse(lse, ref_lse, "fp8 decode full")
