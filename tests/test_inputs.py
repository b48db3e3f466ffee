"""The seeded generators: same seed -> same tensors, documented ranges and dtypes."""
import torch

from sparse_attention_17_b200 import inputs as G


def test_tiny_fp32_ranges_and_determinism():
    a, b = G.tiny_fp32(T=64), G.tiny_fp32(T=64)
    for key in ("q_idx", "k_idx", "w", "q", "k", "v"):
        assert torch.equal(a[key], b[key]) and a[key].dtype == torch.float32
    assert a["q_idx"].min() >= -8 and a["q_idx"].max() <= 8
    assert a["w"].min() >= 1 and a["w"].max() <= 4
    assert torch.equal(a["q_idx"], torch.round(a["q_idx"]))


def test_mla_int_ranges():
    d = G.mla_prefill_int(T=128)
    assert d["q_idx"].dtype == torch.bfloat16 and d["q"].shape == (128, 16, 576)
    assert d["kv"].shape == (128, 576)
    assert int(d["q_idx"].float().abs().max()) <= 4 and d["w"].min() >= 1 and d["w"].max() <= 3
    assert 0.4 < d["kv"].float().std().item() < 0.6


def test_decode_pages_are_a_permutation():
    d = G.mla_decode(B=4, L=300, page_size=64)
    pt = d["page_table"]
    assert pt.shape == (4, 5)
    assert torch.equal(pt.flatten().sort().values, torch.arange(20, dtype=torch.int32))


def test_stack_seeds_per_layer():
    s = G.layer_stack(T=32, pattern="FSS")
    assert "q_idx" in s["layers"][0] and "q_idx" not in s["layers"][1]
    assert not torch.equal(s["layers"][0]["q"], s["layers"][1]["q"])


def test_fp8_latent_codes():
    """E4M3 codes: no NaN code, deterministic, and kv_scale * value ~ N(0, 0.5^2)."""
    a, b = G.mla_layer_fp8(T=256, seed=3), G.mla_layer_fp8(T=256, seed=3)
    assert a["kv"].dtype == torch.uint8 and a["kv"].shape == (256, 576)
    assert torch.equal(a["kv"], b["kv"]) and torch.equal(a["q"], b["q"])
    assert not bool(((a["kv"] & 0x7F) == 0x7F).any())
    val = a["kv"].view(torch.float8_e4m3fn).to(torch.float32) * a["kv_scale"]
    assert 0.45 < val.std().item() < 0.55
    d = G.mla_decode_fp8(B=2, L=130, page_size=64)
    assert d["kv_pool"].shape == (6, 64, 576) and d["kv_pool"].dtype == torch.uint8
    assert torch.equal(d["page_table"], G.mla_decode(B=2, L=130, page_size=64)["page_table"])
