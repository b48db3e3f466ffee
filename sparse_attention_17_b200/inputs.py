"""Seeded synthetic inputs for the DSA hot path.

This module holds random draws and dtype casts only -- none of the method's arithmetic --
so that both the CUDA path and the CPU oracle can be fed the very same values.  Every
tensor is created on the host with a ``torch.Generator('cpu')``; a fixed order of draws
per workload (q_idx, k_idx, w, q, kv, page_table) makes each tensor a function of the seed.

Workloads (sizes from the DSV2-Lite-IndexCache card -- top-2048 budget, 65536 training
length, FSS x 9 -- and the DSA ablation card -- 2 indexer heads x dim 16, top-512, 4 heads,
context 3072; MLA latent 576 = 512 + 64 from the DeepSeek-V2-Lite-Chat SIQ card):

* ``tiny_fp32``      fp32, T=3072, indexer 2x16 integer-valued in [-8,8], w in [1,4],
                     MHA 4 heads x 32, q/k/v ~ N(0,1), k=512.
* ``mla_prefill_int`` bf16, indexer 16x64 integer-valued in [-4,4], w in [1,3];
                     q [T,16,576], latent kv [T,576] ~ N(0, 0.5^2); k=2048.
* ``mla_prefill_gauss`` bf16, indexer q_idx/k_idx ~ N(0,1), w ~ U(0,1); q, kv as above.
* ``mla_decode``     bf16, B sequences of length L over 64-token pages with a random
                     page permutation; integer indexer inputs as above.
* ``*_fp8`` variants the latent cache as E4M3 codes (one byte per element, 576 bytes per
                     token, DeepSeek-V2-Lite-Chat SIQ card) with one fp32 scale per cache:
                     draws of N(0, (0.5/kv_scale)^2), clamped to +-448 and cast to
                     torch.float8_e4m3fn, so that kv_scale * code ~ N(0, 0.5^2) as for bf16.
"""
from __future__ import annotations

import torch

H_I_MLA, D_I_MLA = 16, 64
H_MLA, D_QK_MLA, D_V_MLA = 16, 576, 512
SCALE_MLA = 192 ** -0.5
H_I_TINY, D_I_TINY, H_TINY, D_TINY = 2, 16, 4, 32
SCALE_TINY = 32 ** -0.5


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randint(g, lo: int, hi: int, shape, dtype) -> torch.Tensor:
    """Integers uniform in [lo, hi] (inclusive), cast to dtype (exact for these ranges)."""
    return torch.randint(lo, hi + 1, shape, generator=g, dtype=torch.int64).to(dtype)


def _normal(g, std: float, shape, dtype, chunk: int = 1 << 26) -> torch.Tensor:
    """N(0, std^2) draws rounded to dtype, generated in chunks to bound host memory."""
    n = 1
    for s in shape:
        n *= s
    out = torch.empty(n, dtype=dtype)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        out[i:i + m] = (torch.randn(m, generator=g, dtype=torch.float32) * std).to(dtype)
    return out.view(*shape)


def tiny_fp32(T: int = 3072, seed: int = 0, k: int = 512) -> dict:
    g = _gen(seed)
    d = {}
    d["q_idx"] = _randint(g, -8, 8, (T, H_I_TINY, D_I_TINY), torch.float32)
    d["k_idx"] = _randint(g, -8, 8, (T, D_I_TINY), torch.float32)
    d["w"] = _randint(g, 1, 4, (T, H_I_TINY), torch.float32)
    d["q"] = _normal(g, 1.0, (T, H_TINY, D_TINY), torch.float32)
    d["k"] = _normal(g, 1.0, (T, H_TINY, D_TINY), torch.float32)
    d["v"] = _normal(g, 1.0, (T, H_TINY, D_TINY), torch.float32)
    d.update(T=T, topk=k, scale=SCALE_TINY)
    return d


def indexer_int(T: int, seed: int, H_I: int = H_I_MLA, D_I: int = D_I_MLA, g=None) -> dict:
    """Integer-valued indexer inputs: q_idx, k_idx in [-4,4] (bf16), w in [1,3] (fp32)."""
    g = g or _gen(seed)
    return {"q_idx": _randint(g, -4, 4, (T, H_I, D_I), torch.bfloat16),
            "k_idx": _randint(g, -4, 4, (T, D_I), torch.bfloat16),
            "w": _randint(g, 1, 3, (T, H_I), torch.float32)}


def indexer_gauss(T: int, seed: int, H_I: int = H_I_MLA, D_I: int = D_I_MLA, g=None) -> dict:
    """Gaussian indexer inputs: q_idx, k_idx ~ N(0,1) (bf16), w ~ U(0,1) (fp32)."""
    g = g or _gen(seed)
    return {"q_idx": _normal(g, 1.0, (T, H_I, D_I), torch.bfloat16),
            "k_idx": _normal(g, 1.0, (T, D_I), torch.bfloat16),
            "w": torch.rand((T, H_I), generator=g, dtype=torch.float32)}


def mla_layer(T: int, seed: int, H: int = H_MLA, D: int = D_QK_MLA, g=None) -> dict:
    """One layer's MLA inputs: q [T,H,D], latent kv [T,D], both ~ N(0, 0.5^2) in bf16."""
    g = g or _gen(seed)
    return {"q": _normal(g, 0.5, (T, H, D), torch.bfloat16),
            "kv": _normal(g, 0.5, (T, D), torch.bfloat16)}


KV_SCALE_FP8 = 2.0 ** -7


def _e4m3_codes(g, std: float, shape, chunk: int = 1 << 26) -> torch.Tensor:
    """uint8 E4M3 codes of N(0, std^2) draws clamped to +-448 (a dtype cast per chunk)."""
    n = 1
    for s in shape:
        n *= s
    out = torch.empty(n, dtype=torch.uint8)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        z = (torch.randn(m, generator=g, dtype=torch.float32) * std).clamp_(-448.0, 448.0)
        out[i:i + m] = z.to(torch.float8_e4m3fn).view(torch.uint8)
    return out.view(*shape)


def mla_layer_fp8(T: int, seed: int, kv_scale: float = KV_SCALE_FP8, H: int = H_MLA,
                  D: int = D_QK_MLA, g=None) -> dict:
    """MLA inputs over an fp8 latent cache: q [T,H,D] bf16 ~ N(0, 0.5^2); kv [T,D] uint8
    E4M3 codes with kv_scale * value ~ N(0, 0.5^2)."""
    g = g or _gen(seed)
    return {"q": _normal(g, 0.5, (T, H, D), torch.bfloat16),
            "kv": _e4m3_codes(g, 0.5 / kv_scale, (T, D)), "kv_scale": kv_scale}


def mla_prefill_int(T: int = 8192, seed: int = 0, k: int = 2048) -> dict:
    g = _gen(seed)
    d = indexer_int(T, seed, g=g)
    d.update(mla_layer(T, seed, g=g))
    d.update(T=T, topk=k, scale=SCALE_MLA)
    return d


def mla_prefill_gauss(T: int = 65536, seed: int = 0, k: int = 2048) -> dict:
    g = _gen(seed)
    d = indexer_gauss(T, seed, g=g)
    d.update(mla_layer(T, seed, g=g))
    d.update(T=T, topk=k, scale=SCALE_MLA)
    return d


def mla_prefill_gauss_fp8(T: int = 65536, seed: int = 0, k: int = 2048,
                          kv_scale: float = KV_SCALE_FP8) -> dict:
    """mla_prefill_gauss with the latent cache as E4M3 codes."""
    g = _gen(seed)
    d = indexer_gauss(T, seed, g=g)
    d.update(mla_layer_fp8(T, seed, kv_scale, g=g))
    d.update(T=T, topk=k, scale=SCALE_MLA)
    return d


def layer_stack(T: int = 16384, pattern: str = "FSS" * 9, k: int = 2048,
                mla_seed_base: int = 1000, indexer_seed_base: int = 2000,
                layers: list[int] | None = None) -> dict:
    """IndexCache stack inputs: layer l has MLA inputs seeded mla_seed_base+l and, if it is
    an 'F' layer, integer indexer inputs seeded indexer_seed_base+l.  ``layers`` limits
    generation to a subset (the others are None) to bound host memory."""
    out = []
    for l, ch in enumerate(pattern):
        if layers is not None and l not in layers:
            out.append(None)
            continue
        L = mla_layer(T, mla_seed_base + l)
        if ch == "F":
            L.update(indexer_int(T, indexer_seed_base + l))
        out.append(L)
    return {"layers": out, "pattern": pattern, "T": T, "topk": k, "scale": SCALE_MLA}


def mla_decode(B: int = 64, L: int = 32768, seed: int = 0, k: int = 2048,
               page_size: int = 64, seq_lens=None) -> dict:
    """Paged decode inputs.  The pool holds B*ceil(L/page_size) pages; sequence b owns
    the pages page_table[b] (a random permutation of the pool)."""
    g = _gen(seed)
    max_pages = (L + page_size - 1) // page_size
    num_pages = B * max_pages
    d = {}
    d["q_idx"] = _randint(g, -4, 4, (B, H_I_MLA, D_I_MLA), torch.bfloat16)
    d["w"] = _randint(g, 1, 3, (B, H_I_MLA), torch.float32)
    d["k_idx_pool"] = _randint(g, -4, 4, (num_pages, page_size, D_I_MLA), torch.bfloat16)
    d["q"] = _normal(g, 0.5, (B, H_MLA, D_QK_MLA), torch.bfloat16)
    d["kv_pool"] = _normal(g, 0.5, (num_pages, page_size, D_QK_MLA), torch.bfloat16)
    d["page_table"] = torch.randperm(num_pages, generator=g).to(torch.int32).view(B, max_pages)
    if seq_lens is None:
        seq_lens = [L] * B
    d["seq_lens"] = torch.tensor(seq_lens, dtype=torch.int32)
    d.update(B=B, L=L, topk=k, page_size=page_size, scale=SCALE_MLA)
    return d


def mla_decode_fp8(B: int = 64, L: int = 32768, seed: int = 0, k: int = 2048,
                   page_size: int = 64, seq_lens=None, kv_scale: float = KV_SCALE_FP8) -> dict:
    """mla_decode with the paged latent pool as E4M3 codes (same order of draws)."""
    g = _gen(seed)
    max_pages = (L + page_size - 1) // page_size
    num_pages = B * max_pages
    d = {}
    d["q_idx"] = _randint(g, -4, 4, (B, H_I_MLA, D_I_MLA), torch.bfloat16)
    d["w"] = _randint(g, 1, 3, (B, H_I_MLA), torch.float32)
    d["k_idx_pool"] = _randint(g, -4, 4, (num_pages, page_size, D_I_MLA), torch.bfloat16)
    d["q"] = _normal(g, 0.5, (B, H_MLA, D_QK_MLA), torch.bfloat16)
    d["kv_pool"] = _e4m3_codes(g, 0.5 / kv_scale, (num_pages, page_size, D_QK_MLA))
    d["page_table"] = torch.randperm(num_pages, generator=g).to(torch.int32).view(B, max_pages)
    if seq_lens is None:
        seq_lens = [L] * B
    d["seq_lens"] = torch.tensor(seq_lens, dtype=torch.int32)
    d.update(B=B, L=L, topk=k, page_size=page_size, scale=SCALE_MLA, kv_scale=kv_scale)
    return d
