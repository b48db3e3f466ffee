"""Python face of the CPU oracle (dsa_oracle.c) for the DeepSeek Sparse Attention hot path.

TEST INFRASTRUCTURE ONLY: tests/, the smoke check and the benchmark's CPU-baseline leg
may import this module; the product package never does.  It shares no code with the
CUDA path.  Inputs are numpy/torch arrays on the host; every result is float64.

The C library is compiled here with gcc on first use (``build()``), into
``oracle/_build/``.  ``load(mutant=n)`` builds a copy with a deliberate mistake for the
mutation tests.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "dsa_oracle.c"
_BUILD = _HERE / "_build"
_LIBS: dict[int, ctypes.CDLL] = {}

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")


def build(mutant: int = 0, force: bool = False) -> Path:
    """Compile dsa_oracle.c (optionally with ORACLE_MUTANT=mutant) and return the .so path."""
    _BUILD.mkdir(exist_ok=True)
    out = _BUILD / ("liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so")
    if force or not out.exists() or out.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = out.with_suffix(f".{os.getpid()}.tmp")
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
               f"-DORACLE_MUTANT={mutant}", str(_SRC), "-o", str(tmp), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def load(mutant: int = 0) -> ctypes.CDLL:
    if mutant in _LIBS:
        return _LIBS[mutant]
    lib = ctypes.CDLL(str(build(mutant)))
    L, I, D = ctypes.c_long, ctypes.c_int, ctypes.c_double
    lib.oracle_indexer_scores_prefill.argtypes = [_f32p, _f32p, _f32p, I, I, I, I, I, _f64p]
    lib.oracle_indexer_scores_prefill.restype = None
    lib.oracle_indexer_scores_decode.argtypes = [_f32p, _f32p, _f32p, I, I, I, _i32p, I, I,
                                                 _i32p, I, _f64p]
    lib.oracle_indexer_scores_decode.restype = None
    lib.oracle_topk_rows.argtypes = [_f64p, L, I, _i32p, I, _i32p]
    lib.oracle_topk_rows.restype = None
    lib.oracle_sparse_attention.argtypes = [
        _f32p, L, L, _f32p, _f32p, L, L, I, I, I, I, D, _i32p, L, I,
        ctypes.c_void_p, I, I, _f64p, _f64p]
    lib.oracle_sparse_attention.restype = None
    lib.oracle_num_threads.restype = I
    lib.oracle_mutant_id.restype = I
    _LIBS[mutant] = lib
    return lib


def _f32(x) -> np.ndarray:
    """Exact float32 image of a host tensor/array (bf16 and fp32 both convert exactly)."""
    if hasattr(x, "detach"):  # torch tensor
        import torch
        x = x.detach().to("cpu")
        if x.dtype != torch.float32:
            x = x.to(torch.float32)
        x = x.numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def num_threads(mutant: int = 0) -> int:
    return load(mutant).oracle_num_threads()


# ---------------------------------------------------------------------------------
# indexer scores
# ---------------------------------------------------------------------------------
def indexer_scores_prefill(q_idx, k_idx, w, q_begin: int = 0, rows: int | None = None,
                           S: int | None = None, mutant: int = 0) -> np.ndarray:
    """I(t,s) for t = q_begin..q_begin+rows-1, all s < S; s > t is -inf.

    q_idx [T,H_I,D_I], k_idx [S,D_I], w [T,H_I]."""
    q = _f32(q_idx)
    kk = _f32(k_idx)
    ww = _f32(w)
    T, H_I, D_I = q.shape
    if rows is None:
        rows = T - q_begin
    if S is None:
        S = kk.shape[0]
    assert kk.shape == (kk.shape[0], D_I) and S <= kk.shape[0]
    assert ww.shape == (T, H_I) and 0 <= q_begin and q_begin + rows <= T
    out = np.empty((rows, S), dtype=np.float64)
    load(mutant).oracle_indexer_scores_prefill(q, kk, ww, H_I, D_I, q_begin, rows, S, out)
    return out


def indexer_scores_decode(q_idx, k_pool, w, page_table, seq_lens, S: int | None = None,
                          mutant: int = 0) -> np.ndarray:
    """Decode scores: q_idx [B,H_I,D_I], k_pool [num_pages,page_size,D_I], w [B,H_I],
    page_table [B,max_pages] int32, seq_lens [B] int32 -> [B,S] (invalid = -inf)."""
    q = _f32(q_idx)
    kp = _f32(k_pool)
    ww = _f32(w)
    pt = _i32(page_table)
    sl = _i32(seq_lens)
    B, H_I, D_I = q.shape
    num_pages, page_size, d = kp.shape
    assert d == D_I and pt.shape[0] == B and sl.shape == (B,)
    max_pages = pt.shape[1]
    if S is None:
        S = int(sl.max())
    out = np.empty((B, S), dtype=np.float64)
    load(mutant).oracle_indexer_scores_decode(q, kp.reshape(-1, D_I), ww, H_I, D_I, B, pt,
                                              max_pages, page_size, sl, S, out)
    return out


# ---------------------------------------------------------------------------------
# top-k
# ---------------------------------------------------------------------------------
def topk(scores: np.ndarray, n_valid, k: int, mutant: int = 0) -> np.ndarray:
    """Per row: k highest of the first n_valid[r] scores, ties to the lower index,
    returned ascending and padded with -1.  scores [rows, >=max n_valid] float64."""
    sc = np.ascontiguousarray(scores, dtype=np.float64)
    rows = sc.shape[0]
    nv = _i32(np.broadcast_to(np.asarray(n_valid), (rows,)))
    assert int(nv.max(initial=0)) <= sc.shape[1]
    out = np.empty((rows, k), dtype=np.int32)
    load(mutant).oracle_topk_rows(sc, sc.shape[1], rows, nv, k, out)
    return out


def causal_n_valid(q_begin: int, rows: int) -> np.ndarray:
    """Valid key count of prefill rows q_begin..q_begin+rows-1 (s <= t)."""
    return np.arange(q_begin + 1, q_begin + rows + 1, dtype=np.int32)


# ---------------------------------------------------------------------------------
# sparse attention
# ---------------------------------------------------------------------------------
def sparse_mla_prefill(q, kv, idx, scale: float, d_v: int = 512, mutant: int = 0):
    """Absorbed MLA over selected keys: q [NQ,H,D_qk], kv [S,D_qk] (value = first d_v
    dims), idx [NQ,k] -> (out [NQ,H,d_v], lse [NQ,H]) float64."""
    qq = _f32(q)
    c = _f32(kv)
    ii = _i32(idx)
    NQ, H, D = qq.shape
    out = np.empty((NQ, H, d_v), dtype=np.float64)
    lse = np.empty((NQ, H), dtype=np.float64)
    load(mutant).oracle_sparse_attention(qq, H * D, D, c, c, D, 0, NQ, H, D, d_v, scale,
                                         ii, ii.shape[1], ii.shape[1], None, 0, 0, out, lse)
    return out, lse


def sparse_mla_decode(q, kv_pool, page_table, idx, scale: float, d_v: int = 512,
                      mutant: int = 0):
    """Decode: q [B,H,D_qk], kv_pool [num_pages,page_size,D_qk], page_table [B,max_pages],
    idx [B,k] token positions -> (out [B,H,d_v], lse [B,H])."""
    qq = _f32(q)
    c = _f32(kv_pool)
    pt = _i32(page_table)
    ii = _i32(idx)
    B, H, D = qq.shape
    page_size = c.shape[1]
    out = np.empty((B, H, d_v), dtype=np.float64)
    lse = np.empty((B, H), dtype=np.float64)
    flat = c.reshape(-1, D)
    load(mutant).oracle_sparse_attention(qq, H * D, D, flat, flat, D, 0, B, H, D, d_v, scale,
                                         ii, ii.shape[1], ii.shape[1],
                                         pt.ctypes.data_as(ctypes.c_void_p), pt.shape[1],
                                         page_size, out, lse)
    return out, lse


def sparse_mha(q, k, v, idx, scale: float, mutant: int = 0):
    """Multi-head attention over selected keys (one index set per query shared by all
    heads): q,k,v [T,H,D] -> (out [T,H,D], lse [T,H])."""
    qq, kk, vv = _f32(q), _f32(k), _f32(v)
    ii = _i32(idx)
    T, H, D = qq.shape
    assert kk.shape[1:] == (H, D) and vv.shape[1:] == (H, D)
    out = np.empty((T, H, D), dtype=np.float64)
    lse = np.empty((T, H), dtype=np.float64)
    lib = load(mutant)
    if kk.shape != vv.shape:
        raise ValueError("k and v must have the same shape")
    # k and v are separate tensors with the same strides: pass both.
    lib.oracle_sparse_attention(qq, H * D, D, kk, vv, H * D, D, T, H, D, D, scale,
                                ii, ii.shape[1], ii.shape[1], None, 0, 0, out, lse)
    return out, lse


# ---------------------------------------------------------------------------------
# whole path
# ---------------------------------------------------------------------------------
def prefill_indices(q_idx, k_idx, w, k: int, q_begin: int = 0, rows: int | None = None,
                    mutant: int = 0) -> np.ndarray:
    """Indexer + top-k for prefill rows q_begin..q_begin+rows-1 (causal)."""
    T = q_idx.shape[0]
    if rows is None:
        rows = T - q_begin
    sc = indexer_scores_prefill(q_idx, k_idx, w, q_begin, rows, S=q_begin + rows,
                                mutant=mutant)
    return topk(sc, causal_n_valid(q_begin, rows), k, mutant=mutant)


def prefill_indices_varlen(q_idx, k_idx, w, seq_start, seq_len, k: int, fill: int = -1,
                           mutant: int = 0) -> np.ndarray:
    """Batched prefill of packed sequences (DSV2-Lite-IndexCache card: causal selection per
    query; batched generation with left padding).  Sequence b is an independent prompt
    over the tokens seq_start[b] .. seq_start[b]+seq_len[b]-1: its queries select among
    its own earlier keys only.  Indices are returned as packed token rows; rows outside
    every sequence hold `fill`.  (Mutant 13: the packed offset is left off.)"""
    N = q_idx.shape[0]
    out = np.full((N, k), fill, dtype=np.int32)
    for s0, L in zip(seq_start, seq_len):
        s0, L = int(s0), int(L)
        if L == 0:
            continue
        sl = slice(s0, s0 + L)
        idx = prefill_indices(q_idx[sl], k_idx[sl], w[sl], k, mutant=mutant)
        off = 0 if mutant == 13 else s0
        out[sl] = np.where(idx >= 0, idx + off, -1)
    return out


def layer_stack(pattern: str, layers: list[dict], k: int, scale: float, d_v: int = 512,
                mutant: int = 0):
    """IndexCache layer loop (vLLM IndexCache docs, "How It Works"): an 'F' layer computes
    and stores the top-k indices from its own indexer inputs; each 'S' layer reuses the
    stored indices of the nearest preceding 'F' layer.  layers[l] holds 'q', 'kv' and,
    for F layers, 'q_idx', 'k_idx', 'w'.  Returns (outs, lses, idx_per_layer)."""
    if not pattern or pattern[0] != "F" or set(pattern) - {"F", "S"}:
        raise ValueError("pattern must start with 'F' and contain only 'F'/'S'")
    if len(pattern) != len(layers):
        raise ValueError("one pattern character per layer")
    idx = None
    outs, lses, idxs = [], [], []
    for ch, L in zip(pattern, layers):
        if ch == "F":
            idx = prefill_indices(L["q_idx"], L["k_idx"], L["w"], k, mutant=mutant)
        o, s = sparse_mla_prefill(L["q"], L["kv"], idx, scale, d_v, mutant=mutant)
        outs.append(o)
        lses.append(s)
        idxs.append(idx)
    return outs, lses, idxs


def pattern_from_freq(freq: int, num_layers: int) -> str:
    """index_topk_freq reading (vLLM IndexCache docs, "Configuration Reference"):
    layer i computes top-k iff i % freq == 0; freq 1 computes on every layer."""
    if freq < 1 or num_layers < 1:
        raise ValueError("freq and num_layers must be positive")
    return "".join("F" if i % freq == 0 else "S" for i in range(num_layers))


# ---------------------------------------------------------------------------------
# fp8 latent cache
# ---------------------------------------------------------------------------------
# DeepSeek-V2-Lite-Chat SIQ card (what is quantized, KV-cache bullet): the non-sparse MLA
# backend keeps the KV cache in fp8 at 576 bytes per token, i.e. one byte for each of the
# 576 latent elements.  The card does not spell out the encoding; the reading here is the
# E4M3 variant of the OCP 8-bit floating-point format with one fp32 scale per cache
# tensor, value = kv_scale * e4m3(code).
#
# E4M3 (OCP 8-bit floating point specification): bit 7 sign, bits 6..3 exponent with
# bias 7, bits 2..0 mantissa.  Exponent field 0 encodes subnormals m/8 * 2^-6; the code
# with exponent and mantissa fields all ones (0x7f / 0xff) is NaN; there is no infinity,
# so the largest finite magnitude is 1.75 * 2^8 = 448.
#
# Mutants 9..12 (Python-side planted mistakes for the pin mutation test; 13 is in
# prefill_indices_varlen):
#   9  exponent bias 8 instead of 7        10  subnormals decoded as normals
#   11 encoder ties rounded away from zero 12  kv_scale left off the attention output
def e4m3_decode(codes, mutant: int = 0) -> np.ndarray:
    """Exact float64 values of E4M3 codes (uint8 array of any shape)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    bias = 8 if mutant == 9 else 7
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - bias)
    sub = (m / 8.0) * 2.0 ** (1 - bias)
    mag = normal if mutant == 10 else np.where(e == 0, sub, normal)
    val = np.where(sign == 1, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, val)


def e4m3_encode(x, mutant: int = 0) -> np.ndarray:
    """E4M3 codes of float values, rounded to the nearest code with ties to the even code
    (round-to-nearest-even), magnitudes above 448 saturated to 448 (the finite-saturating
    conversion), the sign kept for values that round to zero; NaN -> 0x7f."""
    xs = np.asarray(x, dtype=np.float64)
    pos = e4m3_decode(np.arange(127, dtype=np.uint8), mutant)  # codes 0..126: 0 .. 448
    a = np.abs(xs)
    hi_i = np.clip(np.searchsorted(pos, a, side="left"), 1, 126)
    lo_i = hi_i - 1
    lo, hi = pos[lo_i], pos[hi_i]
    mid = (lo + hi) / 2.0  # exact: both are short binary fractions
    if mutant == 11:
        tie = hi_i
    else:
        tie = np.where(lo_i % 2 == 0, lo_i, hi_i)
    code = np.where(a < mid, lo_i, np.where(a > mid, hi_i, tie))
    code = np.where(a >= pos[126], 126, code)
    code = code | (np.signbit(xs).astype(np.int64) << 7)
    code = np.where(np.isnan(xs), 0x7F, code)
    return code.astype(np.uint8)


def latent_quantize_fp8(c, kv_scale: float, mutant: int = 0) -> np.ndarray:
    """Codes of a latent cache: e4m3_encode(c / kv_scale), the quotient taken in fp32
    (the precision in which the quantised code is decided)."""
    x = _f32(c) / np.float32(kv_scale)
    return e4m3_encode(x.astype(np.float32), mutant)


def sparse_mla_fp8_prefill(q, kv_codes, kv_scale: float, idx, scale: float, d_v: int = 512,
                           mutant: int = 0):
    """Absorbed MLA over an fp8 latent cache: the latent row of key s is
    kv_scale * e4m3_decode(kv_codes[s]).  The decoded codes are exact in float32, so the
    attention runs on them with the logit scale scale*kv_scale, and the output (a convex
    combination of value rows) is multiplied by kv_scale."""
    codes = kv_codes.detach().cpu().numpy() if hasattr(kv_codes, "detach") else kv_codes
    c = e4m3_decode(codes, mutant).astype(np.float32)
    out, lse = sparse_mla_prefill(q, c, idx, float(scale) * float(kv_scale), d_v, mutant)
    return (out if mutant == 12 else out * float(kv_scale)), lse


def sparse_mla_fp8_decode(q, kv_pool_codes, kv_scale: float, page_table, idx, scale: float,
                          d_v: int = 512, mutant: int = 0):
    """Decode over a paged fp8 latent pool [num_pages, page_size, D_qk] of E4M3 codes."""
    codes = (kv_pool_codes.detach().cpu().numpy() if hasattr(kv_pool_codes, "detach")
             else kv_pool_codes)
    c = e4m3_decode(codes, mutant).astype(np.float32)
    out, lse = sparse_mla_decode(q, c, page_table, idx, float(scale) * float(kv_scale), d_v,
                                 mutant)
    return (out if mutant == 12 else out * float(kv_scale)), lse
