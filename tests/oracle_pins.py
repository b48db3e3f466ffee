"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle (optionally a mutant build
with a planted mistake, see dsa_oracle.c) disagrees with:
  * closed forms and special cases that reduce to a library routine (numpy matmul,
    torch SDPA, torch.topk, numpy.argmax, torch.logsumexp),
  * brute force on tiny inputs,
  * invariants the pages state (all keys selected when the prompt is no longer than k,
    DSA ablation card; S layers reuse the F layer's indices, vLLM IndexCache docs),
  * a hand-worked example.
test_oracle_pins.py runs them on the real oracle; test_oracle_mutants.py checks that
every planted mistake trips at least one of them.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------------
# indexer
# ---------------------------------------------------------------------------------
def pin_indexer_hand_example(mutant=0):
    """Three tokens, 2 indexer heads of dim 2, scores worked out by hand from
    I(t,s) = sum_j w[t,j] max(0, q[t,j].k[s]).  Row 2 has a tie (s=1 and s=2 both 1)."""
    q = np.array([[[1, 2], [-1, 0]],
                  [[0, 1], [2, -1]],
                  [[1, -1], [1, 1]]], dtype=np.float32)
    k = np.array([[2, 1], [-1, 3], [1, 1]], dtype=np.float32)
    w = np.array([[1, 2], [3, 1], [2, 0.5]], dtype=np.float32)
    sc = O.indexer_scores_prefill(q, k, w, mutant=mutant)
    inf = -np.inf
    expect = np.array([[4.0, inf, inf],
                       [6.0, 9.0, inf],
                       [3.5, 1.0, 1.0]])
    assert np.array_equal(sc, expect), sc
    idx2 = O.topk(sc, O.causal_n_valid(0, 3), 2, mutant=mutant)
    assert idx2.tolist() == [[0, -1], [0, 1], [0, 1]], idx2
    idx1 = O.topk(sc, O.causal_n_valid(0, 3), 1, mutant=mutant)
    assert idx1.tolist() == [[0], [1], [0]], idx1


def pin_indexer_linear_regime(mutant=0):
    """With q_idx, k_idx >= 0 every ReLU is the identity, so the score is the matmul
    (sum_j w[t,j] q[t,j]) . k[s] -- a single library GEMM."""
    r = _rng(1)
    T, H_I, D_I = 40, 3, 16
    q = r.integers(0, 5, (T, H_I, D_I)).astype(np.float32)
    k = r.integers(0, 5, (T, D_I)).astype(np.float32)
    w = r.integers(1, 4, (T, H_I)).astype(np.float32)
    sc = O.indexer_scores_prefill(q, k, w, mutant=mutant)
    qw = np.einsum("tj,tjd->td", w.astype(np.float64), q.astype(np.float64))
    full = qw @ k.astype(np.float64).T
    mask = np.tril(np.ones((T, T), dtype=bool))
    assert np.array_equal(sc[mask], full[mask])
    assert np.all(np.isneginf(sc[~mask]))


def pin_indexer_relu_abs(mutant=0):
    """Two heads with q[t,1] = -q[t,0] and unit weights give relu(x) + relu(-x) = |x|,
    x = q[t,0].k[s]: the ReLU and both heads are visible in one closed form."""
    r = _rng(2)
    T, D_I = 33, 8
    q0 = r.integers(-8, 9, (T, D_I)).astype(np.float32)
    q = np.stack([q0, -q0], axis=1)
    k = r.integers(-8, 9, (T, D_I)).astype(np.float32)
    w = np.ones((T, 2), dtype=np.float32)
    sc = O.indexer_scores_prefill(q, k, w, mutant=mutant)
    x = q0.astype(np.float64) @ k.astype(np.float64).T
    mask = np.tril(np.ones((T, T), dtype=bool))
    assert np.array_equal(sc[mask], np.abs(x)[mask])


def pin_indexer_single_head_clamp(mutant=0):
    """One head and w = 2: I = 2 * max(0, q.k), a clamped library GEMM; the diagonal
    s = t is a valid key."""
    r = _rng(3)
    T, D_I = 29, 16
    q = r.normal(size=(T, 1, D_I)).astype(np.float32)
    k = r.normal(size=(T, D_I)).astype(np.float32)
    w = np.full((T, 1), 2.0, dtype=np.float32)
    sc = O.indexer_scores_prefill(q, k, w, mutant=mutant)
    ref = 2.0 * np.maximum(q[:, 0, :].astype(np.float64) @ k.astype(np.float64).T, 0.0)
    mask = np.tril(np.ones((T, T), dtype=bool))
    np.testing.assert_allclose(sc[mask], ref[mask], rtol=1e-12, atol=1e-12)
    assert np.all(np.isfinite(np.diag(sc)))


def pin_decode_equals_prefill_last_row(mutant=0):
    """Paging is only a permutation of rows: scoring the last token of a contiguous
    sequence equals decode scoring through a random page table."""
    r = _rng(4)
    L, P, H_I, D_I = 200, 16, 4, 8
    max_pages = (L + P - 1) // P
    q = r.integers(-4, 5, (L, H_I, D_I)).astype(np.float32)
    k = r.integers(-4, 5, (L, D_I)).astype(np.float32)
    w = r.integers(1, 4, (L, H_I)).astype(np.float32)
    num_pages = max_pages + 3
    perm = r.permutation(num_pages)[:max_pages].astype(np.int32)
    pool = np.zeros((num_pages, P, D_I), dtype=np.float32)
    for s in range(L):
        pool[perm[s // P], s % P] = k[s]
    sc_pre = O.indexer_scores_prefill(q, k, w, q_begin=L - 1, rows=1, mutant=mutant)
    sc_dec = O.indexer_scores_decode(q[L - 1:], pool, w[L - 1:], perm[None, :],
                                     np.array([L], np.int32), mutant=mutant)
    assert np.array_equal(sc_pre, sc_dec)
    ref = np.einsum("jd,sd->js", q[L - 1].astype(np.float64), k.astype(np.float64))
    ref = (w[L - 1, :, None] * np.maximum(ref, 0)).sum(0)
    assert np.array_equal(sc_dec[0], ref)


# ---------------------------------------------------------------------------------
# top-k
# ---------------------------------------------------------------------------------
def _brute_topk(row, n, k):
    order = sorted(range(n), key=lambda s: (-row[s], s))[:k]
    return sorted(order) + [-1] * (k - min(n, k))


def pin_topk_brute_force(mutant=0):
    """Full sort by (score desc, index asc) on tiny rows with heavy ties."""
    r = _rng(5)
    for trial in range(30):
        rows, S = 7, int(r.integers(1, 60))
        k = int(r.integers(1, 20))
        sc = r.integers(0, 4, (rows, S)).astype(np.float64)
        nv = r.integers(1, S + 1, rows).astype(np.int32)
        got = O.topk(sc, nv, k, mutant=mutant)
        for i in range(rows):
            assert got[i].tolist() == _brute_topk(sc[i], int(nv[i]), k), (trial, i)


def pin_topk_argmax(mutant=0):
    """k = 1 is numpy.argmax, which returns the first (lowest-index) maximum."""
    r = _rng(6)
    sc = r.integers(0, 3, (50, 31)).astype(np.float64)
    got = O.topk(sc, 31, 1, mutant=mutant)
    assert np.array_equal(got[:, 0], np.argmax(sc, axis=1))


def pin_topk_values_match_torch(mutant=0):
    """The multiset of selected scores equals torch.topk's values; when n <= k every
    valid key is selected in order, then -1."""
    r = _rng(7)
    sc = r.normal(size=(20, 300))
    got = O.topk(sc, 300, 37, mutant=mutant)
    ref = torch.topk(torch.from_numpy(sc), 37, dim=1).values.numpy()
    sel = np.take_along_axis(sc, got, axis=1)
    assert np.array_equal(np.sort(sel, axis=1), np.sort(ref, axis=1))
    assert np.all(np.diff(got, axis=1) > 0)
    small = O.topk(sc, 10, 37, mutant=mutant)
    assert np.array_equal(small, np.tile(np.r_[np.arange(10), -np.ones(27)], (20, 1)))


# ---------------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------------
def _sdpa64(q, k, v, mask=None, causal=False, scale=None):
    """torch SDPA in float64 on CPU; q [T,H,D], k/v [S,H,D] -> [T,H,Dv]."""
    qt = torch.from_numpy(np.asarray(q, np.float64)).transpose(0, 1)
    kt = torch.from_numpy(np.asarray(k, np.float64)).transpose(0, 1)
    vt = torch.from_numpy(np.asarray(v, np.float64)).transpose(0, 1)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal, scale=scale)
    return o.transpose(0, 1).numpy()


def pin_attention_dense_when_short(mutant=0):
    """At T <= k every causal key is selected and sparse attention equals dense causal
    attention (DSA ablation card, closing note) -- torch SDPA with is_causal=True.
    Checked for MHA (4 heads x 32) and for absorbed MLA (value = first 512 dims)."""
    r = _rng(8)
    T, H, D, k = 50, 4, 32, 64
    q, kk, v = (r.normal(size=(T, H, D)).astype(np.float32) for _ in range(3))
    idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    idx[idx > np.arange(T)[:, None]] = -1
    idx[:, T:] = -1
    out, _ = O.sparse_mha(q, kk, v, idx, D ** -0.5, mutant=mutant)
    ref = _sdpa64(q, kk, v, causal=True, scale=D ** -0.5)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)

    T, H, D, Dv = 40, 2, 576, 512
    q = (0.5 * r.normal(size=(T, H, D))).astype(np.float32)
    c = (0.5 * r.normal(size=(T, D))).astype(np.float32)
    idx = np.tile(np.arange(64, dtype=np.int32), (T, 1))
    idx[idx > np.arange(T)[:, None]] = -1
    out, _ = O.sparse_mla_prefill(q, c, idx, 192 ** -0.5, mutant=mutant)
    kk = np.repeat(c[:, None, :], H, axis=1)
    ref = _sdpa64(q, kk, kk[..., :Dv], causal=True, scale=192 ** -0.5)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def pin_attention_masked_sdpa(mutant=0):
    """With T > k the oracle equals SDPA under the boolean mask built from the indices
    (the DSV2-Lite-IndexCache card's portable runtime: masked SDPA)."""
    r = _rng(9)
    T, H, D, k = 80, 3, 576, 16
    q = (0.5 * r.normal(size=(T, H, D))).astype(np.float32)
    c = (0.5 * r.normal(size=(T, D))).astype(np.float32)
    idx = np.full((T, k), -1, dtype=np.int32)
    mask = np.zeros((T, T), dtype=bool)
    for t in range(T):
        sel = np.sort(r.choice(t + 1, size=min(k, t + 1), replace=False))
        idx[t, :len(sel)] = sel
        mask[t, sel] = True
    out, lse = O.sparse_mla_prefill(q, c, idx, 192 ** -0.5, mutant=mutant)
    kk = np.repeat(c[:, None, :], H, axis=1)
    ref = _sdpa64(q, kk, kk[..., :512], mask=mask, scale=192 ** -0.5)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    logits = np.einsum("thd,sd->ths", q.astype(np.float64), c.astype(np.float64)) * 192 ** -0.5
    logits = np.where(mask[:, None, :], logits, -np.inf)
    ref_lse = torch.logsumexp(torch.from_numpy(logits), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def pin_attention_closed_forms(mutant=0):
    """One selected key gives out = its value exactly; q = 0 gives the plain mean of the
    selected values; a hand example with logits 0 and ln 3 weights values 1/4 and 3/4."""
    r = _rng(10)
    T, H, D = 12, 2, 576
    q = r.normal(size=(T, H, D)).astype(np.float32)
    c = r.normal(size=(T, D)).astype(np.float32)
    idx = np.full((T, 4), -1, dtype=np.int32)
    idx[:, 0] = r.integers(0, T, T)
    out, lse = O.sparse_mla_prefill(q, c, idx, 0.3, mutant=mutant)
    for t in range(T):
        for h in range(H):
            assert np.array_equal(out[t, h], c[idx[t, 0], :512].astype(np.float64))
    np.testing.assert_allclose(
        lse, 0.3 * np.einsum("thd,td->th", q.astype(np.float64), c[idx[:, 0]].astype(np.float64)),
        rtol=1e-12, atol=1e-12)
    qz = np.zeros_like(q)
    idx = np.stack([np.sort(r.choice(T, 5, replace=False)) for _ in range(T)]).astype(np.int32)
    out, lse = O.sparse_mla_prefill(qz, c, idx, 0.3, mutant=mutant)
    mean = c[idx][:, :, :512].astype(np.float64).mean(axis=1)
    np.testing.assert_allclose(out, np.repeat(mean[:, None], H, 1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, math.log(5.0), rtol=1e-12)
    # hand example: MHA, one head of dim 2, scale 1
    qh = np.array([[[1.0, 0.0]]], dtype=np.float32)
    kh = np.array([[[0.0, 0.0]], [[math.log(3.0), 0.0]]], dtype=np.float32)
    vh = np.array([[[1.0, 2.0]], [[5.0, -2.0]]], dtype=np.float32)
    q2 = np.concatenate([qh, qh])
    out, lse = O.sparse_mha(q2, kh, vh, np.array([[0, 1], [0, 1]], np.int32), 1.0,
                            mutant=mutant)
    np.testing.assert_allclose(out[1, 0], [4.0, -1.0], rtol=1e-6)
    np.testing.assert_allclose(lse[1, 0], math.log(4.0), rtol=1e-6)


def pin_decode_attention_equals_prefill(mutant=0):
    """Decode through a page table equals prefill attention on the contiguous rows."""
    r = _rng(11)
    L, P, H, D = 100, 16, 2, 576
    max_pages = (L + P - 1) // P
    q = (0.5 * r.normal(size=(1, H, D))).astype(np.float32)
    c = (0.5 * r.normal(size=(L, D))).astype(np.float32)
    perm = r.permutation(max_pages + 2)[:max_pages].astype(np.int32)
    pool = np.zeros((max_pages + 2, P, D), dtype=np.float32)
    for s in range(L):
        pool[perm[s // P], s % P] = c[s]
    idx = np.sort(r.choice(L, 30, replace=False)).astype(np.int32)[None, :]
    a, la = O.sparse_mla_decode(q, pool, perm[None, :], idx, 192 ** -0.5, mutant=mutant)
    b, lb = O.sparse_mla_prefill(q, c, idx, 192 ** -0.5, mutant=mutant)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


# ---------------------------------------------------------------------------------
# IndexCache and causality
# ---------------------------------------------------------------------------------
def pin_index_cache_reuse(mutant=0):
    """S layers receive exactly the indices of the nearest preceding F layer; each S
    layer's output equals attention with those indices; F layers recompute."""
    r = _rng(12)
    T, k, H, D = 48, 8, 2, 576
    pattern = "FSSFS"
    layers = []
    for ch in pattern:
        L = {"q": (0.5 * r.normal(size=(T, H, D))).astype(np.float32),
             "kv": (0.5 * r.normal(size=(T, D))).astype(np.float32)}
        if ch == "F":
            L["q_idx"] = r.integers(-4, 5, (T, 4, 16)).astype(np.float32)
            L["k_idx"] = r.integers(-4, 5, (T, 16)).astype(np.float32)
            L["w"] = r.integers(1, 4, (T, 4)).astype(np.float32)
        layers.append(L)
    outs, _, idxs = O.layer_stack(pattern, layers, k, 0.1, mutant=mutant)
    assert np.array_equal(idxs[1], idxs[0]) and np.array_equal(idxs[2], idxs[0])
    assert np.array_equal(idxs[4], idxs[3])
    assert not np.array_equal(idxs[3], idxs[0])
    for l in (1, 2):
        o, _ = O.sparse_mla_prefill(layers[l]["q"], layers[l]["kv"], idxs[0], 0.1,
                                    mutant=mutant)
        assert np.array_equal(o, outs[l])
    assert O.pattern_from_freq(4, 9) == "FSSSFSSSF"
    assert O.pattern_from_freq(1, 3) == "FFF"


def pin_causal_prefix_invariance(mutant=0):
    """Appending tokens changes nothing on the shared prefix (a causal negative control,
    as in the llm-atlas deepseek probes): rows < T of a length-T run equal those of a
    length-(T+D) run bit for bit."""
    r = _rng(13)
    T, Dx, k = 60, 25, 10
    q_idx = r.integers(-4, 5, (T + Dx, 4, 16)).astype(np.float32)
    k_idx = r.integers(-4, 5, (T + Dx, 16)).astype(np.float32)
    w = r.integers(1, 4, (T + Dx, 4)).astype(np.float32)
    a = O.prefill_indices(q_idx[:T], k_idx[:T], w[:T], k, mutant=mutant)
    b = O.prefill_indices(q_idx, k_idx, w, k, mutant=mutant)
    assert np.array_equal(a, b[:T])
    # the diagonal is selectable: a row whose only positive score is its own key picks it
    q1 = np.zeros((3, 1, 2), np.float32); q1[2, 0] = [1, 0]
    k1 = np.array([[-1, 0], [-1, 0], [1, 0]], np.float32)
    w1 = np.ones((3, 1), np.float32)
    assert O.prefill_indices(q1, k1, w1, 1, mutant=mutant)[2, 0] == 2



# ---------------------------------------------------------------------------------
# fp8 (E4M3) latent cache
# ---------------------------------------------------------------------------------
def _torch_e4m3_values(codes):
    """Library decode of E4M3 codes (torch.float8_e4m3fn) as float64."""
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def pin_e4m3_decode(mutant=0):
    """Every one of the 256 codes decodes to torch.float8_e4m3fn's value (NaN codes
    0x7f/0xff included), and a few codes to the closed forms of the format: 0x01 is the
    smallest subnormal 2^-9, 0x08 the smallest normal 2^-6, 0x38 is 1, 0x7e is 448."""
    codes = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(codes, mutant)
    t = _torch_e4m3_values(codes)
    assert np.array_equal(np.isnan(v), np.isnan(t))
    fin = ~np.isnan(t)
    assert np.array_equal(v[fin], t[fin])
    assert np.array_equal(np.signbit(v[fin]), np.signbit(t[fin]))
    forms = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x3C: 1.5, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0}
    for c, val in forms.items():
        assert O.e4m3_decode(np.array([c], np.uint8), mutant)[0] == val, hex(c)
    assert np.isnan(O.e4m3_decode(np.array([0x7F], np.uint8), mutant)[0])


def pin_e4m3_encode(mutant=0):
    """Encoding agrees with torch's float32 -> float8_e4m3fn conversion (round to nearest
    even) wherever that conversion is finite (|x| < 448 here), including values exactly
    halfway between neighbouring codes and subnormal magnitudes; brute force (the nearest
    of all finite codes, ties to the even code) agrees too; magnitudes above 448
    saturate to 448 (0x7e / 0xfe); decode(encode(v)) = v for every finite code."""
    r = _rng(30)
    pos = _torch_e4m3_values(np.arange(127, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    x = np.concatenate([
        (r.normal(size=4000) * 60).astype(np.float32),
        (r.normal(size=2000) * 2.0 ** -8).astype(np.float32),
        mids, -mids, pos.astype(np.float32), np.float32([0.0, -0.0, 447.9, -447.9])])
    x = x[np.abs(x) < 448]
    c = O.e4m3_encode(x, mutant)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(c, t), np.nonzero(c != t)
    allv = _torch_e4m3_values(np.arange(256, dtype=np.uint8))
    fin_codes = np.nonzero(~np.isnan(allv))[0]
    xs = x[:600].astype(np.float64)
    d = np.abs(xs[:, None] - allv[fin_codes][None, :])
    best = d.min(axis=1, keepdims=True)
    for i in range(len(xs)):
        cand = fin_codes[d[i] == best[i, 0]]
        cand = cand[np.signbit(allv[cand]) == np.signbit(xs[i])] if len(cand) > 1 else cand
        want = cand[(cand & 1) == 0][0] if len(cand) > 1 else cand[0]
        assert c[i] == want, (xs[i], c[i], want)
    sat = O.e4m3_encode(np.float32([449.0, 500.0, 1e6, -464.0, -3e38]), mutant)
    assert sat.tolist() == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    fin = np.nonzero(~np.isnan(allv))[0].astype(np.uint8)
    assert np.array_equal(O.e4m3_encode(allv[fin].astype(np.float32), mutant), fin)


def pin_latent_quantize(mutant=0):
    """Quantising a bf16 latent row: the fp32 quotient c / kv_scale, then the library's
    round-to-nearest-even E4M3 conversion (values kept inside +-448)."""
    r = _rng(31)
    c = torch.from_numpy((0.5 * r.normal(size=(64, 576))).astype(np.float32)).to(torch.bfloat16)
    for s in (2.0 ** -7, 0.0123):
        got = O.latent_quantize_fp8(c, s, mutant)
        ref = (c.float() / torch.tensor(s, dtype=torch.float32)).clamp(-448, 448)
        ref = ref.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got, ref)


def pin_fp8_attention_masked_sdpa(mutant=0):
    """Attention over an fp8 latent cache equals torch SDPA (fp64) on the latent rows
    decoded by the library (torch.float8_e4m3fn) and multiplied by kv_scale, under the
    mask built from the indices; the log-sum-exp equals torch.logsumexp of the logits;
    paged decode of the last query equals its prefill row."""
    r = _rng(32)
    T, H, D, k = 70, 2, 576, 24
    q = (0.5 * r.normal(size=(T, H, D))).astype(np.float32)
    codes = torch.from_numpy((64 * r.normal(size=(T, D))).clip(-440, 440).astype(np.float32))
    codes = codes.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    idx = np.full((T, k), -1, dtype=np.int32)
    mask = np.zeros((T, T), dtype=bool)
    for t in range(T):
        sel = np.sort(r.choice(t + 1, size=min(k, t + 1), replace=False))
        idx[t, :len(sel)] = sel
        mask[t, sel] = True
    for s in (2.0 ** -7, 0.0123):
        out, lse = O.sparse_mla_fp8_prefill(q, codes, s, idx, 192 ** -0.5, mutant=mutant)
        c = _torch_e4m3_values(codes) * s
        kk = np.repeat(c[:, None, :], H, axis=1)
        ref = _sdpa64(q, kk, kk[..., :512], mask=mask, scale=192 ** -0.5)
        np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
        logits = np.einsum("thd,sd->ths", q.astype(np.float64), c) * 192 ** -0.5
        logits = np.where(mask[:, None, :], logits, -np.inf)
        ref_lse = torch.logsumexp(torch.from_numpy(logits), dim=-1).numpy()
        np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)
    # paged decode: the pool is a permutation of 64-row pages of the same codes
    ps, npg = 8, (T + 7) // 8
    pool = np.zeros((npg * ps, D), np.uint8)
    pool[:T] = codes
    pool = pool.reshape(npg, ps, D)
    perm = r.permutation(npg)
    ppool = np.empty_like(pool)
    ppool[perm] = pool
    pt = perm.astype(np.int32)[None, :]
    od, ld = O.sparse_mla_fp8_decode(q[T - 1:], ppool, 0.0123, pt, idx[T - 1:], 192 ** -0.5,
                                     mutant=mutant)
    op, lp = O.sparse_mla_fp8_prefill(q[T - 1:], codes, 0.0123, idx[T - 1:], 192 ** -0.5,
                                      mutant=mutant)
    np.testing.assert_allclose(od, op, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(ld, lp, rtol=1e-12, atol=1e-15)


def pin_varlen_packed_sequences(mutant=0):
    """Packed batch of independent prompts: scores worked out per sequence with numpy
    (einsum, ReLU, head weights) and a stable full sort per row, indices shifted to packed
    rows; every selected row lies in [seq_start, t]; a gap left between sequences (left
    padding) stays at the fill value."""
    r = _rng(40)
    starts, lens = [0, 9, 30, 33], [9, 20, 0, 14]
    N, H_I, D_I, k = 50, 2, 4, 6
    q = r.integers(-3, 4, (N, H_I, D_I)).astype(np.float32)
    kk = r.integers(-3, 4, (N, D_I)).astype(np.float32)
    w = r.integers(1, 3, (N, H_I)).astype(np.float32)
    got = O.prefill_indices_varlen(q, kk, w, starts, lens, k, fill=-9, mutant=mutant)
    want = np.full((N, k), -9, np.int32)
    for s0, L in zip(starts, lens):
        for t in range(s0, s0 + L):
            keys = np.arange(s0, t + 1)
            dots = np.einsum("jd,sd->js", q[t].astype(np.float64), kk[keys].astype(np.float64))
            sc = (w[t].astype(np.float64)[:, None] * np.maximum(dots, 0)).sum(0)
            order = np.argsort(-sc, kind="stable")[:k]
            sel = np.sort(keys[order])
            want[t] = np.r_[sel, -np.ones(k - len(sel), np.int32)]
            assert np.all((got[t][got[t] >= 0] >= s0) & (got[t][got[t] >= 0] <= t))
    assert np.array_equal(got, want)

ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]
