"""Shared helpers of the GPU parity tests: device placement and the comparison rules.

Tolerances (floating outputs, bf16 MLA path): an element passes when
    |gpu - ref| <= 2e-2 + 1e-2 * |ref|
(max-abs 2e-2 / max-rel 1e-2 in allclose form).  Because MLA outputs are weighted means
of ~N(0, 0.5^2) values over up to 2048 keys (typical magnitude ~1e-2), that bound alone
would accept garbage, so every check also requires |gpu - ref| <= 2e-3 + 8e-3 |ref| and
relative L2 error <= 1e-2; the bf16 rounding of the inputs already fed to the oracle leaves only the
output rounding (2^-9 relative) and the bf16 probabilities fed to the PV product
(~1e-3 relative per weight, averaging out over the keys).  The fp32 path is held to
max-abs 1e-4.  Indices are compared bit for bit, except for Gaussian scores, where two
keys whose oracle scores lie within 1e-3 relative of the k-th score may swap.
"""
from __future__ import annotations

import numpy as np
import torch

ATOL, RTOL = 2e-2, 1e-2
MAX_ABS_BF16 = 2e-3
REL_L2_BF16 = 1e-2
MAX_ABS_F32 = 1e-4
NEAR_TIE_REL = 1e-3


def dev(x):
    if isinstance(x, torch.Tensor):
        return x.contiguous().cuda()
    return x


def check_close_bf16(gpu, ref, what=""):
    g = gpu.detach().float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.abs(g - r)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    assert np.all(err <= ATOL + RTOL * np.abs(r)), f"{what}: allclose fails, max err {err.max()}"
    # bf16 output rounding (2^-9 relative) and bf16 probabilities scale with |ref|; rows
    # with few keys have |ref| ~ 0.5, rows with thousands of keys ~ 1e-2
    gate = MAX_ABS_BF16 + 8e-3 * np.abs(r)
    worst = np.unravel_index(np.argmax(err - gate), err.shape)
    assert np.all(err <= gate), (f"{what}: err {err[worst]:.3e} at {worst} with ref "
                                 f"{r[worst]:.3e} (max-abs {err.max():.3e})")
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert rel <= REL_L2_BF16, f"{what}: rel-L2 {rel:.3e}"
    return float(err.max()), float(rel)


def check_close_f32(gpu, ref, what="", tol=MAX_ABS_F32):
    g = gpu.detach().float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref, dtype=np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: finiteness differs"
    err = np.abs(g[fin] - r[fin])
    assert err.size == 0 or err.max() <= tol, f"{what}: max-abs {err.max():.3e}"
    return float(err.max()) if err.size else 0.0


def check_lse(gpu, ref, what="", tol=1e-3):
    g = gpu.detach().float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref, dtype=np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: finiteness differs"
    if fin.any():
        err = np.abs(g[fin] - r[fin])
        assert err.max() <= tol, f"{what}: lse max-abs {err.max():.3e}"


def check_indices_exact(gpu_idx, ref_idx, what=""):
    g = gpu_idx.detach().cpu().numpy() if isinstance(gpu_idx, torch.Tensor) else gpu_idx
    r = np.asarray(ref_idx)
    if not np.array_equal(g, r):
        bad = np.argwhere(np.any(g != r, axis=1))[:, 0]
        i = int(bad[0])
        raise AssertionError(f"{what}: {len(bad)} rows differ; row {i}: "
                             f"gpu {g[i][:12]}... ref {r[i][:12]}...")


def check_indices_near_ties(gpu_idx, ref_idx, ref_scores_rows, n_valid, what=""):
    """Sets must have the same size, and every key in the symmetric difference must have
    an oracle score within NEAR_TIE_REL of the row's k-th oracle score."""
    g = gpu_idx.detach().cpu().numpy() if isinstance(gpu_idx, torch.Tensor) else gpu_idx
    r = np.asarray(ref_idx)
    k = r.shape[1]
    swaps = 0
    for i in range(r.shape[0]):
        gs = set(int(x) for x in g[i] if x >= 0)
        rs = set(int(x) for x in r[i] if x >= 0)
        assert len(gs) == len(rs), f"{what}: row {i} sizes {len(gs)} vs {len(rs)}"
        assert list(g[i][:len(gs)]) == sorted(gs), f"{what}: row {i} not ascending"
        assert np.all(g[i][len(gs):] == -1), f"{what}: row {i} bad padding"
        diff = gs ^ rs
        if not diff:
            continue
        sc = ref_scores_rows[i][: n_valid[i]]
        tau = np.sort(sc)[::-1][k - 1]
        for s in diff:
            assert 0 <= s < n_valid[i], f"{what}: row {i} key {s} out of range"
            assert abs(sc[s] - tau) <= NEAR_TIE_REL * abs(tau), \
                f"{what}: row {i} key {s} score {sc[s]} vs tau {tau}"
        swaps += len(diff) // 2
    return swaps
