"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol
include/dsa.h declares, and rejects bad arguments before launching anything."""
import ctypes
import re
from pathlib import Path

import pytest

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import _lib
from oracle import oracle as O

HEADER = Path(__file__).resolve().parents[1] / "include" / "dsa.h"


def _declared():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return dsa.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"libdsa.so does not export {n}"
    bound = {n for n, _, _ in _lib.SYMBOLS}
    assert set(names) <= bound, set(names) - bound


def test_version_and_status_strings(lib):
    assert lib.dsa_version() >> 16 == 1
    for code, name in enumerate(["DSA_OK", "DSA_ERR_INVALID_ARG", "DSA_ERR_UNSUPPORTED",
                                 "DSA_ERR_WORKSPACE", "DSA_ERR_CUDA", "DSA_ERR_DEVICE_CHECK"]):
        assert lib.dsa_status_string(code).decode() == name
    assert lib.dsa_status_string(99).decode() == "DSA_ERR_UNKNOWN"


@pytest.mark.parametrize("freq,n", [(1, 5), (2, 7), (3, 27), (4, 61), (100, 3)])
def test_pattern_from_freq_matches_oracle_reading(freq, n):
    assert dsa.pattern_from_freq(freq, n) == O.pattern_from_freq(freq, n)


def test_pattern_from_freq_rejects(lib):
    buf = ctypes.create_string_buffer(4)
    assert lib.dsa_pattern_from_freq(0, 3, buf, 4) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_pattern_from_freq(2, 4, buf, 4) == _lib.DSA_ERR_INVALID_ARG  # no room for NUL


def _arr(n, v=16):
    return (ctypes.c_void_p * n)(*([v] * n))


@pytest.mark.parametrize("pattern,n,msg", [
    (b"SFF", 3, "start"),
    (b"FXS", 3, "not F or S"),
    (b"FS", 3, "length"),
    (b"", 0, "empty"),
])
def test_layer_stack_rejects_bad_patterns(lib, pattern, n, msg):
    a = _arr(max(n, 1))
    st = lib.dsa_layer_stack(pattern, n, 128, 64, 16, 64, 16, 576, 512, 0.1, a, a, a, a, a, a,
                             None, 16, 16, 1 << 20, None)
    assert st == _lib.DSA_ERR_INVALID_ARG
    assert msg in lib.dsa_last_error().decode()


def test_layer_stack_rejects_missing_indexer_inputs_of_f_layer(lib):
    a = _arr(3)
    none = (ctypes.c_void_p * 3)(16, 16, None)
    st = lib.dsa_layer_stack(b"FSF", 3, 128, 64, 16, 64, 16, 576, 512, 0.1, none, a, a, a, a, a,
                             None, 16, 16, 1 << 20, None)
    assert st == _lib.DSA_ERR_INVALID_ARG and "F layer 2" in lib.dsa_last_error().decode()
    # S layers may pass NULL indexer inputs: this one fails later, on the workspace
    none_s = (ctypes.c_void_p * 3)(16, None, None)
    st = lib.dsa_layer_stack(b"FSS", 3, 128, 64, 16, 64, 16, 576, 512, 0.1, none_s, none_s,
                             none_s, a, a, a, None, 16, 16, 64, None)
    assert st == _lib.DSA_ERR_WORKSPACE


def test_layer_stack_rejects_unsupported_shapes(lib):
    a = _arr(1)
    st = lib.dsa_layer_stack(b"F", 1, 128, 64, 2, 16, 4, 32, 32, 0.1, a, a, a, a, a, a, None,
                             16, 16, 1 << 20, None)
    assert st == _lib.DSA_ERR_UNSUPPORTED


def test_indexer_rejects_null_and_misaligned(lib):
    st = lib.dsa_indexer_scores(1, 0, None, 16, 16, 16, 64, 0, 8, 8, None, 0, 0, None, 16, 8, None)
    assert st == _lib.DSA_ERR_INVALID_ARG
    st = lib.dsa_indexer_scores(1, 0, 18, 16, 16, 16, 64, 0, 8, 8, None, 0, 0, None, 16, 8, None)
    assert st == _lib.DSA_ERR_INVALID_ARG and "aligned" in lib.dsa_last_error().decode()
    st = lib.dsa_indexer_scores(1, 0, 16, 16, 16, 16, 64, 0, 8, 8, None, 0, 0, None, 16, 6, None)
    assert st == _lib.DSA_ERR_INVALID_ARG and "multiple of 4" in lib.dsa_last_error().decode()
    # zero rows is a valid no-op and touches no device
    assert lib.dsa_indexer_scores(1, 0, 16, 16, 16, 16, 64, 0, 0, 8, None, 0, 0, None, 16, 8,
                                  None) == _lib.DSA_OK


def test_topk_rejects(lib):
    assert lib.dsa_topk_select(16, 64, 4, 0, None, 64, 0, 16, 4, None) == _lib.DSA_ERR_UNSUPPORTED
    assert lib.dsa_topk_select(16, 64, 4, 0, None, 64, 5000, 16, 5000, None) == _lib.DSA_ERR_UNSUPPORTED
    assert lib.dsa_topk_select(16, 64, 4, 0, None, 64, 8, 16, 4, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk_select(16, 32, 4, 0, None, 64, 8, 16, 8, None) == _lib.DSA_ERR_INVALID_ARG
    # causal rows beyond max_len
    assert lib.dsa_topk_select(16, 64, 70, 0, None, 64, 8, 16, 8, None) == _lib.DSA_ERR_INVALID_ARG
    # score rows must start on 16-byte boundaries (ld a multiple of 4)
    assert lib.dsa_topk_select(16, 66, 4, 0, None, 64, 8, 16, 8, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk_select(16, 64, 0, 0, None, 64, 8, 16, 8, None) == _lib.DSA_OK


def test_attention_rejects(lib):
    f = lib.dsa_sparse_mla_fwd
    # null q
    assert f(1, 0, 4, 16, 1, 576, 512, 0.1, None, 16, None, 8, None, 0, 0, None, 16, 4, 4, 16,
             None, None, 0, None) == _lib.DSA_ERR_INVALID_ARG
    # ld_idx < k_sel
    assert f(1, 0, 4, 16, 1, 576, 512, 0.1, 16, 16, None, 8, None, 0, 0, None, 16, 4, 2, 16,
             None, None, 0, None) == _lib.DSA_ERR_INVALID_ARG
    # non-positive scale
    assert f(1, 0, 4, 16, 1, 576, 512, 0.0, 16, 16, None, 8, None, 0, 0, None, 16, 4, 4, 16,
             None, None, 0, None) == _lib.DSA_ERR_INVALID_ARG
    # empty batch is a no-op
    assert f(1, 0, 0, 16, 1, 576, 512, 0.1, 16, 16, None, 8, None, 0, 0, None, 16, 4, 4, 16,
             None, None, 0, None) == _lib.DSA_OK


def test_fp8_attention_and_quantize_reject(lib):
    f = lib.dsa_sparse_mla_fp8_fwd
    ok = (0, 4, 16, 576, 512, 0.1, 0.01, 16, 16, 8, None, 0, 0, None, 16, 4, 4, 16, None, None,
          0, None)
    # kv_scale must be finite and positive
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        a = list(ok)
        a[6] = bad
        assert f(*a) == _lib.DSA_ERR_INVALID_ARG and "kv_scale" in lib.dsa_last_error().decode()
    a = list(ok)
    a[7] = None  # null q
    assert f(*a) == _lib.DSA_ERR_INVALID_ARG
    a = list(ok)
    a[1] = 0  # empty batch: no-op before any device work
    assert f(*a) == _lib.DSA_OK
    # the bf16 entry point refuses an fp8 dtype (no scale to apply)
    g = lib.dsa_sparse_mla_fwd
    assert g(2, 0, 4, 16, 1, 576, 512, 0.1, 16, 16, None, 8, None, 0, 0, None, 16, 4, 4, 16,
             None, None, 0, None) == _lib.DSA_ERR_INVALID_ARG
    q = lib.dsa_latent_quantize_fp8
    assert q(16, 0, 0.01, 16, None) == _lib.DSA_OK
    assert q(16, -1, 0.01, 16, None) == _lib.DSA_ERR_INVALID_ARG
    assert q(None, 8, 0.01, 16, None) == _lib.DSA_ERR_INVALID_ARG
    assert q(18, 8, 0.01, 16, None) == _lib.DSA_ERR_INVALID_ARG
    assert q(16, 8, 0.0, 16, None) == _lib.DSA_ERR_INVALID_ARG


def test_index_varlen_rejects(lib):
    f = lib.dsa_index_varlen
    arr = ctypes.c_int * 3

    def call(starts, lens, n=100, k=8, ld=8, ws_bytes=1 << 20, H_I=16):
        return f(16, 16, 16, H_I, 64, n, len(starts), ctypes.cast(arr(*starts), ctypes.c_void_p),
                 ctypes.cast(arr(*lens), ctypes.c_void_p), k, 16, ld, 16, ws_bytes, None)

    assert call([0, 10], [20, 5]) == _lib.DSA_ERR_INVALID_ARG    # overlap
    assert call([0, 90], [20, 20]) == _lib.DSA_ERR_INVALID_ARG   # past num_tokens
    assert call([5, 0], [2, 2]) == _lib.DSA_ERR_INVALID_ARG      # not increasing
    assert call([0], [-1]) == _lib.DSA_ERR_INVALID_ARG           # negative length
    assert call([0], [10], k=0) == _lib.DSA_ERR_UNSUPPORTED
    assert call([0], [10], ld=4) == _lib.DSA_ERR_INVALID_ARG     # ld_idx < k
    assert call([0], [10], H_I=2) == _lib.DSA_ERR_UNSUPPORTED
    assert call([0], [10], ws_bytes=16) == _lib.DSA_ERR_WORKSPACE
    assert call([0, 3], [0, 0]) == _lib.DSA_OK                   # nothing to do
    assert lib.dsa_index_varlen_workspace_size(100, 7) == 7 * 100 * 4
    assert lib.dsa_index_varlen_workspace_size(65536, 0) == 4096 << 20


def test_selftest_rejects_bad_pointer(lib):
    assert lib.dsa_selftest_wait_timeout(None, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_selftest_wait_timeout(18, None) == _lib.DSA_ERR_INVALID_ARG


def test_workspace_sizes(lib):
    assert lib.dsa_sparse_mla_workspace_size(0, 100, 16, 512, 2048) == 0
    ws = lib.dsa_sparse_mla_workspace_size(1, 64, 16, 512, 2048)
    assert ws > 0 and ws % (64 * 16 * 513 * 4) == 0
    assert lib.dsa_layer_stack_workspace_size(65536, 0) == 4096 << 20
    assert lib.dsa_layer_stack_workspace_size(1000, 0) == 1000 * 1000 * 4
    assert lib.dsa_layer_stack_workspace_size(100, 16) == 16 * 100 * 4


def test_launch_counters_reset(lib):
    dsa.reset_launch_counts()
    for k in range(5):
        assert dsa.launch_count(k) == 0
    assert dsa.launch_count(9) == -1


def test_index_select_rejects_and_sizes(lib):
    f = lib.dsa_index_select
    # null tensors, unsupported shapes, bad k / ld_idx, keys beyond S: refused before any launch
    assert f(None, 16, 16, 16, 64, 0, 8, 64, 8, 16, 8, 256, 1 << 20, None) == _lib.DSA_ERR_INVALID_ARG
    assert f(16, 16, 16, 2, 16, 0, 8, 64, 8, 16, 8, 256, 1 << 20, None) == _lib.DSA_ERR_UNSUPPORTED
    assert f(16, 16, 16, 16, 64, 0, 8, 64, 0, 16, 8, 256, 1 << 20, None) == _lib.DSA_ERR_UNSUPPORTED
    assert f(16, 16, 16, 16, 64, 0, 8, 64, 8, 16, 6, 256, 1 << 20, None) == _lib.DSA_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 64, 60, 8, 64, 8, 16, 8, 256, 1 << 20, None) == _lib.DSA_ERR_INVALID_ARG
    # workspace: null / misaligned refused; too small for 16 rows refused
    assert f(16, 16, 16, 16, 64, 0, 64, 64, 8, 16, 8, None, 1 << 20, None) == _lib.DSA_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 64, 0, 64, 64, 8, 16, 8, 272, 1 << 30, None) == _lib.DSA_ERR_INVALID_ARG
    small = lib.dsa_index_select_workspace_size(8, 65536)
    assert f(16, 16, 16, 16, 64, 0, 4096, 65536, 8, 16, 8, 256, small, None) == _lib.DSA_ERR_WORKSPACE
    # zero rows is a no-op
    assert f(16, 16, 16, 16, 64, 0, 0, 64, 8, 16, 8, 256, 1 << 20, None) == _lib.DSA_OK
    # the scratch grows with the window and the key count
    a = lib.dsa_index_select_workspace_size(16, 8192)
    assert 0 < a < lib.dsa_index_select_workspace_size(32, 8192) < lib.dsa_index_select_workspace_size(32, 65536)
    assert lib.dsa_index_select_workspace_size(0, 8192) == 0


def test_binding_refuses_host_tensors_before_the_library():
    """Host (CPU) tensors never reach a kernel: the binding raises first."""
    import torch
    with pytest.raises(ValueError):
        dsa.latent_quantize_fp8(torch.zeros(8, dtype=torch.bfloat16), 0.01,
                                torch.zeros(8, dtype=torch.uint8))
    with pytest.raises(ValueError):
        _lib._scratch(torch.zeros(16))
    assert _lib._scratch(None) == (None, 0)
