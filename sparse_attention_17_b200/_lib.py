"""ctypes binding of libdsa.so (include/dsa.h): argument marshalling only.

Every function takes torch CUDA tensors, checks dtype/shape/contiguity, and passes raw
device pointers, sizes and the current CUDA stream to the C ABI.  All arithmetic runs in
the library's kernels; if the library is missing these functions raise -- there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
_LIB_PATH = _PKG / "libdsa.so"
_lib = None

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, \
    DSA_ERR_DEVICE_CHECK = range(6)
DSA_F32, DSA_BF16, DSA_FP8_E4M3 = 0, 1, 2
DSA_PREFILL, DSA_DECODE = 0, 1
KERNEL_INDEXER, KERNEL_TOPK, KERNEL_ATTENTION, KERNEL_COMBINE, KERNEL_QUANTIZE = range(5)
KERNEL_KINDS = 5
DEVERR_INDEX_RANGE, DEVERR_PAGE_RANGE, DEVERR_TIMEOUT = 1, 2, 4

# (name, restype, argtypes) of every exported symbol, in header order.
_P, _I, _LL, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
SYMBOLS = [
    ("dsa_status_string", ctypes.c_char_p, [_I]),
    ("dsa_last_error", ctypes.c_char_p, []),
    ("dsa_version", _I, []),
    ("dsa_indexer_scores", _I, [_I, _I, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _I, _P, _P, _LL, _P]),
    ("dsa_topk_select", _I, [_P, _LL, _I, _I, _P, _I, _I, _P, _LL, _P]),
    ("dsa_index_select", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _LL, _P, _SZ, _P]),
    ("dsa_index_select_workspace_size", _SZ, [_I, _I]),
    ("dsa_sparse_mla_fwd", _I, [_I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _LL, _P, _I, _I, _P,
                                _P, _I, _LL, _P, _P, _P, _SZ, _P]),
    ("dsa_sparse_mla_workspace_size", _SZ, [_I, _I, _I, _I, _I]),
    ("dsa_sparse_mla_decode_noalloc", _I, [_I, _I, _I, _I, _F, _P, _P, _LL, _P, _I, _I, _P, _P, _I,
                                           _LL, _P, _P, _P]),
    ("dsa_index_varlen", _I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _LL, _P, _SZ, _P]),
    ("dsa_index_varlen_workspace_size", _SZ, [_I, _I]),
    ("dsa_sparse_mla_fp8_fwd", _I, [_I, _I, _I, _I, _I, _F, _F, _P, _P, _LL, _P, _I, _I, _P, _P,
                                    _I, _LL, _P, _P, _P, _SZ, _P]),
    ("dsa_latent_quantize_fp8", _I, [_P, _LL, _F, _P, _P]),
    ("dsa_layer_stack", _I, [ctypes.c_char_p, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P,
                             _P, _P, _P, _P, _P, _SZ, _P]),
    ("dsa_layer_stack_workspace_size", _SZ, [_I, _I]),
    ("dsa_pattern_from_freq", _I, [_I, _I, ctypes.c_char_p, _I]),
    ("dsa_selftest_wait_timeout", _I, [_P, _P]),
    ("dsa_check_device_errors", _I, [_P, ctypes.POINTER(ctypes.c_uint)]),
    ("dsa_launch_count", _LL, [_I]),
    ("dsa_reset_launch_counts", None, []),
]


class DSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(what)


def lib_path() -> Path:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Loads libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not _LIB_PATH.exists():
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m sparse_attention_17_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(str(_LIB_PATH))
    for name, res, args in SYMBOLS:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != DSA_OK:
        lib = load()
        raise DSAError(status, f"{lib.dsa_status_string(status).decode()}: "
                               f"{lib.dsa_last_error().decode()}")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t, dtype, ndim, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _scratch(workspace) -> tuple[int | None, int]:
    """(pointer, bytes) of an optional workspace: a contiguous CUDA tensor of any dtype."""
    if workspace is None:
        return None, 0
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda \
            or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def _dt(t) -> int:
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype == torch.float32:
        return DSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------------------------
def indexer_scores(q_idx, k_idx, w, scores, q_begin: int = 0, rows: int | None = None,
                   page_table=None, seq_lens=None) -> None:
    """dsa_indexer_scores.  Prefill: q_idx [T,H_I,D_I], k_idx [S,D_I], w [T,H_I],
    scores [rows, ld].  Decode (page_table given): q_idx [B,H_I,D_I], k_idx pool
    [num_pages,page_size,D_I], page_table [B,max_pages], seq_lens [B], scores [B, ld]."""
    lib = load()
    dt = _dt(q_idx)
    _need(q_idx, q_idx.dtype, 3, "q_idx")
    _need(w, torch.float32, 2, "w")
    _need(scores, torch.float32, 2, "scores")
    H_I, D_I = q_idx.shape[1], q_idx.shape[2]
    if page_table is None:
        _need(k_idx, q_idx.dtype, 2, "k_idx")
        if rows is None:
            rows = q_idx.shape[0] - q_begin
        S = k_idx.shape[0]
        _check(lib.dsa_indexer_scores(dt, DSA_PREFILL, q_idx.data_ptr(), k_idx.data_ptr(),
                                      w.data_ptr(), H_I, D_I, q_begin, rows, S, None, 0, 0, None,
                                      scores.data_ptr(), scores.stride(0), _stream()))
    else:
        _need(k_idx, q_idx.dtype, 3, "k_idx")
        _need(page_table, torch.int32, 2, "page_table")
        _need(seq_lens, torch.int32, 1, "seq_lens")
        B = q_idx.shape[0]
        page_size = k_idx.shape[1]
        S = k_idx.shape[0] * page_size
        _check(lib.dsa_indexer_scores(dt, DSA_DECODE, q_idx.data_ptr(), k_idx.data_ptr(),
                                      w.data_ptr(), H_I, D_I, 0, B, S, page_table.data_ptr(),
                                      page_table.shape[1], page_size, seq_lens.data_ptr(),
                                      scores.data_ptr(), scores.stride(0), _stream()))


def topk_select(scores, k: int, idx, q_begin: int = 0, rows: int | None = None, row_len=None,
                max_len: int | None = None) -> None:
    """dsa_topk_select.  Causal rows (row_len None): row r has q_begin+r+1 valid scores;
    otherwise row r has row_len[r]."""
    lib = load()
    _need(scores, torch.float32, 2, "scores")
    _need(idx, torch.int32, 2, "idx")
    if rows is None:
        rows = scores.shape[0]
    if row_len is not None:
        _need(row_len, torch.int32, 1, "row_len")
    if max_len is None:
        max_len = scores.shape[1] if row_len is not None else q_begin + rows
    _check(lib.dsa_topk_select(scores.data_ptr(), scores.stride(0), rows, q_begin,
                               _ptr(row_len), max_len, k, idx.data_ptr(), idx.stride(0),
                               _stream()))


def index_select_workspace_size(rows_window: int, S: int) -> int:
    return load().dsa_index_select_workspace_size(rows_window, S)


def index_select(q_idx, k_idx, w, idx, k: int, workspace, q_begin: int = 0,
                 rows: int | None = None) -> None:
    """dsa_index_select: indexer + top-k of causal prefill rows without dense score rows.
    q_idx [T,16,64] bf16, k_idx [S,64] bf16, w [T,16] fp32, idx [rows, >=k] int32 (row r is
    query q_begin + r), workspace a CUDA tensor (any dtype) used as scratch."""
    lib = load()
    _need(q_idx, torch.bfloat16, 3, "q_idx")
    _need(k_idx, torch.bfloat16, 2, "k_idx")
    _need(w, torch.float32, 2, "w")
    _need(idx, torch.int32, 2, "idx")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if rows is None:
        rows = q_idx.shape[0] - q_begin
    _check(lib.dsa_index_select(q_idx.data_ptr(), k_idx.data_ptr(), w.data_ptr(), q_idx.shape[1],
                                q_idx.shape[2], q_begin, rows, k_idx.shape[0], k, idx.data_ptr(),
                                idx.stride(0), *_scratch(workspace), _stream()))


def sparse_mla_workspace_size(num_q: int, k_sel: int, decode: bool, H: int = 16,
                              D_v: int = 512) -> int:
    return load().dsa_sparse_mla_workspace_size(DSA_DECODE if decode else DSA_PREFILL, num_q, H,
                                                D_v, k_sel)


def sparse_mla_fwd(q, kv, idx, out, scale: float, lse=None, v=None, page_table=None,
                   seq_lens=None, workspace=None) -> None:
    """dsa_sparse_mla_fwd.  MLA (bf16): q [N,16,576], kv [S,576] (prefill) or page pool
    [num_pages,page_size,576] (decode, with page_table/seq_lens), out [N,16,512].
    MHA (fp32): q [T,H,D], kv (=k) [S,H,D], v [S,H,D], out [T,H,D]."""
    lib = load()
    dt = _dt(q)
    _need(q, q.dtype, 3, "q")
    _need(idx, torch.int32, 2, "idx")
    _need(out, q.dtype, 3, "out")
    if lse is not None:
        _need(lse, torch.float32, 2, "lse")
    num_q, H, D_qk = q.shape
    k_sel = idx.shape[1]
    ws_ptr, ws_bytes = _scratch(workspace)
    if v is not None:  # MHA
        _need(kv, q.dtype, 3, "k")
        _need(v, q.dtype, 3, "v")
        _check(lib.dsa_sparse_mla_fwd(dt, DSA_PREFILL, num_q, H, kv.shape[1], D_qk, v.shape[2],
                                      scale, q.data_ptr(), kv.data_ptr(), v.data_ptr(),
                                      kv.shape[0], None, 0, 0, None, idx.data_ptr(), k_sel,
                                      idx.stride(0), out.data_ptr(), _ptr(lse), ws_ptr, ws_bytes,
                                      _stream()))
        return
    D_v = out.shape[2]
    if page_table is None:
        _need(kv, q.dtype, 2, "kv")
        _check(lib.dsa_sparse_mla_fwd(dt, DSA_PREFILL, num_q, H, 1, D_qk, D_v, scale,
                                      q.data_ptr(), kv.data_ptr(), None, kv.shape[0], None, 0, 0,
                                      None, idx.data_ptr(), k_sel, idx.stride(0), out.data_ptr(),
                                      _ptr(lse), ws_ptr, ws_bytes, _stream()))
    else:
        _need(kv, q.dtype, 3, "kv")
        _need(page_table, torch.int32, 2, "page_table")
        _need(seq_lens, torch.int32, 1, "seq_lens")
        page_size = kv.shape[1]
        _check(lib.dsa_sparse_mla_fwd(dt, DSA_DECODE, num_q, H, 1, D_qk, D_v, scale,
                                      q.data_ptr(), kv.data_ptr(), None, kv.shape[0] * page_size,
                                      page_table.data_ptr(), page_table.shape[1], page_size,
                                      seq_lens.data_ptr(), idx.data_ptr(), k_sel, idx.stride(0),
                                      out.data_ptr(), _ptr(lse), ws_ptr, ws_bytes, _stream()))


def sparse_mla_fp8_fwd(q, kv, kv_scale: float, idx, out, scale: float, lse=None,
                       page_table=None, seq_lens=None, workspace=None) -> None:
    """dsa_sparse_mla_fp8_fwd.  q [N,16,576] bf16; kv uint8 E4M3 codes [S,576] (prefill)
    or page pool [num_pages,page_size,576] (decode, with page_table/seq_lens); latent
    value = kv_scale * code; out [N,16,512] bf16."""
    lib = load()
    _need(q, torch.bfloat16, 3, "q")
    _need(idx, torch.int32, 2, "idx")
    _need(out, torch.bfloat16, 3, "out")
    if lse is not None:
        _need(lse, torch.float32, 2, "lse")
    num_q, H, D_qk = q.shape
    D_v = out.shape[2]
    k_sel = idx.shape[1]
    ws_ptr, ws_bytes = _scratch(workspace)
    if page_table is None:
        _need(kv, torch.uint8, 2, "kv")
        _check(lib.dsa_sparse_mla_fp8_fwd(DSA_PREFILL, num_q, H, D_qk, D_v, scale, kv_scale,
                                          q.data_ptr(), kv.data_ptr(), kv.shape[0], None, 0, 0,
                                          None, idx.data_ptr(), k_sel, idx.stride(0),
                                          out.data_ptr(), _ptr(lse), ws_ptr, ws_bytes, _stream()))
    else:
        _need(kv, torch.uint8, 3, "kv")
        _need(page_table, torch.int32, 2, "page_table")
        _need(seq_lens, torch.int32, 1, "seq_lens")
        page_size = kv.shape[1]
        _check(lib.dsa_sparse_mla_fp8_fwd(DSA_DECODE, num_q, H, D_qk, D_v, scale, kv_scale,
                                          q.data_ptr(), kv.data_ptr(), kv.shape[0] * page_size,
                                          page_table.data_ptr(), page_table.shape[1], page_size,
                                          seq_lens.data_ptr(), idx.data_ptr(), k_sel,
                                          idx.stride(0), out.data_ptr(), _ptr(lse), ws_ptr,
                                          ws_bytes, _stream()))


def index_varlen_workspace_size(max_seq_len: int, rows_window: int = 0) -> int:
    return load().dsa_index_varlen_workspace_size(max_seq_len, rows_window)


def index_varlen(q_idx, k_idx, w, seq_start, seq_len, k: int, idx, workspace) -> None:
    """dsa_index_varlen: packed sequences (host lists seq_start / seq_len) of q_idx
    [N,16,64], k_idx [N,64], w [N,16]; idx [N, >=k] receives packed-row indices."""
    lib = load()
    _need(q_idx, torch.bfloat16, 3, "q_idx")
    _need(k_idx, torch.bfloat16, 2, "k_idx")
    _need(w, torch.float32, 2, "w")
    _need(idx, torch.int32, 2, "idx")
    n = len(seq_start)
    if len(seq_len) != n:
        raise ValueError("seq_start and seq_len must have the same length")
    arr = ctypes.c_int * max(n, 1)
    starts, lens = arr(*[int(v) for v in seq_start]), arr(*[int(v) for v in seq_len])
    _check(lib.dsa_index_varlen(q_idx.data_ptr(), k_idx.data_ptr(), w.data_ptr(), q_idx.shape[1],
                                q_idx.shape[2], q_idx.shape[0], n,
                                ctypes.cast(starts, ctypes.c_void_p),
                                ctypes.cast(lens, ctypes.c_void_p), k, idx.data_ptr(),
                                idx.stride(0), *_scratch(workspace), _stream()))


def selftest_wait_timeout(gave_up) -> None:
    """dsa_selftest_wait_timeout: gave_up is a 1-element int32 CUDA tensor."""
    _need(gave_up, torch.int32, 1, "gave_up")
    _check(load().dsa_selftest_wait_timeout(gave_up.data_ptr(), _stream()))


def latent_quantize_fp8(src, kv_scale: float, dst) -> None:
    """dsa_latent_quantize_fp8: dst (uint8, same shape) = E4M3(src (bf16) / kv_scale)."""
    lib = load()
    _need(src, torch.bfloat16, None, "src")
    _need(dst, torch.uint8, None, "dst")
    if src.numel() != dst.numel():
        raise ValueError("src and dst must have the same number of elements")
    _check(lib.dsa_latent_quantize_fp8(src.data_ptr(), src.numel(), kv_scale, dst.data_ptr(),
                                       _stream()))


def layer_stack_workspace_size(T: int, rows_window: int = 0) -> int:
    return load().dsa_layer_stack_workspace_size(T, rows_window)


def layer_stack(pattern: str, layers: list[dict], idx_buf, workspace, topk: int, scale: float,
                outs: list, lses: list | None = None) -> None:
    """dsa_layer_stack.  layers[l]: dict with 'q' [T,16,576], 'kv' [T,576] and, for 'F'
    layers, 'q_idx' [T,16,64], 'k_idx' [T,64], 'w' [T,16]; outs[l] [T,16,512] bf16."""
    lib = load()
    n = len(pattern)
    if len(layers) != n or len(outs) != n:
        raise ValueError("one layer dict and one output per pattern character")
    T = layers[0]["q"].shape[0]
    arr = ctypes.c_void_p * n

    def ptrs(key, src):
        return arr(*[(src[l][key].data_ptr() if (src[l] is not None and key in src[l]) else None)
                     for l in range(n)])

    for l, L in enumerate(layers):
        _need(L["q"], torch.bfloat16, 3, f"layers[{l}].q")
        _need(L["kv"], torch.bfloat16, 2, f"layers[{l}].kv")
        _need(outs[l], torch.bfloat16, 3, f"outs[{l}]")
        if pattern[l] == "F":
            _need(L["q_idx"], torch.bfloat16, 3, f"layers[{l}].q_idx")
            _need(L["k_idx"], torch.bfloat16, 2, f"layers[{l}].k_idx")
            _need(L["w"], torch.float32, 2, f"layers[{l}].w")
    _need(idx_buf, torch.int32, 2, "idx_buf")
    q_idx = ptrs("q_idx", layers)
    k_idx = ptrs("k_idx", layers)
    w = ptrs("w", layers)
    q = ptrs("q", layers)
    kv = ptrs("kv", layers)
    for l, x in enumerate(lses or []):
        if x is not None:
            _need(x, torch.float32, 2, f"lses[{l}]")
    out = arr(*[o.data_ptr() for o in outs])
    lse = arr(*[(x.data_ptr() if x is not None else None) for x in lses]) if lses else None
    _check(lib.dsa_layer_stack(pattern.encode(), n, T, topk, 16, 64, 16, 576, 512, scale,
                               q_idx, k_idx, w, q, kv, out, lse, idx_buf.data_ptr(),
                               *_scratch(workspace), _stream()))


def pattern_from_freq(freq: int, num_layers: int) -> str:
    buf = ctypes.create_string_buffer(num_layers + 1)
    _check(load().dsa_pattern_from_freq(freq, num_layers, buf, num_layers + 1))
    return buf.value.decode()


def check_device_errors() -> int:
    """Synchronizes the current stream and returns (and clears) the device error bits."""
    bits = ctypes.c_uint(0)
    st = load().dsa_check_device_errors(_stream(), ctypes.byref(bits))
    if st not in (DSA_OK, DSA_ERR_DEVICE_CHECK):
        _check(st)
    return bits.value


def launch_count(kind: int) -> int:
    return load().dsa_launch_count(kind)


def reset_launch_counts() -> None:
    load().dsa_reset_launch_counts()
