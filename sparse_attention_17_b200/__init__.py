"""B200-native DeepSeek Sparse Attention hot path: lightning indexer, per-row top-k,
sparse absorbed-MLA attention and IndexCache index reuse, as sm_100a CUDA kernels behind
a C ABI (``include/dsa.h``).  The Python layer only marshals arguments; importing it
does not load the shared library (the first call does, and raises if it is missing)."""
from ._lib import (KERNEL_ATTENTION, KERNEL_COMBINE, KERNEL_INDEXER, KERNEL_KINDS,  # noqa: F401
                   KERNEL_QUANTIZE, KERNEL_TOPK, DSAError, check_device_errors, index_select,  # noqa: F401
                   index_select_workspace_size, index_varlen,
                   index_varlen_workspace_size, indexer_scores, latent_quantize_fp8,
                   launch_count, layer_stack, layer_stack_workspace_size, lib_path, load,
                   pattern_from_freq, reset_launch_counts, selftest_wait_timeout,
                   sparse_mla_fp8_fwd, sparse_mla_fwd,
                   sparse_mla_workspace_size, topk_select)
