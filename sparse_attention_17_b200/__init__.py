"""B200-native DeepSeek Sparse Attention hot path: lightning indexer, per-row top-k,
sparse absorbed-MLA attention and IndexCache index reuse, as sm_100a CUDA kernels behind
a C ABI (``include/dsa.h``).  The Python layer only marshals arguments."""
