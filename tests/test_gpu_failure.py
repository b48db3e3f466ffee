"""Failure detection without a GPU fault: a pipeline wait that never completes must turn
into an error status the host reads, and leave the context usable.  The self-test kernel
waits on an mbarrier that nothing arrives on, through the same time-bounded wait all
kernels use; afterwards a normal call must still give correct results."""
import numpy as np
import pytest
import torch

import sparse_attention_17_b200 as dsa
from sparse_attention_17_b200 import inputs as G
from oracle import oracle as O
from parity import check_close_bf16, dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    assert dsa.check_device_errors() == 0
    gave_up = torch.zeros(4, dtype=torch.int32, device="cuda")[:1]
    dsa.selftest_wait_timeout(gave_up)
    bits = dsa.check_device_errors()
    assert bits == 4, bits  # DSA_DEVERR_TIMEOUT, and nothing else
    assert int(gave_up.item()) == 1
    assert dsa.check_device_errors() == 0  # the word was cleared by the read
    # the context is intact: a small attention call still matches the oracle
    T, k = 300, 256
    d = G.mla_layer(T, seed=5)
    r = np.random.default_rng(5)
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = min(t + 1, k)
        idx[t, :n] = np.sort(r.choice(t + 1, n, replace=False))
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda")
    dsa.sparse_mla_fwd(dev(d["q"]), dev(d["kv"]), dev(torch.from_numpy(idx)), out, G.SCALE_MLA)
    ref, _ = O.sparse_mla_prefill(d["q"], d["kv"], idx, G.SCALE_MLA)
    check_close_bf16(out, ref, "after the timeout")
    assert dsa.check_device_errors() == 0
