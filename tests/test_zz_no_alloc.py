"""The allocation-free dense FFN entry point (dense_ffn_fwd_noalloc).

Some callers cannot allocate device memory when they call into the library,
for example a runtime whose memory pool owns all device memory, or an
embedding that forbids allocation while it runs.  This entry point keeps the
hidden activations (bf16 hi + lo, M x 2N values) in a fixed 32 MiB array
inside the library instead of a caller buffer.  The test calls it through the
C ABI twice in a row and checks each result against dense_ffn_fwd with a
caller-provided buffer.  One case fills the array exactly (its last element
is written); sizes past it must be rejected.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from activation_sparse_gated_tma_b200 import twell as tw
from activation_sparse_gated_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ELEMS = 16 << 20          # bf16 values in the fixed array; h needs M * 2N of them


def _inputs(M, K, N, seed):
    w = wl.Workload(f"noalloc_{M}", M, K, N, 128, 8, seed, p_mean=0.05)
    d = wl.generate(w)
    return [torch.from_numpy(d[k].view(np.int16)).view(torch.bfloat16).cuda() for k in ("x", "wg_t", "wu_t", "wd")]


@pytest.mark.parametrize("M,K,N", [(512, 1024, 2048), (37, 256, 1024), (2048, 256, 4096)])
def test_noalloc_matches_dense_ffn_twice(M, K, N):
    assert 2 * M * N <= MAX_ELEMS
    L = tw.lib()
    x, wg, wu, wd = _inputs(M, K, N, seed=M)
    ref = tw.dense_ffn(x, wg, wu, wd)
    stream = torch.cuda.current_stream().cuda_stream
    scale = float(ref.abs().max())
    for call in range(2):
        y = torch.full((M, K), float("nan"), dtype=torch.float32, device="cuda")
        st = L.dense_ffn_fwd_noalloc(x.data_ptr(), wg.data_ptr(), wu.data_ptr(), wd.data_ptr(), M, K, N,
                                     y.data_ptr(), ctypes.c_void_p(stream))
        assert st == tw.OK, (L.twell_last_error() or b"").decode()
        torch.cuda.synchronize()
        torch.testing.assert_close(y, ref, rtol=1e-5, atol=1e-5 * scale, msg=f"call {call}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = tw.lib()
    x, wg, wu, wd = _inputs(2048, 256, 4096, seed=3)   # exactly fills the array
    y = torch.zeros((2049, 256), dtype=torch.float32, device="cuda")
    # One more row than fits: rejected before any pointer is used or anything is launched.
    st = L.dense_ffn_fwd_noalloc(x.data_ptr(), wg.data_ptr(), wu.data_ptr(), wd.data_ptr(), 2049, 256, 4096,
                                 y.data_ptr(), None)
    assert st == tw.ERR_INVALID
    assert b"built-in scratch" in L.twell_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0
