"""The allocation-free dense FFN entry point (dense_ffn_fwd_noalloc).

Some callers cannot allocate device memory when they call into the library,
for example a runtime whose pool owns all device memory.  This entry point
keeps the hidden activations in a fixed array inside the library instead of a
caller buffer.  The test calls it through the C ABI twice in a row and checks
each result against dense_ffn_fwd with a caller-provided buffer.  It lives in
a file that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

from activation_sparse_gated_tma_b200 import twell as tw
from activation_sparse_gated_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ELEMS = 16 << 20


def _noalloc():
    L = tw.lib()
    f = L.dense_ffn_fwd_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, I, I, I, P, P]
    f.restype = I
    return L, f


def _inputs(M, K, N, seed):
    w = wl.Workload(f"noalloc_{M}", M, K, N, 128, 8, seed, p_mean=0.05)
    d = wl.generate(w)
    return [torch.from_numpy(d[k].view(np.int16)).view(torch.bfloat16).cuda() for k in ("x", "wg_t", "wu_t", "wd")]


@pytest.mark.parametrize("M,K,N", [(512, 1024, 2048), (37, 256, 1024)])
def test_noalloc_matches_dense_ffn_twice(M, K, N):
    L, f = _noalloc()
    x, wg, wu, wd = _inputs(M, K, N, seed=M)
    ref = tw.dense_ffn(x, wg, wu, wd)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full((M, K), float("nan"), dtype=torch.float32, device="cuda")
        st = f(x.data_ptr(), wg.data_ptr(), wu.data_ptr(), wd.data_ptr(), M, K, N, y.data_ptr(), stream)
        assert st == tw.OK, (L.twell_last_error() or b"").decode()
        torch.cuda.synchronize()
        scale = float(ref.abs().max())
        torch.testing.assert_close(y, ref, rtol=1e-5, atol=1e-5 * scale, msg=f"call {call}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L, f = _noalloc()
    M, K, N = MAX_ELEMS // 1024 + 1, 256, 1024        # one row past the 16 Mi-element limit
    st = f(16, 16, 16, 16, M, K, N, 16, None)          # rejected before any pointer is used
    assert st == tw.ERR_INVALID
    assert b"exceeds the built-in scratch" in L.twell_last_error()
