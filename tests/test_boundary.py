"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/twell.h declares, and rejects invalid arguments before it
touches CUDA."""
import ctypes

import pytest

from activation_sparse_gated_tma_b200 import twell as tw


def test_library_exports_every_header_function():
    L = tw.lib()
    names = tw.header_functions()
    assert {"twell_gate_pack", "twell_ffn_fwd", "dense_ffn_fwd"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    L = tw.lib()
    for s in range(6):
        assert L.twell_status_str(s)
    assert L.twell_status_str(99) == b"unknown status"


@pytest.mark.parametrize("args", [
    (0, 256, 1024, 128, 8, 1),      # M < 1
    (64, 200, 1024, 128, 8, 1),     # K % 64
    (64, 8192, 1024, 128, 8, 1),    # K > 4096
    (64, 256, 1000, 128, 8, 1),     # N % T
    (64, 256, 1024, 64, 8, 1),      # T not in {128, 256}
    (64, 256, 1024, 128, 0, 1),     # C < 1
    (64, 256, 1024, 128, 129, 1),   # C > T
    (64, 256, 1024, 128, 8, 0),     # R_cap < 1
    (64, 256, 128 * 257, 128, 8, 1),  # N / T > 256
])
def test_buf_bytes_rejects_invalid_sizes(args):
    assert tw.lib().twell_buf_bytes(*args) == 0


def test_buf_init_layout_is_aligned_and_disjoint():
    L = tw.lib()
    M, K, N, T, C, R = 100, 256, 1024, 128, 8, 13
    nbytes = L.twell_buf_bytes(M, K, N, T, C, R)
    assert nbytes > 0
    base = 1 << 32                      # host-side pointer arithmetic only; never dereferenced
    b = tw._TwellBuf()
    assert L.twell_buf_init(ctypes.byref(b), base, nbytes, M, K, N, T, C, R) == tw.OK
    NT = N // T
    spans = [("ctrl", 64 * 4), ("counts", M * NT * 2), ("idx", M * NT * C), ("vals", M * NT * C * 4),
             ("row_slot", M * 4), ("slot_row", R * 4), ("dense_rows", R * N * 4), ("x_over", R * K * 2),
             ("h_over", R * N * 4), ("units", M * NT * 16),
             ("z", 4 * M * N * 4 + NT * 4)]  # z (M <= TWELL_SMALL_M): 4 partial-sum slots, then the tile tickets
    ranges = []
    for name, size in spans:
        p = getattr(b, name)
        assert p % 256 == 0
        assert base <= p and p + size <= base + nbytes
        ranges.append((p, p + size))
    ranges.sort()
    assert all(a[1] <= c[0] for a, c in zip(ranges, ranges[1:]))
    assert (b.M, b.K, b.N, b.T, b.C, b.R_cap) == (M, K, N, T, C, R)
    # too small / misaligned
    assert L.twell_buf_init(ctypes.byref(b), base, nbytes - 1, M, K, N, T, C, R) == tw.ERR_INVALID
    assert L.twell_buf_init(ctypes.byref(b), base + 16, nbytes, M, K, N, T, C, R) == tw.ERR_INVALID
    assert b"aligned" in L.twell_last_error()


def test_small_m_scratch_only_for_small_batches():
    L = tw.lib()
    b = tw._TwellBuf()
    for M, has_z in ((128, True), (129, False)):
        assert L.twell_buf_init(ctypes.byref(b), 1 << 32, L.twell_buf_bytes(M, 256, 1024, 128, 8, 8),
                                M, 256, 1024, 128, 8, 8) == tw.OK
        assert (b.z is not None) == has_z
    assert L.twell_buf_bytes(128, 256, 1024, 128, 8, 8) - L.twell_buf_bytes(129, 256, 1024, 128, 8, 8) > 128 * 1024 * 4 - 4096


def _fake_buf():
    L = tw.lib()
    M, K, N, T, C, R = 64, 256, 1024, 128, 8, 8
    b = tw._TwellBuf()
    assert L.twell_buf_init(ctypes.byref(b), 1 << 32, L.twell_buf_bytes(M, K, N, T, C, R), M, K, N, T, C, R) == tw.OK
    return b


def test_gate_pack_validates_before_launch():
    L = tw.lib()
    b = _fake_buf()
    x, w = 1 << 33, 1 << 34           # aligned fake device pointers: validation must fail before any use
    assert L.twell_gate_pack(None, w, 64, 256, 1024, ctypes.byref(b), None, None) == tw.ERR_INVALID
    assert L.twell_gate_pack(x + 8, w, 64, 256, 1024, ctypes.byref(b), None, None) == tw.ERR_INVALID
    assert L.twell_gate_pack(x, w, 65, 256, 1024, ctypes.byref(b), None, None) == tw.ERR_INVALID
    assert L.twell_gate_pack(x, w, 64, 256, 1024, None, None, None) == tw.ERR_INVALID
    empty = tw._TwellBuf()
    assert L.twell_gate_pack(x, w, 64, 256, 1024, ctypes.byref(empty), None, None) == tw.ERR_INVALID


def test_ffn_fwd_and_dense_validate_before_launch():
    L = tw.lib()
    b = _fake_buf()
    p = 1 << 33
    assert L.twell_ffn_fwd(p, p, p, ctypes.byref(b), 128, p, None) == tw.ERR_INVALID     # K mismatch
    assert L.twell_ffn_fwd(p, p, None, ctypes.byref(b), 256, p, None) == tw.ERR_INVALID
    assert L.twell_ffn_fwd(p, p, p, ctypes.byref(b), 256, p + 4, None) == tw.ERR_INVALID
    assert L.dense_ffn_fwd(p, p, p, p, 64, 200, 1024, p, p, None) == tw.ERR_INVALID      # K % 64
    assert L.dense_ffn_fwd(p, p, p, p, 64, 256, 1000, p, p, None) == tw.ERR_INVALID      # N % 128
    assert L.dense_ffn_fwd(p, p, p, p, 64, 256, 1024, None, p, None) == tw.ERR_INVALID
    assert L.dense_ffn_fwd_bf16h(p, p, p, p, 64, 256, 1000, p, p, None) == tw.ERR_INVALID


def test_expire_wait_hook_validates_its_limit():
    L = tw.lib()
    assert L.twell_test_expire_wait(10) == tw.ERR_INVALID
    assert L.twell_test_expire_wait(2_000_000_000) == tw.ERR_INVALID
    assert L.twell_test_expire_wait(5000) == tw.OK
    assert L.twell_test_expire_wait(0) == tw.OK       # disarm: nothing launched here


def test_bwd_slot_route_validates_its_value():
    L = tw.lib()
    for bad in (-1, 3):
        assert L.twell_bwd_slot_route(bad) == tw.ERR_INVALID
    for ok in (1, 2, 0):  # ends on the default
        assert L.twell_bwd_slot_route(ok) == tw.OK


def test_noalloc_rejects_oversize_before_any_cuda_call():
    L = tw.lib()
    p = 1 << 33
    # h needs M * 2N bf16 values; the fixed array holds 16 Mi.
    assert L.dense_ffn_fwd_noalloc(p, p, p, p, 2049, 256, 4096, p, None) == tw.ERR_INVALID
    assert b"built-in scratch" in L.twell_last_error()


def test_python_wrapper_rejects_wrong_tensors():
    import torch
    with pytest.raises(ValueError):
        tw._bf16(torch.zeros(4, 4), "x", (4, 4))          # wrong dtype / not CUDA
