"""Python binding of libtwell.so (include/twell.h): argument marshalling only.

Every step of the forward path runs in the library's CUDA kernels; PyTorch
provides device memory and the current stream.  There is no fallback: if the
library is missing or the device is not an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, Optional

import torch

from . import build as _build

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtwell.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "twell.h")

OK, ERR_INVALID, ERR_CAPACITY, ERR_CUDA, ERR_DEVICE_CHECK, ERR_UNSUPPORTED = range(6)


class TwellError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {message} (status {status})")
        self.status = status


class CapacityError(TwellError):
    def __init__(self, status, where, message, n_over):
        super().__init__(status, where, message)
        self.n_over = n_over


class _TwellBuf(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("counts", "idx", "vals", "dense_rows", "row_slot", "slot_row", "ctrl", "x_over", "h_over",
                 "units", "z")] + \
               [(n, ctypes.c_int) for n in ("M", "K", "N", "T", "C", "R_cap")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libtwell.so (building it first if sources are newer and nvcc exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH) or (_build.needs_build() and os.path.exists(_build.NVCC)):
        _build.build()
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m activation_sparse_gated_tma_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    IP = ctypes.POINTER(ctypes.c_int)
    BP = ctypes.POINTER(_TwellBuf)
    sig = {
        "twell_buf_bytes": (S, [I, I, I, I, I, I]),
        "twell_buf_init": (I, [BP, P, S, I, I, I, I, I, I]),
        "twell_gate_pack": (I, [P, P, I, I, I, BP, IP, P]),
        "twell_ffn_fwd": (I, [P, P, P, BP, I, P, P]),
        "twell_ffn_fused": (I, [P, P, P, P, I, I, I, BP, P, IP, P]),
        "twell_bwd_scratch_bytes": (S, [I, I, I, I, I, I]),
        "twell_ffn_bwd": (I, [P, P, P, P, BP, P, I, P, P, P, P, P, S, P]),
        "twell_bwd_slot_route": (I, [I]),
        "twell_read_status": (I, [BP, IP, IP, P]),
        "dense_ffn_fwd": (I, [P, P, P, P, I, I, I, P, P, P]),
        "dense_ffn_fwd_bf16h": (I, [P, P, P, P, I, I, I, P, P, P]),
        "dense_ffn_fwd_noalloc": (I, [P, P, P, P, I, I, I, P, P]),
        "twell_test_expire_wait": (I, [ctypes.c_longlong]),
        "twell_status_str": (ctypes.c_char_p, [I]),
        "twell_last_error": (ctypes.c_char_p, []),
        "twell_last_launch_count": (I, []),
        "twell_trace_events": (I, [P, I]),
        "twell_trace_count": (I, []),
        "twell_trace_name": (ctypes.c_char_p, [I]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    _lib = L
    return L


def header_functions() -> list:
    """Names of the functions include/twell.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:twell|dense)_\w+)\s*\(", text)))


def _check(status: int, where: str):
    if status != OK:
        L = lib()
        msg = (L.twell_last_error() or b"").decode() or L.twell_status_str(status).decode()
        raise TwellError(status, where, msg)


def last_launch_count() -> int:
    return lib().twell_last_launch_count()


class KernelTrace:
    """Brackets every kernel the library launches (on this thread) with CUDA
    events, for per-kernel device times of live runs.

        with KernelTrace(capacity=16) as tr:
            ...library calls...
        torch.cuda.synchronize(); tr.times_ms() -> [(kernel name, ms), ...]
    """

    def __init__(self, capacity: int = 16):
        self.capacity = capacity
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.events:      # torch creates the CUDA event lazily, on first record
            e.record()
        self._arr = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.events])
        self.count = 0
        self.names = []

    def __enter__(self):
        _check(lib().twell_trace_events(self._arr, self.capacity), "twell_trace_events")
        return self

    def __exit__(self, *exc):
        L = lib()
        self.count = L.twell_trace_count()
        self.names = [L.twell_trace_name(i).decode() for i in range(self.count)]
        L.twell_trace_events(None, 0)
        return False

    def times_ms(self):
        return [(self.names[i], self.events[2 * i].elapsed_time(self.events[2 * i + 1])) for i in range(self.count)]


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _bf16(t: torch.Tensor, name: str, shape) -> int:
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")
    return t.data_ptr()


class TwellBuffers:
    """TwELL activations + dense-row backup in one device allocation.

    Views (torch tensors over the same memory): counts [M][N/T] uint16 (as
    int16), idx [M][N/T][C] uint8, vals [M][N/T][C] float32, dense_rows
    [R_cap][N] float32, row_slot [M] int32, slot_row [R_cap] int32, ctrl [64] int32.
    """

    def __init__(self, M: int, K: int, N: int, T: int, C: int, R_cap: Optional[int] = None, device=None):
        L = lib()
        R_cap = R_cap if R_cap is not None else max(1, -(-M // 8))
        nbytes = L.twell_buf_bytes(M, K, N, T, C, R_cap)
        if nbytes == 0:
            raise ValueError(f"unsupported TwELL sizes M={M} K={K} N={N} T={T} C={C} R_cap={R_cap}")
        device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.storage = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.storage.data_ptr()
        self._off0 = (-base) % 256
        self.buf = _TwellBuf()
        _check(L.twell_buf_init(ctypes.byref(self.buf), base + self._off0, nbytes, M, K, N, T, C, R_cap),
               "twell_buf_init")
        self.M, self.K, self.N, self.T, self.C, self.R_cap = M, K, N, T, C, R_cap
        self.n_over_known: Optional[int] = None

    def _view(self, field: str, dtype, shape):
        off = getattr(self.buf, field) - self.storage.data_ptr()
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return self.storage[off:off + nbytes].view(dtype).view(*shape)

    @property
    def counts(self):
        return self._view("counts", torch.int16, (self.M, self.N // self.T))

    @property
    def idx(self):
        return self._view("idx", torch.uint8, (self.M, self.N // self.T, self.C))

    @property
    def vals(self):
        return self._view("vals", torch.float32, (self.M, self.N // self.T, self.C))

    @property
    def dense_rows(self):
        return self._view("dense_rows", torch.float32, (self.R_cap, self.N))

    @property
    def row_slot(self):
        return self._view("row_slot", torch.int32, (self.M,))

    @property
    def slot_row(self):
        return self._view("slot_row", torch.int32, (self.R_cap,))

    @property
    def ctrl(self):
        return self._view("ctrl", torch.int32, (64,))

    def to_host(self) -> Dict[str, "object"]:
        """Copy the TwELL arrays to host numpy (counts as uint16)."""
        import numpy as np
        return {
            "counts": self.counts.cpu().numpy().view(np.uint16),
            "idx": self.idx.cpu().numpy(),
            "vals": self.vals.cpu().numpy(),
            "dense_rows": self.dense_rows.cpu().numpy(),
            "row_slot": self.row_slot.cpu().numpy(),
            "slot_row": self.slot_row.cpu().numpy(),
            "ctrl": self.ctrl.cpu().numpy(),
        }


def gate_pack(x: torch.Tensor, wg_t: torch.Tensor, tw: TwellBuffers, sync: bool = False, stream=None) -> Optional[int]:
    """twell_gate_pack.  With sync=True returns n_over and raises CapacityError when > R_cap."""
    M, K = x.shape
    N = wg_t.shape[0]
    px = _bf16(x, "x", (M, K))
    pw = _bf16(wg_t, "wg_t", (N, K))
    L = lib()
    n_over = ctypes.c_int(-1)
    st = L.twell_gate_pack(px, pw, M, K, N, ctypes.byref(tw.buf), ctypes.byref(n_over) if sync else None,
                           _stream(stream))
    if st == ERR_CAPACITY:
        raise CapacityError(st, "twell_gate_pack", (L.twell_last_error() or b"").decode(), n_over.value)
    _check(st, "twell_gate_pack")
    tw.n_over_known = n_over.value if sync else None
    return n_over.value if sync else None


def ffn_fwd(x: torch.Tensor, wu_t: torch.Tensor, wd: torch.Tensor, tw: TwellBuffers,
            y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """twell_ffn_fwd: y [M][K] fp32 from TwELL (fused sparse up+down, then the dense-row path)."""
    M, K = x.shape
    N = wu_t.shape[0]
    if y is None:
        y = torch.empty((M, K), dtype=torch.float32, device=x.device)
    if y.dtype != torch.float32 or not y.is_contiguous() or tuple(y.shape) != (M, K):
        raise ValueError("y must be a contiguous float32 tensor of shape (M, K)")
    st = lib().twell_ffn_fwd(_bf16(x, "x", (M, K)), _bf16(wu_t, "wu_t", (N, K)), _bf16(wd, "wd", (N, K)),
                             ctypes.byref(tw.buf), K, y.data_ptr(), _stream(stream))
    _check(st, "twell_ffn_fwd")
    return y


def ffn_fused(x: torch.Tensor, wg_t: torch.Tensor, wu_t: torch.Tensor, wd: torch.Tensor, tw: TwellBuffers,
              y: Optional[torch.Tensor] = None, sync: bool = False, stream=None) -> torch.Tensor:
    """twell_ffn_fused: the whole sparse forward in one call (one persistent
    kernel after the reset for M <= TWELL_SMALL_M).  With sync=True raises
    CapacityError when the dense-row slots ran out."""
    M, K = x.shape
    N = wg_t.shape[0]
    if y is None:
        y = torch.empty((M, K), dtype=torch.float32, device=x.device)
    if y.dtype != torch.float32 or not y.is_contiguous() or tuple(y.shape) != (M, K):
        raise ValueError("y must be a contiguous float32 tensor of shape (M, K)")
    L = lib()
    n_over = ctypes.c_int(-1)
    st = L.twell_ffn_fused(_bf16(x, "x", (M, K)), _bf16(wg_t, "wg_t", (N, K)), _bf16(wu_t, "wu_t", (N, K)),
                           _bf16(wd, "wd", (N, K)), M, K, N, ctypes.byref(tw.buf), y.data_ptr(),
                           ctypes.byref(n_over) if sync else None, _stream(stream))
    if st == ERR_CAPACITY:
        raise CapacityError(st, "twell_ffn_fused", (L.twell_last_error() or b"").decode(), n_over.value)
    _check(st, "twell_ffn_fused")
    tw.n_over_known = n_over.value if sync else None
    return y


def ffn_bwd(x: torch.Tensor, wg_t: torch.Tensor, wu_t: torch.Tensor, wd: torch.Tensor, tw: TwellBuffers,
            dy: torch.Tensor, scratch: Optional[torch.Tensor] = None, stream=None):
    """twell_ffn_bwd: (dx, dwg_t, dwu_t, dwd), all fp32, from the forward's TwELL
    buffer `tw` and the upstream gradient dy [M][K] fp32."""
    M, K = x.shape
    N = wg_t.shape[0]
    if dy.dtype != torch.float32 or not dy.is_contiguous() or tuple(dy.shape) != (M, K):
        raise ValueError("dy must be a contiguous float32 tensor of shape (M, K)")
    L = lib()
    need = L.twell_bwd_scratch_bytes(M, K, N, tw.T, tw.C, tw.R_cap)
    if need == 0:
        raise ValueError("invalid sizes for twell_ffn_bwd")
    if scratch is None or scratch.numel() < need:
        scratch = torch.empty(need, dtype=torch.uint8, device=x.device)
    dx = torch.empty((M, K), dtype=torch.float32, device=x.device)
    dg, du, dd = (torch.empty((N, K), dtype=torch.float32, device=x.device) for _ in range(3))
    st = L.twell_ffn_bwd(_bf16(x, "x", (M, K)), _bf16(wg_t, "wg_t", (N, K)), _bf16(wu_t, "wu_t", (N, K)),
                         _bf16(wd, "wd", (N, K)), ctypes.byref(tw.buf), dy.data_ptr(), K, dx.data_ptr(),
                         dg.data_ptr(), du.data_ptr(), dd.data_ptr(), scratch.data_ptr(), scratch.numel(),
                         _stream(stream))
    _check(st, "twell_ffn_bwd")
    return dx, dg, du, dd


def read_status(tw: TwellBuffers, stream=None):
    """Synchronise and return (status, n_over, device_flags)."""
    n = ctypes.c_int(0)
    f = ctypes.c_int(0)
    st = lib().twell_read_status(ctypes.byref(tw.buf), ctypes.byref(n), ctypes.byref(f), _stream(stream))
    return st, n.value, f.value


def dense_ffn(x: torch.Tensor, wg_t: torch.Tensor, wu_t: torch.Tensor, wd: torch.Tensor,
              h_scratch: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None, stream=None,
              bf16_h: bool = False) -> torch.Tensor:
    """dense_ffn_fwd: the same y with dense tensor-core GEMMs.

    h is materialised as bf16 hi + lo halves (h_scratch [M][2N]); with
    bf16_h=True, dense_ffn_fwd_bf16h keeps it as one bf16 (h_scratch [M][N]).
    """
    M, K = x.shape
    N = wg_t.shape[0]
    hcols = N if bf16_h else 2 * N
    if h_scratch is None:
        h_scratch = torch.empty((M, hcols), dtype=torch.bfloat16, device=x.device)
    if y is None:
        y = torch.empty((M, K), dtype=torch.float32, device=x.device)
    if y.dtype != torch.float32 or not y.is_contiguous() or tuple(y.shape) != (M, K):
        raise ValueError("y must be a contiguous float32 tensor of shape (M, K)")
    f = lib().dense_ffn_fwd_bf16h if bf16_h else lib().dense_ffn_fwd
    st = f(_bf16(x, "x", (M, K)), _bf16(wg_t, "wg_t", (N, K)), _bf16(wu_t, "wu_t", (N, K)),
           _bf16(wd, "wd", (N, K)), M, K, N, _bf16(h_scratch, "h_scratch", (M, hcols)), y.data_ptr(),
           _stream(stream))
    _check(st, "dense_ffn_fwd_bf16h" if bf16_h else "dense_ffn_fwd")
    return y


def dense_ffn_noalloc(x: torch.Tensor, wg_t: torch.Tensor, wu_t: torch.Tensor, wd: torch.Tensor,
                      y: torch.Tensor, stream=None) -> torch.Tensor:
    """dense_ffn_fwd_noalloc: dense_ffn with h in the library's fixed device array."""
    M, K = x.shape
    N = wg_t.shape[0]
    if y.dtype != torch.float32 or not y.is_contiguous() or tuple(y.shape) != (M, K) or not y.is_cuda:
        raise ValueError("y must be a contiguous CUDA float32 tensor of shape (M, K)")
    st = lib().dense_ffn_fwd_noalloc(_bf16(x, "x", (M, K)), _bf16(wg_t, "wg_t", (N, K)),
                                     _bf16(wu_t, "wu_t", (N, K)), _bf16(wd, "wd", (N, K)), M, K, N,
                                     y.data_ptr(), _stream(stream))
    _check(st, "dense_ffn_fwd_noalloc")
    return y


def bwd_slot_route(route: int) -> None:
    """twell_bwd_slot_route: 0 chooses the slotted rows' backward route by
    their entry count, 1 forces the dense-slot GEMMs, 2 the gather passes
    (for the calling thread)."""
    _check(lib().twell_bwd_slot_route(int(route)), "twell_bwd_slot_route")


def test_expire_wait(limit_ns: int) -> None:
    """twell_test_expire_wait: arm a one-shot expiring device wait for the next
    ffn_fwd (large batches) or ffn_fused (small batches)."""
    _check(lib().twell_test_expire_wait(int(limit_ns)), "twell_test_expire_wait")


def sparse_ffn(x: torch.Tensor, wg_t: torch.Tensor, wu_t: torch.Tensor, wd: torch.Tensor, T: int, C: int,
               tw: Optional[TwellBuffers] = None, y: Optional[torch.Tensor] = None, sync: bool = True):
    """Whole sparse forward: gate_pack (+ one retry with a larger dense-row buffer
    on capacity overflow, when sync) then ffn_fwd.  Returns (y, tw)."""
    M, K = x.shape
    N = wg_t.shape[0]
    if tw is None:
        tw = TwellBuffers(M, K, N, T, C, device=x.device)
    try:
        gate_pack(x, wg_t, tw, sync=sync)
    except CapacityError as e:
        tw = TwellBuffers(M, K, N, T, C, R_cap=e.n_over, device=x.device)
        gate_pack(x, wg_t, tw, sync=True)
    return ffn_fwd(x, wu_t, wd, tw, y), tw
