"""fp64 CPU oracle for the ReLU-gated sparse FFN forward (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and the
two share no code; see ``oracle.c`` for the definitions and their sources
("Sparser, Faster, Lighter Transformer Language Models" review page, §1-1,
§3-4, §3-5, §3-6).

Every function takes bf16 bit patterns (``uint16`` numpy arrays, layouts as in
``activation_sparse_gated_tma_b200.workloads``) and returns float64 results.
Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(library-routine cross-checks, closed forms, invariants and a hand-worked
golden example); none is "parity unpinned".  The backward pass lives in
``oracle.backward`` (numpy float64), pinned there by central differences of
the float64 forward.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I, L = ctypes.c_int, ctypes.c_int64
        lib.oracle_bf16_to_f64.argtypes = [P, L, P]
        lib.oracle_gate.argtypes = [P, P, I, I, P, L, P, I]
        lib.oracle_twell_pack.argtypes = [P, L, I, I, I, P, P, P, P, P]
        lib.oracle_ffn_twell.argtypes = [P, P, P, I, I, I, I, P, L, P, P, P, P, P, P, I]
        lib.oracle_ffn_dense.argtypes = [P, P, P, P, I, I, P, L, P, I]
        for f in (lib.oracle_bf16_to_f64, lib.oracle_gate, lib.oracle_twell_pack,
                  lib.oracle_ffn_twell, lib.oracle_ffn_dense):
            f.restype = None
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint16)


def _rows(M: int, rows) -> np.ndarray:
    if rows is None:
        return np.arange(M, dtype=np.int64)
    r = np.ascontiguousarray(rows, dtype=np.int64)
    assert r.ndim == 1 and (r.size == 0 or (r.min() >= 0 and r.max() < M))
    return r


def bf16_to_f64(bits) -> np.ndarray:
    b = _u16(bits)
    out = np.empty(b.shape, dtype=np.float64)
    _load().oracle_bf16_to_f64(_p(b), b.size, _p(out))
    return out


def gate(x, wg_t, rows=None, nthreads: Optional[int] = None) -> np.ndarray:
    """z = x W_g for the selected rows, fp64.  Shape [len(rows), N]."""
    x, wg_t = _u16(x), _u16(wg_t)
    M, K = x.shape
    N = wg_t.shape[0]
    assert wg_t.shape == (N, K)
    r = _rows(M, rows)
    z = np.empty((r.size, N), dtype=np.float64)
    _load().oracle_gate(_p(x), _p(wg_t), K, N, _p(r), r.size, _p(z), nthreads or default_threads())
    return z


def twell_pack(z: np.ndarray, T: int, C: int) -> Dict[str, np.ndarray]:
    """TwELL (+ dense backup for overflow tiles) of a block of gate pre-activations."""
    z = np.ascontiguousarray(z, dtype=np.float64)
    R, N = z.shape
    assert N % T == 0 and 1 <= C <= T
    NT = N // T
    counts = np.empty((R, NT), dtype=np.int32)
    idx = np.empty((R, NT, C), dtype=np.int32)
    vals = np.empty((R, NT, C), dtype=np.float64)
    overflow = np.empty((R, NT), dtype=np.uint8)
    dense = np.empty((R, N), dtype=np.float64)
    _load().oracle_twell_pack(_p(z), R, N, T, C, _p(counts), _p(idx), _p(vals), _p(overflow), _p(dense))
    return {"counts": counts, "idx": idx, "vals": vals, "overflow": overflow, "dense": dense,
            "T": T, "C": C}


def ffn_twell(x, wu_t, wd, tw: Dict[str, np.ndarray], rows=None,
              nthreads: Optional[int] = None) -> np.ndarray:
    """y for the selected rows by the sparse rewrite, reading the active set from TwELL.

    ``tw`` must be the TwELL of exactly those rows (row r of tw <-> rows[r]).
    """
    x, wu_t, wd = _u16(x), _u16(wu_t), _u16(wd)
    M, K = x.shape
    N = wu_t.shape[0]
    r = _rows(M, rows)
    T, C = tw["T"], tw["C"]
    assert tw["counts"].shape == (r.size, N // T)
    y = np.empty((r.size, K), dtype=np.float64)
    _load().oracle_ffn_twell(_p(x), _p(wu_t), _p(wd), K, N, T, C, _p(r), r.size,
                             _p(tw["counts"]), _p(tw["idx"]), _p(tw["vals"]),
                             _p(tw["overflow"]), _p(tw["dense"]), _p(y),
                             nthreads or default_threads())
    return y


def ffn_dense(x, wg_t, wu_t, wd, rows=None, nthreads: Optional[int] = None) -> np.ndarray:
    """y for the selected rows by the dense definition (every hidden unit)."""
    x, wg_t, wu_t, wd = _u16(x), _u16(wg_t), _u16(wu_t), _u16(wd)
    M, K = x.shape
    N = wg_t.shape[0]
    r = _rows(M, rows)
    y = np.empty((r.size, K), dtype=np.float64)
    _load().oracle_ffn_dense(_p(x), _p(wg_t), _p(wu_t), _p(wd), K, N, _p(r), r.size, _p(y),
                             nthreads or default_threads())
    return y


def forward(x, wg_t, wu_t, wd, T: int, C: int, rows=None,
            nthreads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """The whole sparse path for the selected rows: gate, TwELL pack, sparse y."""
    z = gate(x, wg_t, rows, nthreads)
    tw = twell_pack(z, T, C)
    y = ffn_twell(x, wu_t, wd, tw, rows, nthreads)
    tw["z"] = z
    tw["y"] = y
    return tw
