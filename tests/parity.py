"""Acceptance rules for comparing the CUDA path with the fp64 oracle.

Readings of the rules (the pages fix no numeric tolerance; these follow the
stated targets and the arithmetic of each side):

  * Ambiguous gate entries: |z64[m,n]| <= 1e-3 * rms_m with
    rms_m = sqrt(mean_n z64[m,n]^2).  Only there may the GPU's fp32 sign
    decision differ from the fp64 one.
  * Support: {G_gpu > 0} and {z64 > 0} differ only on ambiguous entries.
  * Counts: exact on tiles without ambiguous entries; always equal to the
    number of positive decoded GPU entries of the tile.
  * Indices: bit-exact (ascending) on such tiles when count <= C.
  * Values (stored in fp32): |vals - z64| <= 2^-23 |z64| + K * 2^-22 * S with
    S = sum_k |x_k w_k| (fp32 accumulation of K exact bf16 products in any
    order is within K * u * S; u = 2^-22 is four times the fp32 unit roundoff,
    room for the tensor core's internal alignment of partial sums).
  * Overflow classification equals the oracle's unless ambiguous entries
    straddle C (then both count sides stay within the ambiguous range).
  * y (sparse path and dense_ffn_fwd, both with fp32 or hi+lo bf16
    intermediates): max |y_gpu - y64| <= 2e-2 * rms(y64) over all compared
    entries, rms taken over the whole compared block.
  * y of the bf16-h dense variant (dense_ffn_fwd_bf16h, reported next to the
    dense path but not held to the rule above): elementwise
    |y_gpu - y64| <= sum_n dh[m,n] |W_d[n,k]| + N * 2^-23 * A + 1e-6 * rms(y64)
    with A[m,k] = sum_n |h64[m,n]| |W_d[n,k]| and the error of the stored h
    dh = 2^-9 |h64| + K * 2^-22 * (S_u |g64| + S_g |u64|): rounding h to bf16
    (relative error <= 2^-9) plus the fp32 accumulation of u and g (the values
    rule above, S_u and S_g the absolute-product sums of each); then the fp32
    accumulation of N products in the second GEMM.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from activation_sparse_gated_tma_b200 import workloads as wl

Y_REL_TOL = 2e-2
AMBIG_REL = 1e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_f64(bits) -> np.ndarray:
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def abs_bits(bits: np.ndarray) -> np.ndarray:
    return (bits & np.uint16(0x7FFF)).astype(np.uint16)


def decode_gpu_gate(h: dict, rows: np.ndarray, N: int, T: int, C: int) -> np.ndarray:
    """Dense [R][N] view of the GPU's TwELL slots and dense-row backup for `rows`."""
    R = rows.size
    NT = N // T
    counts = h["counts"][rows].astype(np.int64)
    idx = h["idx"][rows].astype(np.int64)
    vals = h["vals"][rows].astype(np.float64)
    ov = counts > C
    G = np.zeros((R, N))
    used = (np.arange(C)[None, None, :] < np.minimum(counts, C)[:, :, None]) & ~ov[:, :, None]
    r_i, t_i, s_i = np.nonzero(used)
    li = idx[r_i, t_i, s_i]
    assert (li < T).all(), "local index out of tile"
    np.add.at(G, (r_i, t_i * T + li), vals[r_i, t_i, s_i])
    slots = h["row_slot"][rows]
    r_o, t_o = np.nonzero(ov)
    if r_o.size:
        assert (slots[r_o] >= 0).all(), "overflow tile without a dense-row slot"
        for r, t in zip(r_o, t_o):
            G[r, t * T:(t + 1) * T] = h["dense_rows"][slots[r], t * T:(t + 1) * T].astype(np.float64)
    return G


def check_twell(h: dict, rows: np.ndarray, z64: np.ndarray, S: np.ndarray, K: int, T: int, C: int) -> dict:
    """Apply the TwELL rules to the GPU arrays `h` for `rows` (oracle z64, abs-sum S)."""
    R, N = z64.shape
    NT = N // T
    rms = np.sqrt((z64 ** 2).mean(1))
    amb = np.abs(z64) <= AMBIG_REL * rms[:, None]
    G = decode_gpu_gate(h, rows, N, T, C)
    counts = h["counts"][rows].astype(np.int64)
    gpos, opos = G > 0, z64 > 0
    bad_support = (gpos ^ opos) & ~amb
    assert not bad_support.any(), f"{bad_support.sum()} unambiguous support mismatches"
    tile_amb = amb.reshape(R, NT, T).any(2)
    cnt_or = opos.reshape(R, NT, T).sum(2)
    cnt_gpu_decoded = gpos.reshape(R, NT, T).sum(2)
    assert np.array_equal(counts, cnt_gpu_decoded), "count disagrees with the stored entries"
    assert np.array_equal(counts[~tile_amb], cnt_or[~tile_amb]), "count mismatch on an unambiguous tile"
    # indices of unambiguous non-overflow tiles
    sel = (~tile_amb) & (cnt_or <= C)
    idx = h["idx"][rows].astype(np.int64)
    for r, t in zip(*np.nonzero(sel & (cnt_or > 0))):
        want = np.nonzero(opos[r, t * T:(t + 1) * T])[0]
        assert np.array_equal(idx[r, t, :want.size], want), f"indices differ at row {rows[r]} tile {t}"
    # overflow classification
    ov_gpu, ov_or = counts > C, cnt_or > C
    amb_cnt = amb.reshape(R, NT, T).sum(2)
    differs = ov_gpu != ov_or
    assert not (differs & (np.abs(cnt_or - C) > amb_cnt)).any(), "overflow classification differs"
    # values
    tol = 2.0 ** -23 * np.abs(z64) + K * 2.0 ** -22 * S
    err = np.abs(G - np.maximum(z64, 0.0))
    vmask = gpos | (opos & ~amb)
    worst = float((err[vmask] / np.maximum(tol[vmask], 1e-300)).max()) if vmask.any() else 0.0
    assert worst <= 1.0, f"value error {worst:.3g} x tolerance"
    return {"rows": int(R), "active": int(gpos.sum()), "ambiguous": int(amb.sum()),
            "overflow_tiles": int(ov_gpu.sum()), "value_err_over_tol": worst,
            "max_abs_err_over_rms": float((err[vmask] / rms[np.nonzero(vmask)[0]]).max()) if vmask.any() else 0.0}


def check_y(y_gpu: np.ndarray, y64: np.ndarray, what: str = "y") -> dict:
    rms = float(np.sqrt((y64 ** 2).mean()))
    err = float(np.abs(y_gpu.astype(np.float64) - y64).max())
    if rms == 0.0:
        assert err == 0.0, f"{what}: expected exact zeros, max |y| = {err}"
        return {"rms": 0.0, "max_err": err, "rel": 0.0}
    assert err <= Y_REL_TOL * rms, f"{what}: max err {err:.3g} > {Y_REL_TOL} * rms {rms:.3g}"
    return {"rms": rms, "max_err": err, "rel": err / rms}


def check_y_bf16h(y_gpu: np.ndarray, y64: np.ndarray, u64: np.ndarray, z64: np.ndarray, S_u: np.ndarray,
                  S_g: np.ndarray, wd_bits: np.ndarray, K: int, what: str = "bf16-h dense y") -> dict:
    """Elementwise bound for the dense variant that rounds h to one bf16."""
    g64 = np.maximum(z64, 0.0)
    h64 = u64 * g64
    # S_g |u| also covers units the fp32 gate turns on where z64 <= 0 (then g_gpu <= K 2^-22 S_g)
    dh = 2.0 ** -9 * np.abs(h64) + K * 2.0 ** -22 * (S_u * g64 + S_g * np.abs(u64))
    wd = np.abs(bf16_f64(wd_bits))
    N = wd.shape[0]
    tol = dh @ wd + N * 2.0 ** -23 * (np.abs(h64) @ wd)
    rms = float(np.sqrt((y64 ** 2).mean()))
    tol += 1e-6 * rms
    err = np.abs(y_gpu.astype(np.float64) - y64)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"{what}: error {worst:.3g} x the bf16-h bound"
    return {"rms": rms, "max_err": float(err.max()), "rel": float(err.max() / rms) if rms else 0.0,
            "err_over_bound": worst}
