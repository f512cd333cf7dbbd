"""GPU parity of the backward pass over the hybrid activations
(twell_ffn_bwd) against the fp64 oracle in oracle/backward.py, on the active
set the forward chose (TwELL + dense-row slots).  The rule is the one the y
of the forward is held to, per output: max|gpu - oracle| <= 2e-2 rms(oracle);
rows of units that no token activates must be exactly zero."""
import numpy as np
import pytest
import torch

from activation_sparse_gated_tma_b200 import twell as tw
from activation_sparse_gated_tma_b200 import workloads as wl
from oracle import backward as ob
from tests.test_gpu_parity import _small, _workload

pytestmark = pytest.mark.gpu


def _active_mask(h, N, T, C):
    """[M][N] bool: the units the forward treats as active."""
    counts = h["counts"].astype(np.int64)
    M, NT = counts.shape
    mask = np.zeros((M, N), bool)
    for m in range(M):
        for t in range(NT):
            c = counts[m, t]
            if 0 < c <= C:
                mask[m, t * T + h["idx"][m, t, :c].astype(np.int64)] = True
            elif c > C and h["row_slot"][m] >= 0:
                mask[m, t * T:(t + 1) * T] = h["dense_rows"][h["row_slot"][m], t * T:(t + 1) * T] > 0
    return mask


def _check(name, got, ref, zero_rows=None):
    got = got.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.abs(got - ref).max())
    assert err <= 2e-2 * rms, f"{name}: max err {err:.3e} > 2e-2 rms ({rms:.3e})"
    if zero_rows is not None and zero_rows.any():
        assert not got[zero_rows].any(), f"{name}: rows of inactive units are not zero"
    return err / rms


def _run(w, d, dev, R_cap=None, seed=0, route=0):
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C, R_cap=R_cap if R_cap is not None else w.R_cap)
    tw.gate_pack(dev["x"], dev["wg_t"], t, sync=True)
    dy = np.random.default_rng(seed).standard_normal((w.M, w.K)).astype(np.float32)
    tw.bwd_slot_route(route)
    try:
        dx, dg, du, dd = tw.ffn_bwd(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], t, torch.from_numpy(dy).cuda())
        torch.cuda.synchronize()
    finally:
        tw.bwd_slot_route(0)
    h = t.to_host()
    mask = _active_mask(h, w.N, w.T, w.C)
    ref = ob.ffn_backward(d["x"], d["wg_t"], d["wu_t"], d["wd"], dy.astype(np.float64), active=mask)
    idle = ~mask.any(axis=0)
    out = {"dx": _check("dx", dx, ref["dx"]),
           "dwg_t": _check("dwg_t", dg, ref["dwg_t"], idle),
           "dwu_t": _check("dwu_t", du, ref["dwu_t"], idle),
           "dwd": _check("dwd", dd, ref["dwd"], idle)}
    _run.last_unit_entries = mask[h["row_slot"] < 0].sum(axis=0)  # TwELL entries per hidden unit
    return out, int(mask.sum()), int((h["row_slot"] >= 0).sum())


@pytest.mark.parametrize("M,T,C", [(1, 128, 4), (37, 128, 4), (64, 256, 8), (300, 128, 4)])
def test_backward_small_shapes(M, T, C):
    w, d, dev = _small(M, 192, 2 * T, T, C, None, seed=M + T + 7, R_cap=M)
    out, active, slotted = _run(w, d, dev, R_cap=M)
    print(M, T, C, out, active, slotted)


@pytest.mark.parametrize("route", [0, 1, 2])
def test_backward_all_gates_on_goes_through_the_dense_rows(route):
    w, d, dev = _small(40, 128, 512, 128, 4, bias=-1e2, seed=2, R_cap=40)
    out, active, slotted = _run(w, d, dev, R_cap=40, route=route)
    assert slotted == 40 and active == 40 * 512
    print(out)


@pytest.mark.parametrize("name", ["tiny_m64_k256_n1024_p98", "sweep_m64_k2048_n8192_p99",
                                  "m2048_k1536_n4096_p99_lognormal05"])
def test_backward_workloads(name):
    w, d, dev = _workload(name)
    out, active, slotted = _run(w, d, dev, seed=3)
    print(name, out, active, slotted)


@pytest.mark.parametrize("route", [1, 2])
def test_backward_slotted_rows_by_either_route(route):
    # 201 of 2048 rows hold dense-row slots (half of all active entries):
    # the dense-slot GEMMs and the gather passes both meet the rule.
    w, d, dev = _workload("m2048_k1536_n4096_p99_lognormal05")
    out, active, slotted = _run(w, d, dev, seed=3, route=route)
    assert slotted > 8
    print(route, out, active, slotted)


@pytest.mark.parametrize("C,R_cap,route", [(32, None, 0), (16, None, 0), (12, 2000, 0), (12, 2000, 1)])
def test_backward_units_with_many_entries(C, R_cap, route):
    # 5% activation over 2000 rows: about 100 TwELL entries per hidden unit, so
    # the unit pass cuts units into pieces of at most 64 entries that add into
    # the same weight-gradient rows.  C=32: no row overflows; C=16: a few rows
    # do, and (at most 8 of them) their entries join the gather passes; C=12:
    # dozens do, through either route.
    w, d, dev = _small(2000, 192, 256, 128, C, None, seed=11, R_cap=R_cap)
    out, active, slotted = _run(w, d, dev, R_cap=R_cap, seed=5, route=route)
    per_unit = _run.last_unit_entries
    assert per_unit.max() > 64, per_unit.max()
    if C == 16:
        assert 0 < slotted <= 8, slotted
    if C == 12:
        assert slotted > 8, slotted
    print(C, out, active, slotted, int(per_unit.min()), int(per_unit.max()))
