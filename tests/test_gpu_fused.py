"""GPU parity of twell_ffn_fused (the whole sparse forward in one call; one
persistent kernel after the reset for small batches) against the fp64
oracle, through the C ABI.  Rules in tests/parity.py."""
import numpy as np
import pytest
import torch

from activation_sparse_gated_tma_b200 import twell as tw
from activation_sparse_gated_tma_b200 import workloads as wl
from tests import parity as P
from tests.test_gpu_parity import _compare, _sample_rows, _small, _workload

pytestmark = pytest.mark.gpu


def _run_fused(dev, w, R_cap=None):
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C, R_cap=R_cap if R_cap is not None else w.R_cap)
    y = tw.ffn_fused(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], t, sync=True)
    st, n_over, flags = tw.read_status(t)
    assert st == tw.OK and flags == 0 and n_over == t.n_over_known
    torch.cuda.synchronize()
    return t, n_over, y


@pytest.mark.parametrize("name", ["sweep_m16_k2048_n8192_p99", "sweep_m64_k2048_n8192_p99",
                                  "sweep_m16_k2048_n8192_p90", "tiny_m64_k256_n1024_p98"])
def test_fused_small_batch_full_compare(name):
    w, d, dev = _workload(name)
    t, n_over, y = _run_fused(dev, w)
    print(name, n_over, _compare(w, d, t, y, np.arange(w.M)))


@pytest.mark.parametrize("M", [1, 17, 128])
@pytest.mark.parametrize("T,C", [(128, 4), (256, 8)])
def test_fused_ragged_full_compare(M, T, C):
    w, d, dev = _small(M, 192, 2 * T, T, C, None, seed=M + T + 1, R_cap=M)
    t, n_over, y = _run_fused(dev, w, R_cap=M)
    _compare(w, d, t, y, np.arange(M))


def test_fused_k4096_full_compare():
    # The largest K: two ring stages per warp in the up/down phase.
    w, d, dev = _small(20, 4096, 1024, 128, 8, None, seed=41, R_cap=20)
    t, n_over, y = _run_fused(dev, w, R_cap=20)
    _compare(w, d, t, y, np.arange(20))


def test_fused_all_gates_on_serves_every_tile_from_dense_rows():
    w, d, dev = _small(40, 128, 512, 128, 4, bias=-1e2, seed=2, R_cap=40)
    t, n_over, y = _run_fused(dev, w, R_cap=40)
    assert n_over == 40
    assert (t.to_host()["counts"] == 128).all()
    _compare(w, d, t, y, np.arange(40))


def test_fused_capacity_exceeded_then_retry():
    w, d, dev = _small(96, 128, 512, 128, 2, bias=0.0, seed=4)
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C, R_cap=1)
    with pytest.raises(tw.CapacityError) as e:
        tw.ffn_fused(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], t, sync=True)
    assert e.value.n_over > 1
    t2 = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C, R_cap=e.value.n_over)
    y = tw.ffn_fused(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], t2, sync=True)
    torch.cuda.synchronize()
    _compare(w, d, t2, y, np.arange(96))


def test_fused_large_batch_matches_the_two_call_path():
    w, d, dev = _workload("m2048_k1536_n4096_p99_lognormal05")
    t, n_over, y = _run_fused(dev, w)
    print(_compare(w, d, t, y, _sample_rows(w, t.to_host(), n=128)))


def test_fused_small_batch_is_one_kernel_after_the_reset():
    w, d, dev = _workload("sweep_m64_k2048_n8192_p99")
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C)
    with tw.KernelTrace(capacity=8) as tr:
        tw.ffn_fused(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], t)
        assert tw.last_launch_count() == 2
    torch.cuda.synchronize()
    assert [n for n, _ in tr.times_ms()] == ["twell_reset", "twell_fused_small"]


def test_fused_grid_barrier_expiry_is_reported_and_the_next_call_recovers():
    # The barrier is given one CTA more than the grid holds and a 5 us limit
    # (host-side injection): every CTA gives up, flags it and returns.
    w, d, dev = _workload("sweep_m16_k2048_n8192_p99")
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C)
    tw.test_expire_wait(5000)
    tw.ffn_fused(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], t)
    st, n_over, flags = tw.read_status(t)
    assert st == tw.ERR_DEVICE_CHECK and (flags & 1), (st, flags)
    t2, n_over, y = _run_fused(dev, w)
    _compare(w, d, t2, y, np.arange(w.M))
