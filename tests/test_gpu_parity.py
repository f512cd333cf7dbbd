"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Rules in tests/parity.py."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gated_tma_b200 import twell as tw
from activation_sparse_gated_tma_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu

_CACHE = {}


def _workload(name):
    if name not in _CACHE:
        w = wl.WORKLOADS[name]
        d = wl.generate(w)
        dev = {k: P.to_dev(d[k]) for k in ("x", "wg_t", "wu_t", "wd")}
        _CACHE.clear()
        _CACHE[name] = (w, d, dev)
    return _CACHE[name]


def _sample_rows(w, h, n=256):
    rows = wl.subsample_rows(w.M, n, seed=w.seed + 99)
    slotted = np.nonzero(h["row_slot"] >= 0)[0]
    if slotted.size:
        extra = slotted[wl.subsample_rows(slotted.size, 64, seed=w.seed + 7)]
        rows = np.unique(np.concatenate([rows, extra]))
    return rows


def _run_sparse(dev, w, R_cap=None):
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C, R_cap=R_cap if R_cap is not None else w.R_cap)
    n_over = tw.gate_pack(dev["x"], dev["wg_t"], t, sync=True)
    y = tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], t)
    st, n2, flags = tw.read_status(t)
    assert st == tw.OK and n2 == n_over and flags == 0
    torch.cuda.synchronize()
    return t, n_over, y


def _compare(w, d, t, y, rows, dense_y=None):
    h = t.to_host()
    ref = oracle.forward(d["x"], d["wg_t"], d["wu_t"], d["wd"], w.T, w.C, rows=rows)
    S = oracle.gate(P.abs_bits(d["x"]), P.abs_bits(d["wg_t"]), rows=rows)
    stats = P.check_twell(h, rows, ref["z"], S, w.K, w.T, w.C)
    yg = y[torch.from_numpy(rows).cuda()].cpu().numpy()
    out = {"twell": stats, "y": P.check_y(yg, ref["y"], "twell y")}
    if dense_y is not None:
        out["dense"] = P.check_y(dense_y[torch.from_numpy(rows).cuda()].cpu().numpy(), ref["y"], "dense y")
    return out


@pytest.mark.parametrize("name", wl.PARITY_WORKLOADS)
def test_full_size_parity(name):
    w, d, dev = _workload(name)
    t, n_over, y = _run_sparse(dev, w)
    assert n_over <= w.R_cap
    yd = tw.dense_ffn(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"])
    rows = _sample_rows(w, t.to_host(), n=w.M if w.M <= 64 else 256)
    stats = _compare(w, d, t, y, rows, dense_y=yd)
    print(name, "n_over", n_over, stats)
    if name.startswith("m16384"):
        assert n_over > 0, "the boosted workload must exercise the dense-row path"


@pytest.mark.parametrize("name", [n for n in wl.WORKLOADS if n.startswith("sweep_")])
def test_sweep_parity(name):
    w, d, dev = _workload(name)
    t, n_over, y = _run_sparse(dev, w)
    yd = tw.dense_ffn(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"])
    rows = _sample_rows(w, t.to_host(), n=min(w.M, 96))
    _compare(w, d, t, y, rows, dense_y=yd)


@pytest.mark.parametrize("name", ["tiny_m64_k256_n1024_p98", "m2048_k1536_n4096_p99_lognormal05",
                                  "m8192_k2048_n5632_loguniform_lognormal07"])
def test_dense_bf16h_variant_within_its_rounding_bound(name):
    # The labelled second dense number: h rounded to one bf16.  Held to the
    # bound that rounding implies, on sampled rows.
    w, d, dev = _workload(name)
    y = tw.dense_ffn(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], bf16_h=True)
    rows = wl.subsample_rows(w.M, 64, seed=w.seed + 3)
    z = oracle.gate(d["x"], d["wg_t"], rows=rows)
    u = oracle.gate(d["x"], d["wu_t"], rows=rows)       # x W_u: the same fp64 product
    S_g = oracle.gate(P.abs_bits(d["x"]), P.abs_bits(d["wg_t"]), rows=rows)
    S_u = oracle.gate(P.abs_bits(d["x"]), P.abs_bits(d["wu_t"]), rows=rows)
    ref = oracle.ffn_dense(d["x"], d["wg_t"], d["wu_t"], d["wd"], rows=rows)
    stats = P.check_y_bf16h(y[torch.from_numpy(rows).cuda()].cpu().numpy(), ref, u, z, S_u, S_g, d["wd"], w.K)
    print(name, stats)


def _small(M, K, N, T, C, bias, seed, R_cap=None):
    w = wl.Workload(f"small_{M}_{K}_{N}", M, K, N, T, C, seed, p_mean=0.05, r_cap=R_cap)
    d = wl.generate(w)
    if bias is not None:
        d["wg_t"][:, K - 1] = wl.f32_to_bf16_bits(np.array([-bias], np.float32))[0]
    dev = {k: P.to_dev(d[k]) for k in ("x", "wg_t", "wu_t", "wd")}
    return w, d, dev


@pytest.mark.parametrize("M", [1, 17, 127, 129, 300])
@pytest.mark.parametrize("T,C", [(128, 4), (256, 8)])
def test_ragged_shapes_full_compare(M, T, C):
    w, d, dev = _small(M, 192, 2 * T, T, C, None, seed=M + T, R_cap=M)
    t, n_over, y = _run_sparse(dev, w, R_cap=M)
    rows = np.arange(M)
    _compare(w, d, t, y, rows, dense_y=tw.dense_ffn(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"]))


@pytest.mark.parametrize("M", [33, 200])
def test_smallest_k_full_compare(M):
    # K = 64: one K block for every GEMM (both gate paths: M = 33 and 200).
    w, d, dev = _small(M, 64, 512, 128, 4, None, seed=M + 5, R_cap=M)
    t, n_over, y = _run_sparse(dev, w, R_cap=M)
    _compare(w, d, t, y, np.arange(M), dense_y=tw.dense_ffn(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"]))


def test_all_gates_off_gives_exact_zero():
    w, d, dev = _small(130, 128, 512, 128, 4, bias=1e4, seed=1)
    t, n_over, y = _run_sparse(dev, w)
    assert n_over == 0
    assert int(t.counts.abs().sum()) == 0
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("M", [130, 40])
def test_all_gates_on_routes_every_tile_to_dense_rows(M):
    # M = 130: dense-row GEMMs; M = 40: the small-batch kernel serves the slots.
    w, d, dev = _small(M, 128, 512, 128, 4, bias=-1e2, seed=2, R_cap=M)
    t, n_over, y = _run_sparse(dev, w, R_cap=M)
    assert n_over == M
    h = t.to_host()
    assert (h["counts"] == 128).all()
    _compare(w, d, t, y, np.arange(M))


def test_capacity_equal_tile_never_overflows():
    w, d, dev = _small(64, 128, 256, 128, 128, bias=-1e2, seed=3, R_cap=1)
    t, n_over, y = _run_sparse(dev, w, R_cap=1)
    assert n_over == 0
    _compare(w, d, t, y, np.arange(64))


def test_capacity_exceeded_reports_and_retry_succeeds():
    w, d, dev = _small(96, 128, 512, 128, 2, bias=0.0, seed=4)
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C, R_cap=1)
    with pytest.raises(tw.CapacityError) as e:
        tw.gate_pack(dev["x"], dev["wg_t"], t, sync=True)
    assert e.value.n_over > 1
    y, t2 = tw.sparse_ffn(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], w.T, w.C, tw=tw.TwellBuffers(
        w.M, w.K, w.N, w.T, w.C, R_cap=1))
    assert t2.R_cap == e.value.n_over
    torch.cuda.synchronize()
    _compare(w, d, t2, y, np.arange(96))
    # asynchronous mode: the capacity problem is reported by read_status
    t3 = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C, R_cap=1)
    tw.gate_pack(dev["x"], dev["wg_t"], t3, sync=False)
    st, n_over, flags = tw.read_status(t3)
    assert st == tw.ERR_CAPACITY and n_over == e.value.n_over


def test_repeat_calls_are_deterministic():
    w, d, dev = _workload("m2048_k1536_n4096_p99_lognormal05")
    t1, _, y1 = _run_sparse(dev, w)
    h1 = t1.to_host()
    y1 = y1.clone()
    t2, _, y2 = _run_sparse(dev, w)
    h2 = t2.to_host()
    assert np.array_equal(h1["counts"], h2["counts"])
    C = w.C
    cnt = np.minimum(h1["counts"], C)
    used = np.arange(C)[None, None, :] < cnt[:, :, None]
    assert np.array_equal(h1["idx"][used], h2["idx"][used])
    assert np.array_equal(h1["vals"][used], h2["vals"][used])
    # Rows without overflow and with at most one work unit of TwELL entries are
    # produced by one warp alone: bit-identical.  Rows split across warps and
    # slotted rows add partials with fp32 atomics, whose order varies.
    listed = np.where(h1["counts"] <= C, h1["counts"], 0).astype(np.int64).sum(1)
    plain = torch.from_numpy((h1["row_slot"] < 0) & (listed <= 8)).cuda()
    assert int(plain.sum()) > w.M // 4
    assert torch.equal(y1[plain], y2[plain])
    torch.testing.assert_close(y1[~plain], y2[~plain], rtol=1e-5, atol=1e-5 * float(y1.abs().max()))
    # the fused kernel reuses its work queue across launches
    y3 = tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], t2)
    assert torch.equal(y1[plain], y3[plain])


def test_expired_device_wait_is_reported_and_the_next_call_recovers():
    # The fused kernel's wait for the row scan is given an unreachable target
    # and a 5 us limit (host-side injection): the kernel must give up, flag
    # it, and leave the buffers usable for the next pass.
    w, d, dev = _workload("m2048_k1536_n4096_p99_lognormal05")
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C)
    tw.gate_pack(dev["x"], dev["wg_t"], t, sync=True)
    tw.test_expire_wait(5000)
    tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], t)
    st, n_over, flags = tw.read_status(t)
    assert st == tw.ERR_DEVICE_CHECK and (flags & 1), (st, flags)
    tw.gate_pack(dev["x"], dev["wg_t"], t, sync=True)
    y = tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], t)
    st, n_over, flags = tw.read_status(t)
    assert st == tw.OK and flags == 0
    torch.cuda.synchronize()
    _compare(w, d, t, y, _sample_rows(w, t.to_host(), n=128))


def test_launch_accounting():
    w, d, dev = _workload("m2048_k1536_n4096_p99_lognormal05")
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C)
    tw.gate_pack(dev["x"], dev["wg_t"], t)
    assert tw.last_launch_count() == 2
    tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], t)
    assert tw.last_launch_count() == 3
    tw.dense_ffn(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"])
    assert tw.last_launch_count() == 2


def test_kernel_trace_brackets_every_launch():
    w, d, dev = _workload("m2048_k1536_n4096_p99_lognormal05")
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C)
    with tw.KernelTrace(capacity=8) as tr:
        tw.gate_pack(dev["x"], dev["wg_t"], t)
        tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], t)
    torch.cuda.synchronize()
    names = [n for n, _ in tr.times_ms()]
    assert names == ["twell_reset", "gate_twell_gemm", "twell_updown", "overflow_up_gemm", "overflow_down_gemm"]
    assert all(ms > 0 for _, ms in tr.times_ms())


def test_small_batch_takes_the_stream_path():
    # M <= TWELL_SMALL_M: the stream-K gate kernel packs TwELL itself; y is
    # cleared and one static-unit kernel serves TwELL and overflow tiles.
    w, d, dev = _workload("sweep_m64_k2048_n8192_p99")
    t = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C)
    with tw.KernelTrace(capacity=8) as tr:
        tw.gate_pack(dev["x"], dev["wg_t"], t)
        assert tw.last_launch_count() == 2
        y = tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], t)
        assert tw.last_launch_count() == 1
    torch.cuda.synchronize()
    assert [n for n, _ in tr.times_ms()] == ["twell_reset", "gate_stream_pack", "twell_updown_small"]
    _compare(w, d, t, y, np.arange(w.M))


@pytest.mark.parametrize("K,N,T", [(192, 256, 128), (192, 512, 256), (4096, 1024, 256)])
def test_small_batch_gate_pieces_from_several_ctas(K, N, T):
    # Few k blocks per 128-unit tile: every tile's sum is split over two to
    # four CTAs and added by the last one, for T = 128 and for T = 256 (a
    # TwELL tile spans two 128-unit tiles).
    w, d, dev = _small(24, K, N, T, 8, None, seed=K + N, R_cap=24)
    t, n_over, y = _run_sparse(dev, w, R_cap=24)
    _compare(w, d, t, y, np.arange(24))


def test_maximum_sizes_on_both_gate_paths():
    # K = 4096 (the largest K: the fused kernel's four-warp shape) and N/T = 256
    # (the largest tile count), on the gate GEMM's own packing (M = 130) and on
    # the small-batch path (the first 64 rows).
    w = wl.Workload("max_m130_k4096_n32768_p99", 130, 4096, 32768, 128, 8, 7, p_mean=0.01, r_cap=130)
    d = wl.generate(w)
    _CACHE.clear()
    for M in (130, 64):
        wm = dataclasses.replace(w, M=M)
        dm = dict(d, x=d["x"][:M])
        dev = {k: P.to_dev(dm[k]) for k in ("x", "wg_t", "wu_t", "wd")}
        t, n_over, y = _run_sparse(dev, wm, R_cap=M)
        stats = _compare(wm, dm, t, y, np.arange(M))
        print("max sizes M", M, "n_over", n_over, stats)
        del dev, t, y
        torch.cuda.empty_cache()
