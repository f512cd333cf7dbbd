"""Pins of the fp64 CPU oracle to facts outside itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle fails at least one of
them: a dropped term, a wrong sign, a transposed weight, swapped gate/up roles,
a non-strict ReLU test, a wrong tile offset or slot order, a lost overflow tile.

  * library routine: the gate and the dense FFN against numpy float64 matmul
    (the §1-1 definition evaluated by a different implementation);
  * closed form: permutation-structured weights, where y reduces to one
    product per output coordinate;
  * invariants: TwELL unpacked == ReLU(z) exactly; sparse rewrite (§3-5) ==
    dense definition (§1-1);
  * special cases: all gates off, all gates on, C = T, exact zeros;
  * a hand-worked golden example (tests/golden/tiny_ffn_handworked.txt).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gated_tma_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_ffn_handworked.txt")


def _bf16(a):
    return wl.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _f64(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def _rand_problem(M, K, N, seed, bias=None):
    rng = np.random.default_rng(seed)
    x = _bf16(rng.standard_normal((M, K)))
    wg = _bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    wu = _bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    wd = _bf16(rng.standard_normal((N, K)) / np.sqrt(N))
    if bias is not None:
        x[:, K - 1] = _bf16([1.0])[0]
        wg[:, K - 1] = _bf16([-bias])[0]
    return x, wg, wu, wd


def _numpy_ffn(x, wg, wu, wd):
    X, G, U, D = (_f64(a) for a in (x, wg, wu, wd))
    return ((X @ U.T) * np.maximum(X @ G.T, 0.0)) @ D


def _unpack(tw, N):
    """Dense [R][N] view of TwELL slots plus the dense backup."""
    counts, idx, vals, ov, dense = tw["counts"], tw["idx"], tw["vals"], tw["overflow"], tw["dense"]
    T, C = tw["T"], tw["C"]
    R, NT = counts.shape
    out = dense.copy()
    for r in range(R):
        for t in range(NT):
            if not ov[r, t]:
                for s in range(counts[r, t]):
                    out[r, t * T + idx[r, t, s]] += vals[r, t, s]
    return out


# ---------------------------------------------------------------- bf16 decode
def test_bf16_decode_matches_torch_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ---------------------------------------------------------------- gate GEMM
@pytest.mark.parametrize("M,K,N", [(1, 64, 128), (37, 192, 320), (5, 256, 1024)])
def test_gate_matches_numpy_float64_matmul(M, K, N):
    x, wg, _, _ = _rand_problem(M, K, N, seed=M + K + N)
    z = oracle.gate(x, wg)
    ref = _f64(x) @ _f64(wg).T
    assert np.max(np.abs(z - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_gate_one_hot_rows_pick_a_weight_column():
    K, N = 64, 256
    _, wg, _, _ = _rand_problem(1, K, N, seed=3)
    x = np.zeros((K, K), dtype=np.float32)
    np.fill_diagonal(x, 1.0)
    z = oracle.gate(_bf16(x), wg)
    assert np.array_equal(z, _f64(wg).T)          # z[k][n] = W_g[k][n] = wg_t[n][k]


def test_gate_row_selection():
    x, wg, _, _ = _rand_problem(50, 128, 256, seed=9)
    rows = np.array([49, 0, 17, 17])
    assert np.array_equal(oracle.gate(x, wg, rows), oracle.gate(x, wg)[rows])


# ---------------------------------------------------------------- TwELL pack
def _check_twell_invariants(z, tw):
    T, C = tw["T"], tw["C"]
    R, N = z.shape
    counts, idx, vals, ov = tw["counts"], tw["idx"], tw["vals"], tw["overflow"]
    assert np.array_equal(_unpack(tw, N), np.maximum(z, 0.0))
    for r in range(R):
        for t in range(N // T):
            zt = z[r, t * T:(t + 1) * T]
            act = np.nonzero(zt > 0)[0]
            assert counts[r, t] == act.size
            assert ov[r, t] == (act.size > C)
            if act.size <= C:
                assert np.array_equal(idx[r, t, :act.size], act)       # ascending local indices
                assert np.array_equal(vals[r, t, :act.size], zt[act])
                assert not idx[r, t, act.size:].any() and not vals[r, t, act.size:].any()
                assert not tw["dense"][r, t * T:(t + 1) * T].any()


@pytest.mark.parametrize("T,C", [(4, 1), (8, 3), (16, 16), (128, 8)])
def test_twell_invariants_random(T, C):
    rng = np.random.default_rng(T * 100 + C)
    N = 256
    z = rng.standard_normal((9, N)) - 1.0
    z[rng.random(z.shape) < 0.1] = 0.0            # exact zeros are inactive
    z[rng.random(z.shape) < 0.05] = -0.0
    z[3, :] = 1.0 + rng.random(N)                 # a row where every tile overflows (C < T)
    tw = oracle.twell_pack(z, T, C)
    _check_twell_invariants(z, tw)
    if C == T:
        assert not tw["overflow"].any()


def test_twell_special_cases():
    N, T, C = 64, 16, 4
    tw = oracle.twell_pack(-np.ones((2, N)), T, C)       # all gates off
    assert not tw["counts"].any() and not tw["overflow"].any() and not tw["dense"].any()
    tw = oracle.twell_pack(np.zeros((2, N)), T, C)       # ReLU(0) = 0 is not active
    assert not tw["counts"].any()
    z = np.arange(1, 2 * N + 1, dtype=np.float64).reshape(2, N)
    tw = oracle.twell_pack(z, T, C)                      # all gates on
    assert (tw["counts"] == T).all() and tw["overflow"].all()
    assert np.array_equal(tw["dense"], z)


# ---------------------------------------------------------------- FFN output
def test_sparse_rewrite_equals_dense_definition_and_numpy():
    M, K, N, T, C = 24, 128, 512, 128, 4
    x, wg, wu, wd = _rand_problem(M, K, N, seed=11, bias=1.6)
    out = oracle.forward(x, wg, wu, wd, T, C)
    assert out["overflow"].any() and (~out["overflow"].astype(bool)).any()
    yd = oracle.ffn_dense(x, wg, wu, wd)
    yn = _numpy_ffn(x, wg, wu, wd)
    scale = np.max(np.abs(yn))
    assert scale > 0
    assert np.max(np.abs(out["y"] - yd)) <= 1e-12 * scale
    assert np.max(np.abs(yd - yn)) <= 1e-12 * scale


def test_overflow_partition_does_not_change_y():
    M, K, N = 8, 128, 256
    x, wg, wu, wd = _rand_problem(M, K, N, seed=5, bias=0.5)
    ys = [oracle.forward(x, wg, wu, wd, T, C)["y"] for T, C in [(256, 256), (128, 2), (64, 1), (32, 32)]]
    for y in ys[1:]:
        assert np.max(np.abs(y - ys[0])) <= 1e-12 * np.max(np.abs(ys[0]))


def test_closed_form_permutation_weights():
    # W_g, W_u, W_d are scaled permutation matrices (K = N).  Then
    #   z[m][n] = a x[m][pi(n)],  h_u[m][n] = c x[m][sig(n)],
    #   y[m][tau(n)] = d * c x[m][sig(n)] * max(a x[m][pi(n)], 0).
    # tau is not an involution, so a transposed W_d gives a different y.
    K = N = 64
    rng = np.random.default_rng(21)
    pi, sig, tau = rng.permutation(N), rng.permutation(N), np.roll(np.arange(N), 5)
    a, c, d = 0.5, 2.0, -1.5
    wg = np.zeros((N, K), np.float32); wg[np.arange(N), pi] = a
    wu = np.zeros((N, K), np.float32); wu[np.arange(N), sig] = c
    wd = np.zeros((N, K), np.float32); wd[np.arange(N), tau] = d
    x = _bf16(rng.standard_normal((6, K)))
    X = _f64(x)
    out = oracle.forward(x, _bf16(wg), _bf16(wu), _bf16(wd), 16, 4)
    assert np.array_equal(out["z"], a * X[:, pi])
    expect = np.zeros((6, K))
    expect[:, tau] = d * c * X[:, sig] * np.maximum(a * X[:, pi], 0.0)
    assert np.max(np.abs(out["y"] - expect)) <= 1e-13
    assert np.max(np.abs(oracle.ffn_dense(x, _bf16(wg), _bf16(wu), _bf16(wd)) - expect)) <= 1e-13


def test_all_gates_off_and_all_on():
    M, K, N = 4, 64, 128
    x, wg, wu, wd = _rand_problem(M, K, N, seed=8, bias=1e4)        # b = +large: all off
    out = oracle.forward(x, wg, wu, wd, 32, 4)
    assert not out["counts"].any() and not out["y"].any()
    x, wg, wu, wd = _rand_problem(M, K, N, seed=8, bias=-1e4)       # b = -large: all on
    out = oracle.forward(x, wg, wu, wd, 32, 4)
    assert out["overflow"].all()
    yn = _numpy_ffn(x, wg, wu, wd)
    assert np.max(np.abs(out["y"] - yn)) <= 1e-12 * np.max(np.abs(yn))


# ---------------------------------------------------------------- golden
def _read_golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [float(v) for v in rest]
    return vals


def test_hand_worked_golden_example():
    g = _read_golden()
    M, K, N, T, C = (int(g[k][0]) for k in ("M", "K", "N", "T", "C"))
    x = _bf16(np.array(g["x"]).reshape(M, K))
    wg = _bf16(np.array(g["wg_t"]).reshape(N, K))
    wu = _bf16(np.array(g["wu_t"]).reshape(N, K))
    wd = _bf16(np.array(g["wd"]).reshape(N, K))
    out = oracle.forward(x, wg, wu, wd, T, C)
    assert np.array_equal(out["z"], np.array(g["z"]).reshape(M, N))
    assert np.array_equal(out["counts"], np.array(g["counts"]).reshape(M, N // T))
    assert np.array_equal(out["overflow"], np.array(g["overflow"]).reshape(M, N // T))
    assert np.array_equal(out["idx"], np.array(g["idx"]).reshape(M, N // T, C))
    assert np.array_equal(out["vals"], np.array(g["vals"]).reshape(M, N // T, C))
    assert np.array_equal(out["dense"], np.array(g["dense"]).reshape(M, N))
    assert np.array_equal(out["y"], np.array(g["y"]).reshape(M, K))
    assert np.array_equal(oracle.ffn_dense(x, wg, wu, wd), np.array(g["y"]).reshape(M, K))


# ---------------------------------------------------------------- generator
def test_generator_hits_target_activation_fraction():
    # Closed form E_s[Q(b/(s sigma))] vs the measured fraction on a fresh draw.
    w = wl.Workload("t", 512, 256, 512, 128, 8, 7, p_mean=0.02, scale_sigma=0.5)
    d = wl.generate(w)
    z = oracle.gate(d["x"], d["wg_t"])
    measured = (z > 0).mean()
    expected = wl.expected_active_fraction(d["sigma"], d["bias"], 0.5).mean()
    assert abs(expected - 0.02) < 0.002       # bf16 rounding of the bias moves it a little
    assert abs(measured - expected) < 0.25 * expected


def test_generator_truncation_keeps_prefix():
    full = wl.generate(wl.TINY_WORKLOAD)
    part = wl.generate(wl.TINY_WORKLOAD, M=10)
    assert np.array_equal(full["x"][:10], part["x"])
    assert np.array_equal(full["wg_t"], part["wg_t"])


# ---------------------------------------------------------------- backward oracle
from oracle import backward as ob  # noqa: E402


def _fd_problem(seed):
    """A tiny float64 problem whose gate pre-activations all stay at least 0.05
    away from 0, so that central differences never cross a ReLU kink."""
    for s in range(seed, seed + 500):
        rng = np.random.default_rng(s)
        M, K, N = 3, 8, 6
        X = rng.standard_normal((M, K))
        G = rng.standard_normal((N, K)) / np.sqrt(K)
        U = rng.standard_normal((N, K)) / np.sqrt(K)
        D = rng.standard_normal((N, K)) / np.sqrt(N)
        z = X @ G.T
        if np.abs(z).min() > 0.05 and 0 < (z > 0).sum() < z.size:
            return X, G, U, D, rng.standard_normal((M, K))
    raise AssertionError("no problem without kinks found")


@pytest.mark.parametrize("seed", [0, 100, 200])
def test_backward_matches_central_differences_of_the_forward(seed):
    # L = sum(R * y): dL/dy = R.  Every entry of x and of the three weights is
    # perturbed by +-eps in the plain float64 forward.
    X, G, U, D, R = _fd_problem(seed)
    got = ob.backward_f64(X, G, U, D, R)
    eps = 1e-6
    for name, A, key in (("x", X, "dx"), ("wg_t", G, "dwg_t"), ("wu_t", U, "dwu_t"), ("wd", D, "dwd")):
        fd = np.empty_like(A)
        for i in np.ndindex(A.shape):
            keep = A[i]
            A[i] = keep + eps
            lp = np.sum(R * ob.ffn_forward_f64(X, G, U, D))
            A[i] = keep - eps
            lm = np.sum(R * ob.ffn_forward_f64(X, G, U, D))
            A[i] = keep
            fd[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(got[key], fd, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_all_gates_off_is_zero_and_the_mask_argument_is_the_active_set():
    X, G, U, D, R = _fd_problem(300)
    off = ob.backward_f64(X, G, U, D, R, active=np.zeros((3, 6), bool))
    for k in ("dx", "dwg_t", "dwu_t", "dwd"):
        assert not off[k].any()
    a = ob.backward_f64(X, G, U, D, R)
    b = ob.backward_f64(X, G, U, D, R, active=(X @ G.T) > 0)
    for k in ("dx", "dwg_t", "dwu_t", "dwd"):
        assert np.array_equal(a[k], b[k])


def test_backward_bits_entry_point_widens_bf16_exactly():
    x, wg, wu, wd, *_ = _rand_problem(4, 64, 128, seed=5)
    dy = np.random.default_rng(6).standard_normal((4, 64))
    a = ob.ffn_backward(x, wg, wu, wd, dy)
    b = ob.backward_f64(_f64(x), _f64(wg), _f64(wu), _f64(wd), dy)
    for k in ("dx", "dwg_t", "dwu_t", "dwd"):
        assert np.array_equal(a[k], b[k])
