"""Host logic of the N-sharded forward (activation_sparse_gated_tma_b200.tp):
shard bounds, and two gloo ranks on CPU with the fp64 oracle standing in for
the CUDA compute step."""
import os

import numpy as np
import pytest

import oracle
from activation_sparse_gated_tma_b200 import tp
from activation_sparse_gated_tma_b200 import workloads as wl
from tests.test_multirank import ROOT, _torchrun


@pytest.mark.parametrize("N,T,world", [(1024, 128, 2), (5632, 128, 3), (10240, 256, 8), (256, 128, 2)])
def test_shards_cover_the_hidden_units_in_whole_tiles(N, T, world):
    bounds = [tp.shard_bounds(N, T, world, r) for r in range(world)]
    assert bounds[0][0] == 0 and bounds[-1][1] == N
    for (a0, a1), (b0, b1) in zip(bounds, bounds[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in bounds]
    assert all(s % T == 0 and s > 0 for s in sizes)
    assert max(sizes) - min(sizes) <= T


def test_shard_bounds_reject_too_many_ranks():
    with pytest.raises(ValueError):
        tp.shard_bounds(256, 128, 4, 0)
    with pytest.raises(ValueError):
        tp.scatter_rows(10, 4, 0)


def test_two_gloo_ranks_reduce_the_shard_partials_to_the_full_ffn():
    out = os.path.join(ROOT, "_build", "tp")
    os.makedirs(out, exist_ok=True)
    for k in range(2):
        p = os.path.join(out, f"rank{k}.npz")
        if os.path.exists(p):
            os.remove(p)
    r = _torchrun([os.path.join("tests", "_tp_helper.py"), out])
    assert r.returncode == 0, r.stderr[-3000:]
    w = wl.Workload("tp_m8_k192_n1024", 8, 192, 1024, 128, 2, 21, p_mean=0.06)
    d = wl.generate(w)
    ref = oracle.forward(d["x"], d["wg_t"], d["wu_t"], d["wd"], w.T, w.C)["y"]
    got = [np.load(os.path.join(out, f"rank{k}.npz")) for k in range(2)]
    assert [int(g["n0"]) for g in got] == [0, 512] and [int(g["n1"]) for g in got] == [512, 1024]
    scale = np.abs(ref).max()
    for k, g in enumerate(got):
        np.testing.assert_allclose(g["y_all"], ref, rtol=0, atol=1e-12 * scale)
        np.testing.assert_allclose(g["y_rows"], ref[4 * k:4 * k + 4], rtol=0, atol=1e-12 * scale)
    # The first pass ran out of dense-row slots (rank 1 also claims one more
    # than it is given): both ranks agreed on the largest demand, redid their
    # shards with it, and the second forward started from it.
    demand = []
    for k in range(2):
        n0, n1 = tp.shard_bounds(w.N, w.T, 2, k)
        sh = oracle.forward(d["x"], d["wg_t"][n0:n1], d["wu_t"][n0:n1], d["wd"][n0:n1], w.T, w.C)
        demand.append(int(sh["overflow"].any(axis=1).sum()))
    cap = max(demand + [2])
    assert cap > 1
    for g in got:
        assert int(g["r_cap"]) == cap
        assert list(g["calls"]) == [1, cap, cap]
