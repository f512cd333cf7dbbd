"""The N-sharded forward's arithmetic on one GPU: the shards of
activation_sparse_gated_tma_b200.tp are computed one after another with the
CUDA path (each with its own TwELL and dense-row slots) and their partial y
added, which is what the all-reduce does across ranks; compared with the
fp64 oracle of the unsharded FFN."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gated_tma_b200 import tp
from tests import parity as P
from tests.test_gpu_parity import _small

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,world", [(16, 2), (16, 4), (300, 2), (300, 3)])
def test_shard_partials_add_up_to_the_full_ffn(M, world):
    w, d, dev = _small(M, 256, 2048, 128, 4, None, seed=M + world, R_cap=M)
    y = torch.zeros(M, w.K, dtype=torch.float32, device="cuda")
    for r in range(world):
        n0, n1 = tp.shard_bounds(w.N, w.T, world, r)
        yr, n_over = tp.cuda_compute(dev["x"], dev["wg_t"][n0:n1].contiguous(), dev["wu_t"][n0:n1].contiguous(),
                                     dev["wd"][n0:n1].contiguous(), w.T, w.C, M)
        y += yr
    torch.cuda.synchronize()
    ref = oracle.forward(d["x"], d["wg_t"], d["wu_t"], d["wd"], w.T, w.C)["y"]
    print(M, world, P.check_y(y.cpu().numpy(), ref, "sharded y"))
