"""Run under torch.distributed.run on CPU (gloo): every rank runs its shard of
the N-sharded sparse FFN with the fp64 oracle as the compute step (a test
double for the CUDA path), reduces y, and writes what it got to
<out_dir>/rank<r>.npz (argv[1])."""
import datetime
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
from activation_sparse_gated_tma_b200 import tp  # noqa: E402
from activation_sparse_gated_tma_b200 import workloads as wl  # noqa: E402


def main():
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w = wl.Workload("tp_m8_k192_n1024", 8, 192, 1024, 128, 2, 21, p_mean=0.06)
        d = wl.generate(w)
        x = torch.from_numpy(d["x"].view(np.int16))
        calls = []

        def oracle_compute(x_, wg_t, wu_t, wd, T, C, r_cap):
            # Rank 1 claims one slot more than it is given on its first call:
            # both ranks must then agree on the retry.
            ref = oracle.forward(x_.numpy(), wg_t.numpy(), wu_t.numpy(), wd.numpy(), T, C)
            n_over = int(ref["overflow"].any(axis=1).sum())
            calls.append(r_cap)
            if rank == 1 and len(calls) == 1:
                raise tp.CapacityNeeded(r_cap + 1)
            if n_over > r_cap:
                raise tp.CapacityNeeded(n_over)
            return torch.from_numpy(ref["y"]), n_over

        full = {k: torch.from_numpy(d[k].view(np.int16)) for k in ("wg_t", "wu_t", "wd")}
        f = tp.ShardedFFN(full["wg_t"], full["wu_t"], full["wd"], w.N, w.T, w.C, rank, world,
                          compute=oracle_compute)
        y_all = f.forward(x, "all_reduce")
        y_rows = f.forward(x, "reduce_scatter")
        np.savez(os.path.join(sys.argv[1], f"rank{rank}.npz"), y_all=y_all.numpy(), y_rows=y_rows.numpy(),
                 n0=f.n0, n1=f.n1, calls=np.array(calls), r_cap=f.r_cap)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
