"""Hidden-unit (N) sharded forward of the sparse gated FFN over P ranks.

Rank r holds the hidden units [n0_r, n1_r) of all three weights (rows of
W_g^T, W_u^T and W_d; every shard a whole number of TwELL tiles).  Because y
is a sum over hidden units ("Sparser, Faster, Lighter Transformer Language
Models", §3-5: y_m = sum over the active n of g (x_m W_u[:,n]) W_d[n,:]), each
rank computes the full sparse forward of its shard -- its own TwELL tiles,
its own dense-row slots for its own overflow tiles -- and the partial sums
are added across ranks with one collective: all-reduce (every rank gets y) or
reduce-scatter (rank r gets rows [r*M/P, (r+1)*M/P) of y).  The gate bias
lives in column K-1 of each unit's W_g^T row, so it shards with its unit.

Every rank takes the same collective steps in the same order: the local
forwards run in synchronous mode, the ranks agree on a capacity retry with one
MAX all-reduce of the dense-row demand, and only then reduce y.  The compute
step is injectable (`compute=`), so the host logic runs on CPU gloo ranks in
the tests; the default compute is the CUDA path (twell_ffn_fused).
"""
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist


def shard_bounds(N: int, T: int, world: int, rank: int) -> Tuple[int, int]:
    """Hidden units [n0, n1) of `rank`: the N/T TwELL tiles dealt out in
    contiguous runs whose lengths differ by at most one tile."""
    if N % T:
        raise ValueError(f"N={N} is not a multiple of T={T}")
    tiles = N // T
    if tiles < world:
        raise ValueError(f"{tiles} TwELL tiles cannot be shared by {world} ranks")
    t0 = rank * tiles // world
    t1 = (rank + 1) * tiles // world
    return t0 * T, t1 * T


def scatter_rows(M: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [m0, m1) of y that `rank` receives from the reduce-scatter."""
    if M % world:
        raise ValueError(f"M={M} rows do not split evenly over {world} ranks")
    return rank * M // world, (rank + 1) * M // world


# compute(x, wg_t, wu_t, wd, T, C, r_cap) -> (y_partial fp32 [M][K], n_over);
# raises CapacityNeeded when the dense-row slots ran out.
Compute = Callable[..., Tuple[torch.Tensor, int]]


class CapacityNeeded(RuntimeError):
    def __init__(self, n_over: int):
        super().__init__(f"{n_over} rows need a dense-row slot")
        self.n_over = n_over


def cuda_compute(x, wg_t, wu_t, wd, T, C, r_cap):
    """The local forward on this rank's GPU (twell_ffn_fused, synchronous)."""
    from . import twell as tw

    M, K = x.shape
    N = wg_t.shape[0]
    buf = tw.TwellBuffers(M, K, N, T, C, R_cap=r_cap, device=x.device)
    try:
        y = tw.ffn_fused(x, wg_t, wu_t, wd, buf, sync=True)
    except tw.CapacityError as e:
        raise CapacityNeeded(e.n_over) from None
    return y, buf.n_over_known


class ShardedFFN:
    """One rank's part of the N-sharded sparse FFN.

    wg_t, wu_t, wd are the FULL [N][K] weights or this rank's shard already
    ([n1 - n0][K]); T, C the TwELL tile width and capacity."""

    def __init__(self, wg_t, wu_t, wd, N: int, T: int, C: int, rank: int, world: int, group=None,
                 compute: Optional[Compute] = None):
        self.N, self.T, self.C = N, T, C
        self.rank, self.world, self.group = rank, world, group
        self.n0, self.n1 = shard_bounds(N, T, world, rank)
        rows = self.n1 - self.n0

        def local(w):
            return w if w.shape[0] == rows and rows != N else w[self.n0:self.n1].contiguous()

        self.wg_t, self.wu_t, self.wd = local(wg_t), local(wu_t), local(wd)
        self.compute = compute or cuda_compute
        self.r_cap = None  # dense-row slots of the last pass (None: the library default, M/8)

    def _local(self, x) -> Tuple[torch.Tensor, int]:
        M = x.shape[0]
        cap = self.r_cap or max(1, -(-M // 8))
        need = 0
        try:
            y, n_over = self.compute(x, self.wg_t, self.wu_t, self.wd, self.T, self.C, cap)
        except CapacityNeeded as e:
            y, n_over, need = None, e.n_over, e.n_over
        # Every rank learns the largest demand; ranks that ran out redo their
        # shard with room for it (one retry is enough: the demand is exact).
        demand = torch.tensor([need], dtype=torch.int64, device=x.device)
        if self.world > 1:
            dist.all_reduce(demand, op=dist.ReduceOp.MAX, group=self.group)
        if int(demand.item()) > 0:
            self.r_cap = max(cap, int(demand.item()))
            if y is None:
                y, n_over = self.compute(x, self.wg_t, self.wu_t, self.wd, self.T, self.C, self.r_cap)
        return y, n_over

    def forward(self, x: torch.Tensor, mode: str = "all_reduce") -> torch.Tensor:
        """y (fp32) of the whole FFN: all of it ("all_reduce") or this rank's
        rows of it ("reduce_scatter")."""
        y, _ = self._local(x)
        if self.world == 1:
            return y
        if mode == "all_reduce":
            dist.all_reduce(y, group=self.group)
            return y
        if mode == "reduce_scatter":
            m0, m1 = scatter_rows(y.shape[0], self.world, self.rank)
            out = torch.empty((m1 - m0, y.shape[1]), dtype=y.dtype, device=y.device)
            if dist.get_backend(self.group) == "nccl":
                dist.reduce_scatter_tensor(out, y, group=self.group)
            else:  # gloo has no reduce-scatter: reduce everything, keep this rank's rows
                dist.all_reduce(y, group=self.group)
                out.copy_(y[m0:m1])
            return out
        raise ValueError(f"unknown mode {mode!r}")
