"""Seeded synthetic inputs for the ReLU-gated sparse FFN.

This module is shared by the CUDA path, the CPU oracle, the tests and the
benchmark.  It holds no arithmetic of the method itself: it draws random
numbers, rounds them to bf16 and picks per-neuron gate biases so that the gate
``ReLU(x W_g)`` fires with a chosen probability.  Everything it returns is raw
bf16 bit patterns (``uint16`` arrays) so that both sides start from the same
bytes.

Workload shapes follow the pages' model (K=2048, N=5632, "Sparser, Faster,
Lighter Transformer Language Models", §4-1 model table) and their sparsity
regime (tens of active neurons per token out of 5632, §5-1/§5-2; per-token
counts varying more than 10x, §5-3).  The pages measure trained checkpoints
on FineWeb; neither exists here, so these generators stand in for them.

Layout (all row-major):
  x     [M][K]  tokens; column K-1 is fixed to 1.0 so the gate bias rides in
                the GEMM (W_g row K-1 holds -b_n)
  wg_t  [N][K]  W_g transposed (row n = input weights of gate neuron n)
  wu_t  [N][K]  W_u transposed (row n = input weights of up neuron n)
  wd    [N][K]  W_d (row n = output weights of hidden neuron n)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np
from scipy import special as _sp


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); returns uint16 bits.

    Inputs here are finite, so the NaN special case is not needed.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic gated-FFN problem.

    Activation model: for token m and neuron n the gate pre-activation is
    z = s_m * (x_m[:K-1] . w_n[:K-1]) - b_n with x ~ N(0,1) i.i.d., so
    P(z > 0) = E_s[Q(b_n / (s * sigma_n))], sigma_n = ||w_n[:K-1]||.
    b_n is solved per neuron so that this probability equals the target p_n.
    """
    name: str
    M: int
    K: int
    N: int
    T: int            # TwELL tile width (= gate GEMM output tile width)
    C: int            # TwELL capacity per (row, tile)
    seed: int
    p_mean: Optional[float] = None                     # same target for every neuron
    p_loguniform: Optional[Tuple[float, float]] = None  # per-neuron target ~ log-uniform
    scale_sigma: float = 0.0                          # token scale s ~ lognormal(0, sigma)
    boost_frac: float = 0.0                           # fraction of tokens with s = boost_scale
    boost_scale: float = 1.0
    r_cap: Optional[int] = None                       # dense-row capacity; default ceil(M/8)

    @property
    def R_cap(self) -> int:
        return self.r_cap if self.r_cap is not None else max(1, -(-self.M // 8))

    def describe(self) -> dict:
        d = dataclasses.asdict(self)
        d["R_cap"] = self.R_cap
        return d


def _sweep(M: int, p: float, seed: int) -> Workload:
    C = 32 if p >= 0.05 else 8
    tag = {0.1: "p90", 0.01: "p99", 0.001: "p999"}[p]
    return Workload(f"sweep_m{M}_k2048_n8192_{tag}", M, 2048, 8192, 128, C, seed, p_mean=p)


#: The five workload families.  Names say what each one is.
WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny_m64_k256_n1024_p98", 64, 256, 1024, 128, 16, 0, p_mean=0.02),
        Workload("m2048_k1536_n4096_p99_lognormal05", 2048, 1536, 4096, 128, 8, 1,
                 p_mean=0.01, scale_sigma=0.5),
        Workload("m8192_k2048_n5632_loguniform_lognormal07", 8192, 2048, 5632, 128, 8, 2,
                 p_loguniform=(1e-4, 5e-2), scale_sigma=0.7),
        Workload("m16384_k2560_n10240_p99_boost3pct", 16384, 2560, 10240, 256, 16, 3,
                 p_mean=0.01, boost_frac=0.03, boost_scale=4.0),
    ] + [_sweep(M, p, 10 + i * 3 + j)
         for i, M in enumerate([16, 64, 256, 1024, 4096])
         for j, p in enumerate([0.1, 0.01, 0.001])]
}

#: The single-GPU throughput workload: the largest configuration at 99% sparsity.
BENCH_WORKLOAD = "m16384_k2560_n10240_p99_boost3pct"
#: The small case the oracle finishes in seconds.
TINY_WORKLOAD = "tiny_m64_k256_n1024_p98"
PARITY_WORKLOADS: List[str] = [
    "tiny_m64_k256_n1024_p98",
    "m2048_k1536_n4096_p99_lognormal05",
    "m8192_k2048_n5632_loguniform_lognormal07",
    "m16384_k2560_n10240_p99_boost3pct",
]


def _scale_nodes(scale_sigma: float, boost_frac: float, boost_scale: float):
    """Quadrature (values, weights) for the distribution of the token scale s."""
    if scale_sigma > 0:
        xi, w = np.polynomial.hermite_e.hermegauss(64)
        s = np.exp(scale_sigma * xi)
        w = w / w.sum()
    else:
        s, w = np.array([1.0]), np.array([1.0])
    if boost_frac > 0:
        s = np.concatenate([s, s * boost_scale])
        w = np.concatenate([w * (1 - boost_frac), w * boost_frac])
    return s, w


def solve_bias(sigma: np.ndarray, p: np.ndarray, s_nodes: np.ndarray, s_w: np.ndarray) -> np.ndarray:
    """Per-neuron b_n >= 0 with E_s[Q(b_n / (s sigma_n))] = p_n (bisection, fp64)."""
    sigma = np.asarray(sigma, dtype=np.float64)
    p = np.broadcast_to(np.asarray(p, dtype=np.float64), sigma.shape)
    lo = np.zeros_like(sigma)
    hi = np.full_like(sigma, 40.0) * sigma * s_nodes.max()

    def frac(b):
        return (s_w[None, :] * _sp.ndtr(-(b[:, None] / (sigma[:, None] * s_nodes[None, :])))).sum(1)

    for _ in range(80):
        mid = 0.5 * (lo + hi)
        too_many = frac(mid) > p          # fires too often -> raise the bias
        lo = np.where(too_many, mid, lo)
        hi = np.where(too_many, hi, mid)
    return 0.5 * (lo + hi)


def expected_active_fraction(sigma, b, scale_sigma=0.0, boost_frac=0.0, boost_scale=1.0) -> np.ndarray:
    """Closed-form P(z > 0) per neuron for the given biases."""
    s, w = _scale_nodes(scale_sigma, boost_frac, boost_scale)
    sigma = np.asarray(sigma, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return (w[None, :] * _sp.ndtr(-(b[:, None] / (sigma[:, None] * s[None, :])))).sum(1)


def generate(wl: Workload | str, M: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw one workload.  Returns bf16 bit arrays plus generator metadata.

    ``M`` optionally truncates the token count (the weights, biases and the
    first M tokens are identical to the full draw's).
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    Mfull, K, N = wl.M, wl.K, wl.N
    rng = np.random.default_rng(wl.seed)
    # Weights first so that truncating M leaves them unchanged.
    wg = rng.standard_normal((N, K), dtype=np.float32) * np.float32(1.0 / math.sqrt(K))
    wu = rng.standard_normal((N, K), dtype=np.float32) * np.float32(1.0 / math.sqrt(K))
    wd = rng.standard_normal((N, K), dtype=np.float32) * np.float32(1.0 / math.sqrt(N))
    wg_t = f32_to_bf16_bits(wg)
    wu_t = f32_to_bf16_bits(wu)
    wd_b = f32_to_bf16_bits(wd)
    del wg, wu, wd
    if wl.p_loguniform is not None:
        lo, hi = wl.p_loguniform
        p = np.exp(rng.uniform(math.log(lo), math.log(hi), size=N))
    else:
        p = np.full(N, float(wl.p_mean))
    sigma = np.sqrt((bf16_bits_to_f32(wg_t[:, :K - 1]).astype(np.float64) ** 2).sum(1))
    s_nodes, s_w = _scale_nodes(wl.scale_sigma, wl.boost_frac, wl.boost_scale)
    b = solve_bias(sigma, p, s_nodes, s_w)
    wg_t[:, K - 1] = f32_to_bf16_bits((-b).astype(np.float32))
    b_used = -bf16_bits_to_f32(wg_t[:, K - 1]).astype(np.float64)

    # Token scales and activations.
    if wl.scale_sigma > 0:
        s = np.exp(rng.normal(0.0, wl.scale_sigma, size=Mfull))
    else:
        s = np.ones(Mfull)
    if wl.boost_frac > 0:
        nb = int(round(wl.boost_frac * Mfull))
        boosted = rng.choice(Mfull, size=nb, replace=False)
        s[boosted] *= wl.boost_scale
    Muse = Mfull if M is None else int(M)
    assert 0 <= Muse <= Mfull
    x = rng.standard_normal((Mfull, K), dtype=np.float32)[:Muse]
    x *= s[:Muse, None].astype(np.float32)
    x[:, K - 1] = 1.0
    x_b = f32_to_bf16_bits(x)
    del x
    return {
        "x": x_b, "wg_t": wg_t, "wu_t": wu_t, "wd": wd_b,
        "scale": s[:Muse], "p_target": p, "sigma": sigma, "bias": b_used,
    }


def subsample_rows(M: int, n: int, seed: int = 1234) -> np.ndarray:
    """Sorted seeded sample of n distinct rows in [0, M) (all rows if n >= M)."""
    if n >= M:
        return np.arange(M, dtype=np.int64)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(M, size=n, replace=False)).astype(np.int64)
