"""fp64 CPU oracle of the ReLU-gated FFN backward pass (TEST INFRASTRUCTURE).

Only ``tests/`` may import this module; the CUDA library never calls it and
the two share no code.

The forward pass ("Sparser, Faster, Lighter Transformer Language Models"
review page, §1-1) is, per token row x (weights stored as rows: wg_t[n],
wu_t[n], wd[n] are hidden unit n's rows of W_g^T, W_u^T and W_d):

    z_n = x . wg_t[n],  g_n = ReLU(z_n),  u_n = x . wu_t[n],  h_n = u_n g_n,
    y = sum_n h_n wd[n].

Its gradients for an upstream gradient dy of y follow by the chain rule, the
derivative of ReLU taken as 1 where the unit is active (z_n > 0) and 0 where it
is not (the training path of §3-6 and §3-7 keeps exactly the active set):

    dh_n = dy . wd[n]
    du_n = dh_n g_n                       (d h_n / d u_n = g_n)
    dz_n = dh_n u_n [active_n]            (d h_n / d z_n = u_n ReLU'(z_n))
    dx   = sum_n du_n wu_t[n] + dz_n wg_t[n]
    dwd[n]   = sum over rows of h_n dy
    dwu_t[n] = sum over rows of du_n x
    dwg_t[n] = sum over rows of dz_n x

Inactive units contribute nothing: g_n = h_n = du_n = dz_n = 0.  `active`
defaults to z > 0 computed here; a caller may pass the active set a forward
pass chose instead (the two differ only where z is within rounding of 0).

Every input is taken as bf16 bit patterns (uint16) except dy (any float
array); all arithmetic is float64 with numpy matmuls as the only library step.
Pinned by tests/test_oracle_pins.py (finite differences of the fp64 forward,
a closed form with permutation weights, and the all-off case).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np


def _f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def backward_f64(X, G, U, D, dy, active: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """The gradients above on float64 arrays X [M][K], G, U, D [N][K]."""
    dy = np.asarray(dy, dtype=np.float64)
    z = X @ G.T
    u = X @ U.T
    a = (z > 0) if active is None else np.asarray(active, dtype=bool)
    g = np.where(a, z, 0.0)
    h = u * g
    dh = dy @ D.T
    du = dh * g
    dz = np.where(a, dh * u, 0.0)
    return {
        "dx": du @ U + dz @ G,
        "dwg_t": dz.T @ X,
        "dwu_t": du.T @ X,
        "dwd": h.T @ dy,
        "active": a,
        "z": z,
    }


def ffn_backward(x, wg_t, wu_t, wd, dy, active: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """dx [M][K], dwg_t, dwu_t, dwd [N][K] (float64) for upstream gradient dy [M][K];
    x and the weights as bf16 bit patterns."""
    return backward_f64(_f64(x), _f64(wg_t), _f64(wu_t), _f64(wd), dy, active)


def ffn_forward_f64(X, G, U, D):
    """The §1-1 forward on float64 arrays (for finite-difference pins)."""
    z = X @ G.T
    return ((X @ U.T) * np.maximum(z, 0.0)) @ D
