"""B200-native (sm_100a) forward path of the ReLU-gated sparse FFN with TwELL.

    y = (x W_u  (.)  ReLU(x W_g)) W_d

computed as a tcgen05 gate GEMM whose epilogue packs the ReLU gate into TwELL
(Tile-wise ELLPACK), a fused sparse up+down kernel over the active units, and
a dense-row tensor-core path for tiles that overflow the TwELL capacity.
"""
from .twell import (  # noqa: F401
    CapacityError,
    KernelTrace,
    TwellBuffers,
    TwellError,
    dense_ffn,
    ffn_fwd,
    gate_pack,
    last_launch_count,
    lib,
    read_status,
    sparse_ffn,
)
