"""The roofline arithmetic bench.py reports, recomputed by hand (CPU only).

The path roofline of the sparse gated FFN forward is
T_roof = max(2MKN / P_tc, B_alg / BW_hbm); the reported fraction is T_roof
divided by the measured step time.  These tests pin the byte and FLOP counts
on a case small enough to add up by hand, and check that every fraction in the
reported objects follows from the other fields of the same object."""
import math

import bench

PEAKS = {"hbm_gbs": 1000.0, "bf16_tflops": 1.0}  # 1 TB/s, 1 TFLOP/s


def test_path_roofline_hand_case():
    # M=2 rows, K=4, N=8 hidden units in tiles of T=4 (two tiles), C=1 slot,
    # U=3 unique up/down rows gathered, R=1 dense-row slot.
    r = bench.path_roofline(M=2, K=4, N=8, T=4, C=1, U=3, R=1, peaks=PEAKS, ms=1.0, entries=5)
    # W_g 2*4*8 = 64; W_u, W_d rows 4*4*3 = 48; x 2*2*4 = 16; y fp32 4*2*4 = 32;
    # TwELL 2*2*2*(2 + 3*1) = 40; dense-row backup 4*1*8 = 32.
    assert r["bytes"] == 64 + 48 + 16 + 32 + 40 + 32 == 232
    assert r["flops"] == 2 * 2 * 4 * 8 == 128
    t_hbm_ms = 232 / 1000e9 * 1e3
    t_tc_ms = 128 / 1e12 * 1e3
    assert math.isclose(r["t_roof_ms"], max(t_hbm_ms, t_tc_ms))
    assert r["bound"] == "hbm"
    assert math.isclose(r["frac"], r["t_roof_ms"] / 1.0)
    # fp32 ALU time of the sparse products: 4K FLOP per listed entry at 74.4 TFLOP/s.
    assert math.isclose(r["t_alu_sparse_ms"], 4 * 4 * 5 / 74.4e12 * 1e3)
    # The stored-format variant: fp32 values (5 bytes per slot) and fp32 gates.
    assert r["bytes_fp32_vals_variant"] == 64 + 48 + 16 + 32 + 2 * 2 * 2 * (2 + 5) + 8 * 8


def test_path_roofline_tensor_bound_when_flops_dominate():
    r = bench.path_roofline(M=4096, K=2048, N=8192, T=128, C=8, U=8192, R=0,
                            peaks={"hbm_gbs": 1e6, "bf16_tflops": 1.0}, ms=200.0)
    assert r["bound"] == "tensor"
    assert math.isclose(r["t_roof_ms"], 2.0 * 4096 * 2048 * 8192 / 1e12 * 1e3)


def test_path_roofline_fraction_follows_from_its_fields():
    for (M, K, N, T, C, U, R, ms) in [(4096, 2048, 8192, 128, 8, 6000, 17, 1.2),
                                      (128, 2048, 5632, 64, 4, 900, 0, 0.05),
                                      (16, 4096, 11008, 128, 16, 300, 2, 0.03)]:
        r = bench.path_roofline(M, K, N, T, C, U, R, PEAKS, ms)
        t_roof = max(r["flops"] / (r["P_tc_tflops"] * 1e12), r["bytes"] / (r["BW_hbm_gbs"] * 1e9)) * 1e3
        assert math.isclose(r["t_roof_ms"], t_roof)
        assert math.isclose(r["frac"], t_roof / ms)
        assert r["t_step_ms"] == ms
