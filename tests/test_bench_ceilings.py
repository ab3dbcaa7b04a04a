"""The benchmark's triangle-attention ceilings, checked on CPU against values
worked out by hand for tri1024 (N = 1024, H = 4, D = 32)."""
import math

import bench


def test_tri1024_counts_and_fractions():
    c = bench.tri_ceilings(1024, 4, 32, ms_per_call=2.0, tensor_tflops=1000.0, hbm_gbs=5000.0, sm_mhz=2000.0,
                           n_sms=100)
    # 4 N^3 H D = 2^2 * 2^30 * 2^2 * 2^5 = 2^39 FLOPs; N^3 H = 2^32 exponentials
    assert c["flops_per_call"] == 2.0 ** 39
    assert c["exps_per_call"] == 2.0 ** 32
    # q, k, v, gate, out: 5 * 2^20 * 128 * 2 B; lse 2^20 * 4 * 4 B; bias 4 * 2^20 * 2 B
    assert c["bytes_per_call"] == 5 * 2 ** 20 * 128 * 2 + 2 ** 20 * 16 + 4 * 2 ** 20 * 2
    assert math.isclose(c["floor_ms"]["tensor"], 2.0 ** 39 / 1e15 * 1e3)
    assert math.isclose(c["floor_ms"]["hbm"], c["bytes_per_call"] / 5e12 * 1e3)
    assert math.isclose(c["floor_ms"]["exp2"], 2.0 ** 32 / (16 * 100 * 2e9) * 1e3)
    for k in ("tensor", "hbm", "exp2"):
        assert math.isclose(c["frac"][k], c["floor_ms"][k] / 2.0)
