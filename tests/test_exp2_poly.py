"""The software 2^x of the attention kernels (pba_ptx.cuh, exp2_poly2).

CPU: the same steps replayed in numpy fp32 (range reduction with the
1.5*2^23 + 127 shifter, degree-4 polynomial, exponent-field scale) against
float64 2^x.  GPU: the kernel's own routine through pba_selftest_exp2 against
torch.exp2 in float64 and against the hardware exp2.
"""
import numpy as np
import pytest
import torch

# the coefficients compiled into pba_ptx.cuh (written by fit_exp2_poly.py)
C = np.array([1.0, 6.931241155e-01, 2.402410656e-01, 5.590682849e-02, 9.582576342e-03], dtype=np.float32)


def replay(x):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    shift = np.float32(12583039.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = np.full_like(f, C[4])
    for c in C[3::-1]:  # fused multiply-add: one rounding of the exact q*f + c
        q = (q.astype(np.float64) * f.astype(np.float64) + np.float64(c)).astype(np.float32)
    scale = (t.view(np.uint32) << np.uint32(23)).view(np.float32)
    return (q * scale).astype(np.float32)


def test_replay_accuracy_and_zero_flush():
    x = np.linspace(-126.0, 9.0, 2_000_001, dtype=np.float32)
    y = replay(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-5
    z = replay(np.array([-np.inf, -127.0, -127.4, -200.0, -1e30], dtype=np.float32))
    assert np.all(z == 0.0)
    # integers are exact powers of two (the constant term is exactly 1)
    k = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(replay(k).astype(np.float64), np.exp2(k.astype(np.float64)))


@pytest.mark.gpu
def test_kernel_exp2_matches_exp2(cuda_device):
    import pair_biased_attention_b200 as pba

    x = torch.linspace(-126.0, 9.0, 1 << 22, device=cuda_device)
    y = pba.pba_selftest_exp2(x)
    ref = torch.exp2(x.double())
    rel = (y.double() / ref - 1.0).abs().max().item()
    assert rel < 1e-5, rel
    specials = torch.tensor([-float("inf"), -127.0, -130.0, -1e30], device=cuda_device)
    assert torch.all(pba.pba_selftest_exp2(specials) == 0)
    # agrees with the CPU replay of the same fp32 steps to within one unit in the last place
    xs = torch.linspace(-30.0, 8.0, 100_003, device=cuda_device)
    g = pba.pba_selftest_exp2(xs).cpu().numpy()
    r = replay(xs.cpu().numpy())
    assert np.abs(g.view(np.int32).astype(np.int64) - r.view(np.int32).astype(np.int64)).max() <= 1
    k = torch.arange(-126, 9, dtype=torch.float32, device=cuda_device)
    assert torch.equal(pba.pba_selftest_exp2(k).double(), torch.exp2(k.double()))
