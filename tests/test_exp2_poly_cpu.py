"""Float32 emulation of the FMA-pipe 2^x (same operations as exp2_poly in tc_ptx.cuh)."""
import numpy as np

C = np.array([9.999992847e-01, 6.931217909e-01, 2.402473241e-01, 5.591790378e-02,
              9.570610709e-03], dtype=np.float32)


def exp2_poly(x):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = C[4]
    for k in (3, 2, 1, 0):
        p = (p * f + C[k]).astype(np.float32)   # fma emulated in fp32 (one rounding more)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32)
    y = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y - ref) / ref) <= 4e-6


def test_exact_integers_and_flush():
    for k in range(-120, 9):
        assert abs(exp2_poly(np.float32(k)) / 2.0 ** k - 1) <= 2e-6
    for v in (-126.0, -127.0, -1e30, -np.inf):
        y = exp2_poly(np.float32(v))
        assert np.isfinite(y) and 0.0 <= y <= 2.0 ** -125
