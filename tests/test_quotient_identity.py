"""The NVFP4 quantizers' division shortcut, checked on the CPU in exact arithmetic.

The kernels divide each value of a block by its E4M3 scale s as r = RN(1/s), y = RN(x r),
q = RN(y + (x - y s) r) (the remainder x - y s is exact in one fma), which is RN(x / s) by
Markstein's theorem; the oracle divides.  Here the sequence is emulated in float32 with exact
float64 products for every positive E4M3 scale and x drawn over the block's range plus the E2M1
grid midpoints times s and their float32 neighbours, and compared with the correctly rounded
quotient.  (The GPU tests compare the quantizers' NVFP4 codes with the oracle bit for bit.)"""
import numpy as np


def _e4m3_positive():
    vals = []
    for b in range(0x7F):  # 0x7F is NaN
        e, m = b >> 3, b & 7
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        if v > 0:
            vals.append(v)
    return np.array(vals)


def _round32(x64):
    return x64.astype(np.float32)


def test_markstein_quotient_is_the_correctly_rounded_quotient():
    rng = np.random.default_rng(7)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    scales = _e4m3_positive()
    assert len(scales) == 126 and scales.max() == 448.0
    checked = 0
    for s64 in scales:
        s = np.float32(s64)
        assert np.float64(s) == s64
        r = _round32(np.float64(1.0) / s64)
        x = _round32(rng.uniform(0, 7, 4000) * s64)
        xm = _round32(mids * s64)
        near = np.concatenate([xm + k * np.spacing(xm) for k in range(-3, 4)]).astype(np.float32)
        x = np.concatenate([x, near, np.float32([0.0, 1e-30])])
        y = _round32(x.astype(np.float64) * np.float64(r))
        rem = _round32(x.astype(np.float64) - y.astype(np.float64) * s64)  # exact
        assert np.array_equal(rem.astype(np.float64), x.astype(np.float64) - y.astype(np.float64) * s64)
        q = _round32(y.astype(np.float64) + rem.astype(np.float64) * np.float64(r))
        exact = _round32(x.astype(np.float64) / s64)
        assert np.array_equal(q, exact), f"scale {s64}: {np.count_nonzero(q != exact)} differ"
        checked += x.size
    assert checked > 500_000
