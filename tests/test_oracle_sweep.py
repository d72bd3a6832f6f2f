"""Pins of the oracle's per-block Qmax sweep (the scale-rule diagnostic).

A block holding one nonzero value v in (6, 8) (times 2^k) has a closed form: for a boundary q < v
the ceiling rule takes the next exponent, so v/2 in (3, 4) rounds to the nearer of 3 and 4 (ties to
the even code, 4) and comes back doubled; for q >= v the scale keeps v, which saturates to 6.  The
optimal boundaries are those with the smaller squared error.  Zero elements cost nothing."""
import numpy as np
import pytest

import oracle

QS = oracle.qmax_grid()  # 6.00, 6.05, ..., 8.00 (41 values)


def _lone(v: float, k: int = 0) -> np.ndarray:
    x = np.zeros((1, 32), np.float32)
    x[0, 5] = np.float32(v * 2.0 ** k)
    return x


def _closed_form(v: float):
    v = float(np.float32(v))  # the value the block holds
    half = v / 2
    lo, hi = 3.0, 4.0
    below = hi if (half - lo) > (hi - half) or (half - lo) == (hi - half) else lo  # ties to 4 (even code)
    err_below = (v - 2 * below) ** 2      # q < v
    err_above = (v - 6.0) ** 2            # q >= v
    sse = np.where(QS < np.float32(v), err_below, err_above)
    return sse, (sse == sse.min()).astype(np.uint64)


def test_grid_is_six_to_eight_in_steps_of_0_05():
    assert QS.size == 41 and QS[0] == 6.0 and QS[-1] == 8.0
    assert np.allclose(np.diff(QS.astype(np.float64)), 0.05, atol=1e-6)
    assert np.float32(7.25) in QS


@pytest.mark.parametrize("v", [6.25, 6.5, 7.0, 7.25, 7.5, 7.75, 7.9])
@pytest.mark.parametrize("k", [0, -3, 5])
def test_lone_value_matches_the_closed_form(v, k):
    counts, sums = oracle.qmax_sweep(_lone(v, k), QS)
    sse, opt = _closed_form(v)
    np.testing.assert_array_equal(counts, opt)
    np.testing.assert_allclose(sums, sse * 4.0 ** k, rtol=0, atol=0)


def test_values_on_the_grid_are_free_for_every_boundary():
    x = np.zeros((2, 32), np.float32)
    x[0, :8] = [6, 4, 3, 2, 1.5, 1, 0.5, 0]
    x[1, :4] = [-6, -0.5, 3, 1.5]
    x[1] *= np.float32(2.0 ** -7)
    counts, sums = oracle.qmax_sweep(x, QS)
    assert (counts == 2).all() and (sums == 0).all()


def test_scaling_a_block_by_a_power_of_two_scales_only_the_error():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 96)).astype(np.float32)
    c0, s0 = oracle.qmax_sweep(x, QS)
    c1, s1 = oracle.qmax_sweep(x * np.float32(2.0 ** 9), QS)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_allclose(s1, s0 * 4.0 ** 9, rtol=1e-15)


def test_every_group_counts_for_at_least_one_boundary_and_tails_are_padded():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((10, 70)).astype(np.float32)  # 3 groups per row, the last 6 wide
    counts, _ = oracle.qmax_sweep(x, QS)
    groups = 10 * 3
    assert counts.max() <= groups and counts.sum() >= groups
    # the padded tail: the same as explicit zeros
    xp = np.zeros((10, 96), np.float32)
    xp[:, :70] = x
    cp, sp = oracle.qmax_sweep(xp, QS)
    c2, s2 = oracle.qmax_sweep(x, QS)
    np.testing.assert_array_equal(cp, c2)
    np.testing.assert_array_equal(sp, s2)


def test_rotation_flag_sweeps_the_rotated_rows():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    c0, s0 = oracle.qmax_sweep(oracle.rotate_rows(x), QS)
    c1, s1 = oracle.qmax_sweep(x, QS, rotate=True)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_array_equal(s0, s1)


def test_rowsum_decomposition_hand_example():
    """One row, one 64-key tile: group 0 holds the row max 1.0 (UOS exponent -2, step 0.25 at the
    top), group 1 has max 0.9 (exponent -3: 0.9 / 2^-3 = 7.2 saturates to 6)."""
    pt = np.zeros((1, 1, 64), np.float32)
    pt[0, 0, :5] = [1.0, 0.1, 0.05, 0.7, 0.6]
    pt[0, 0, 32:34] = [0.9, 0.3]
    codes, scales = oracle.quantize(pt.reshape(1, 64), axis=0)
    # hand quantization: 1.0 -> 1.0, 0.1 -> 0.125 (up), 0.05 -> 0 (zeroing), 0.7 -> 0.75 (up),
    # 0.6 -> 0.5 (down); 0.9 -> 0.75 (saturation), 0.3 -> 0.25 (down)
    assert list(scales[0]) == [127 - 2, 127 - 3]
    r = oracle.rowsum_decomposition(pt, codes.reshape(1, 1, 64), scales.reshape(1, 1, 2), np.zeros((1, 1)))
    total = 1.0 + 0.1 + 0.05 + 0.7 + 0.6 + 0.9 + 0.3
    expect = {"zeroing": -0.05, "saturation": -0.15, "down": -0.1 - 0.05, "up": 0.025 + 0.05}
    for k, v in expect.items():
        assert abs(r[k][0] - v / total) < 1e-7, (k, r[k][0], v / total)
    assert abs(r["rowsum_direct"][0] - (1 + sum(expect.values()) / total)) < 1e-7


def test_rowsum_decomposition_rescales_earlier_tiles_to_the_final_max():
    """Two tiles whose running max moved by 1 (log2): the first tile's values count half."""
    pt = np.zeros((2, 1, 64), np.float32)
    pt[0, 0, 0] = 1.0          # exact under its own scale
    pt[1, 0, 0] = 1.0
    pt[1, 0, 1] = 0.05         # zeroed (its group's step is 0.25)
    codes, scales = oracle.quantize(pt.reshape(2, 64), axis=0)
    m = np.array([[0.0], [1.0]])
    r = oracle.rowsum_decomposition(pt, codes.reshape(2, 1, 64), scales.reshape(2, 1, 2), m)
    total = 0.5 * 1.0 + 1.0 + 0.05
    assert abs(r["zeroing"][0] - (-0.05 / total)) < 1e-7
    assert r["saturation"][0] == 0 and r["up"][0] == 0 and r["down"][0] == 0
