"""Pins of the oracle's element format, scale rules and rotation against what
the MXAttention pages fix (golden fixtures), closed forms and brute force."""
import math

import numpy as np
import pytest

import oracle
from conftest import golden


FMT = golden("e2m1_format.json")
RULES = golden("scale_rules.json")


def test_decode_table_matches_grid():
    mags = FMT["magnitude_by_code"]
    for code in range(16):
        want = mags[code & 7] * (-1 if code & 8 else 1)
        assert oracle.e2m1_decode(code) == want


@pytest.mark.parametrize("value,code", FMT["rounding_cases"]["cases"])
def test_encode_hand_cases(value, code):
    assert oracle.e2m1_encode(value) == code


def _nearest_brute(v):
    """Second, independent statement of round-to-nearest-even with saturation:
    pick among the 8 magnitudes by (distance, mantissa bit), magnitude >= 6 -> 6."""
    mags = FMT["magnitude_by_code"]
    a = abs(v)
    if a >= mags[-1]:
        idx = 7
    else:
        idx = min(range(8), key=lambda i: (abs(a - mags[i]), i & 1))
    return (8 if math.copysign(1.0, v) < 0 else 0) | idx


def test_encode_sweep_and_boundaries():
    vals = list(np.linspace(-8, 8, 4001))
    mags = FMT["magnitude_by_code"]
    mids = [0.5 * (a + b) for a, b in zip(mags[:-1], mags[1:])] + [7.0]
    for m in mids:
        f = np.float32(m)
        vals += [float(np.nextafter(f, np.float32(-np.inf))), float(f),
                 float(np.nextafter(f, np.float32(np.inf)))]
        vals += [-v for v in vals[-3:]]
    for v in vals:
        assert oracle.e2m1_encode(v) == _nearest_brute(v), v


def _q_of(rule, qmax=7.25):
    return {oracle.RULE_UOS: 7.25, oracle.RULE_QMAX6: 6.0, oracle.RULE_CUSTOM: qmax}[rule]


def _amax_samples(seed=0):
    rng = np.random.default_rng(seed)
    xs = [float(np.float32(2.0 ** rng.uniform(-130, 127))) for _ in range(400)]
    for q in (7.25, 6.0, 7.0, 4.0, 8.0):
        for k in range(-127, 126, 7):
            v = q * 2.0 ** k
            if not (1e-45 < v < 3.0e38):
                continue
            b = np.float32(v)
            xs += [float(b), float(np.nextafter(b, np.float32(0))), float(np.nextafter(b, np.float32(np.inf)))]
    return [x for x in xs if np.isfinite(x) and x > 0]


@pytest.mark.parametrize("rule", [oracle.RULE_UOS, oracle.RULE_QMAX6])
def test_ceiling_rule_exhaustive(rule):
    """Every E8M0 exponent is tried: the chosen one is the smallest that covers amax."""
    q = _q_of(rule)
    for amax in _amax_samples():
        e = oracle.scale_exponent(amax, rule)
        covering = [k for k in range(-127, 128) if amax <= math.ldexp(q, k)]
        want = min(covering) if covering else 127
        assert e == max(want, -127), (amax, e, want)


def test_custom_rule_exhaustive():
    for q in (7.0, 7.25, 6.5, 5.0):
        for amax in _amax_samples(1)[:300]:
            e = oracle.scale_exponent(amax, oracle.RULE_CUSTOM, q)
            covering = [k for k in range(-127, 128) if amax <= math.ldexp(q, k)]
            assert e == max(min(covering), -127)


def test_ocp_floor_rule():
    for amax in _amax_samples(2):
        e = oracle.scale_exponent(amax, oracle.RULE_OCP)
        fl = math.floor(math.log2(amax))
        # exact floor(log2) check without trusting log2 rounding
        while math.ldexp(1.0, fl) > amax:
            fl -= 1
        while math.ldexp(1.0, fl + 1) <= amax:
            fl += 1
        assert e == min(max(fl - 2, -127), 127)


@pytest.mark.parametrize("name,rule", [("uos", oracle.RULE_UOS), ("qmax6", oracle.RULE_QMAX6),
                                       ("ocp", oracle.RULE_OCP)])
def test_normalized_max_intervals(name, rule):
    """Fig. 3: the normalized block maximum lands in the rule's interval."""
    iv = RULES["normalized_max_interval"][name]
    for amax in _amax_samples(3):
        e = oracle.scale_exponent(amax, rule)
        if e in (-127, 127):
            continue  # clamped exponents are outside the interval argument
        x = math.ldexp(amax, -e)
        assert (x > iv["lo"]) if iv["lo_open"] else (x >= iv["lo"]), (name, amax, x)
        assert (x < iv["hi"]) if iv["hi_open"] else (x <= iv["hi"]), (name, amax, x)


def test_oas_special_case_eq96():
    """Eq. (96): the q = 7 ceiling rule lowers the TFS exponent by one exactly on (3, 3.5]."""
    rng = np.random.default_rng(4)
    lo, mid = RULES["oas_eq96"]["shift_minus_one_interval"]
    for _ in range(2000):
        e6 = int(rng.integers(-100, 100))
        x6 = float(rng.uniform(3.0, 6.0))
        if rng.random() < 0.1:
            x6 = float(rng.choice([3.5, 6.0, float(np.nextafter(3.5, 4)), float(np.nextafter(3.0, 4))]))
        amax = math.ldexp(x6, e6)
        assert oracle.scale_exponent(amax, oracle.RULE_QMAX6) == e6
        e7 = oracle.scale_exponent(amax, oracle.RULE_CUSTOM, 7.0)
        assert e7 == (e6 - 1 if lo < x6 <= mid else e6), x6


@pytest.mark.parametrize("name,rule", [("uos", oracle.RULE_UOS), ("qmax6", oracle.RULE_QMAX6),
                                       ("ocp", oracle.RULE_OCP)])
def test_group_example(name, rule):
    ex = RULES["group_example"]
    x = np.zeros((1, 32), np.float32)
    x[0, :len(ex["values"])] = ex["values"]
    codes, scales = oracle.quantize(x, 0, rule)
    assert scales[0, 0] == ex[name]["scale_byte"]
    assert list(codes[0, :len(ex["values"])]) == ex[name]["codes"]
    assert not codes[0, len(ex["values"]):].any()


@pytest.mark.parametrize("name,rule", [("uos", oracle.RULE_UOS), ("ocp", oracle.RULE_OCP)])
def test_overflow_example(name, rule):
    ex = RULES["overflow_example"]
    codes, scales = oracle.quantize(np.array([ex["values"]], np.float32), 0, rule)
    assert scales[0, 0] == ex[name]["scale_byte"]
    assert codes[0, 0] == ex[name]["codes"][0]


def test_zero_group_and_tail_padding():
    x = np.zeros((2, 40), np.float32)
    x[1, 33] = -1.0
    codes, scales = oracle.quantize(x, 0, oracle.RULE_UOS)
    assert scales.shape == (2, 2) and codes.shape == (2, 64)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and not codes[0].any()
    # group 1 of row 1: amax 1 -> e = -2 -> -1 * 4 = -4 -> code 8|6
    assert scales[1, 1] == 125 and codes[1, 33] == 14 and not codes[1, 40:].any()


def test_axis1_is_transpose_of_axis0():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((70, 45)).astype(np.float32)
    c0, s0 = oracle.quantize(np.ascontiguousarray(x.T), 0, oracle.RULE_UOS)
    c1, s1 = oracle.quantize(x, 1, oracle.RULE_UOS)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


def test_dequantize_roundtrip_on_grid():
    """Values already on a scaled grid quantize losslessly."""
    rng = np.random.default_rng(6)
    mags = np.array(FMT["magnitude_by_code"])
    for _ in range(50):
        e = int(rng.integers(-20, 20))
        idx = rng.integers(0, 8, 32)
        idx[0] = 7
        sign = rng.choice([-1.0, 1.0], 32)
        x = (sign * mags[idx] * 2.0 ** e).astype(np.float32)[None]
        c, s = oracle.quantize(x, 0, oracle.RULE_QMAX6)   # max 6 * 2^e maps to exactly 6
        assert np.array_equal(oracle.dequantize(c, s)[0], x[0].astype(np.float64))


@pytest.mark.parametrize("d", [64, 128])
def test_hadamard_matches_sylvester_matrix(d):
    """The rotation equals x @ H_d / sqrt(d) for scipy's Sylvester Hadamard matrix
    and is orthonormal (QK^T preserved)."""
    from scipy.linalg import hadamard
    eye = np.eye(d, dtype=np.float32)
    Hr = oracle.rotate_rows(eye).astype(np.float64)
    c = float(np.float32(1 / math.sqrt(d)))
    assert np.array_equal(Hr, hadamard(d).astype(np.float64) * c)
    assert np.allclose(Hr @ Hr.T, np.eye(d), atol=1e-6)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((33, d)).astype(np.float32)
    y = oracle.rotate_rows(x).astype(np.float64)
    ref = x.astype(np.float64) @ hadamard(d) / math.sqrt(d)
    assert np.allclose(y, ref, rtol=0, atol=1e-5)
    q = rng.standard_normal((17, d)).astype(np.float32)
    k = rng.standard_normal((19, d)).astype(np.float32)
    s0 = q.astype(np.float64) @ k.astype(np.float64).T
    s1 = oracle.rotate_rows(q).astype(np.float64) @ oracle.rotate_rows(k).astype(np.float64).T
    assert np.max(np.abs(s1 - s0)) <= 1e-5 * np.max(np.abs(s0))


def test_rotate_quantize_rows_equals_rotate_then_quantize():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((50, 128)).astype(np.float32)
    c1, s1 = oracle.rotate_quantize_rows(x, True, oracle.RULE_UOS)
    c2, s2 = oracle.quantize(oracle.rotate_rows(x), 0, oracle.RULE_UOS)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
