"""The attention kernels' arithmetic shortcuts, each held against its definition on the GPU
through mxattn_arith_probe:

* the 64-key kernel's FMA-pipe exp2 polynomial: relative error against 2^x (fp64) over the
  arguments it sees, [-64, 8], within the bound its comment states;
* the 128-key kernel's FMA-pipe stand-in for 2^u: the E2M1 code it yields equals the code of the
  exact 2^u (round to nearest even, saturating at 6) except within a few fp32 ulps of a grid
  midpoint;
* the softmax's shared exponent taken in the log2 domain: equal to the exact rule
  e = ceil(t - log2 q) (ceiling rules) or floor(t) - 2 (OCP floor rule) for a group maximum 2^t,
  away from a hair's breadth of each boundary, and exact at t = 0 (the group holding the running
  max).  Scale rules: Pith review page, Fig. 3 (UOS (3.625, 7.25], TFS (3, 6], OCP floor [4, 8)).
"""
import math

import numpy as np
import pytest

import oracle
from mxfp4_bit_attention_b200 import binding

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MIDPOINTS = (E2M1[1:] + E2M1[:-1]) / 2


def e2m1_code_exact(v: np.ndarray) -> np.ndarray:
    """E2M1 magnitude code of non-negative v: nearest grid value, ties to the even code (code
    parity = mantissa bit), saturating at 6."""
    v = np.asarray(v, dtype=np.float64)
    idx = np.searchsorted(MIDPOINTS, v, side="left")  # values above midpoint i go to i + 1
    code = idx.copy()
    tie = np.isin(v, MIDPOINTS)
    # at a tie, searchsorted(left) gives the lower code: take the even one of the two
    lower = idx[tie]
    code[tie] = np.where(lower % 2 == 0, lower, lower + 1)
    return np.minimum(code, 7)


def test_reference_encoder_matches_the_oracle():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(0, 8, 2000), MIDPOINTS, np.nextafter(MIDPOINTS, 0), np.nextafter(MIDPOINTS, 9)])
    ours = e2m1_code_exact(v)
    ref = np.array([oracle.e2m1_encode(x) for x in v])
    assert np.array_equal(ours, ref)


def _probe(op, x, opts=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    out = binding.mxattn_arith_probe(op, t, opts)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_exp2_polynomial_error_bound():
    x = np.concatenate([np.linspace(-64, 8, 2_000_001, dtype=np.float32),
                        np.float32(np.arange(-64, 9)) + np.float32(0.5),  # the reduction's tie points
                        np.float32(np.arange(-64, 9))])
    y = _probe(binding.PROBE_EXP2_POLY, x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y / exact - 1.0)
    print(f"DIAG exp2 polynomial: max relative error {rel.max():.3e} over [-64, 8]")
    assert rel.max() <= 2.5e-7


@pytest.mark.parametrize("op", [binding.PROBE_E2M1_STANDIN, binding.PROBE_E2M1_MUFU])
def test_e2m1_code_of_exp2(op):
    u = np.linspace(-8, 4, 6_000_001, dtype=np.float32)
    # every midpoint's log2 and its fp32 neighbours
    mids = np.log2(MIDPOINTS).astype(np.float32)
    near = np.concatenate([mids + k * np.spacing(mids) for k in range(-4, 5)]).astype(np.float32)
    u = np.concatenate([u, near, np.float32([-200.0, -1e30, -np.inf, 40.0])])
    got = _probe(op, u)
    exact = e2m1_code_exact(np.exp2(u.astype(np.float64)))
    bad = np.nonzero(got != exact)[0]
    # a disagreement is allowed only within 1e-6 (relative) of a midpoint
    v = np.exp2(u[bad].astype(np.float64))
    dist = np.min(np.abs(v[:, None] / MIDPOINTS[None, :] - 1.0), axis=1) if bad.size else np.zeros(0)
    print(f"DIAG e2m1 code of exp2, probe {op}: {bad.size} of {u.size} codes differ, all within "
          f"{dist.max() if bad.size else 0:.2e} of a midpoint")
    assert np.all(dist <= 1e-6)
    assert bad.size <= 1e-5 * u.size


@pytest.mark.parametrize("rule,qmax", [(binding.SCALE_UOS, 7.25), (binding.SCALE_QMAX6, 6.0),
                                       (binding.SCALE_OCP, 7.25), (binding.SCALE_CEIL_CUSTOM, 7.0)])
def test_shared_exponent_in_the_log2_domain(rule, qmax):
    opts = binding.Opts(scale_rule=rule, qmax=qmax)
    t = np.concatenate([np.linspace(-140, 140, 2_000_001, dtype=np.float32),
                        np.float32([0.0, -np.inf, 1e30, -1e30])])
    got = _probe(binding.PROBE_SCALE_EXP_LOG2, t, opts)
    t64 = t.astype(np.float64)
    if rule == binding.SCALE_OCP:
        exact = np.floor(t64) - 2
        frac = t64 - np.round(t64)
    else:
        lq = math.log2(qmax)
        exact = np.ceil(t64 - lq)
        frac = t64 - lq - np.round(t64 - lq)
    exact = np.clip(np.where(np.isfinite(exact), exact, -127), -127, 127)
    exact[np.isposinf(t64)] = 127
    # away from a boundary (a few fp32 ulps of t) the two agree exactly
    ulp = np.spacing(np.abs(t).astype(np.float32)).astype(np.float64)
    far = ~(np.abs(frac) <= 4 * ulp + 1e-7)
    assert np.array_equal(got[far], exact[far].astype(np.int64))
    # the group holding the running max (t = 0) takes its exponent from the exact rule
    assert got[-4] == oracle.scale_exponent(1.0, rule, qmax)
    assert got[-3] == -127 and got[-2] == 127 and got[-1] == -127


@pytest.mark.parametrize("rule,qmax", [(binding.SCALE_UOS, 7.25), (binding.SCALE_QMAX6, 6.0),
                                       (binding.SCALE_OCP, 7.25), (binding.SCALE_CEIL_CUSTOM, 7.5)])
def test_shared_exponent_integer_rule_matches_the_oracle(rule, qmax):
    """The quantizers' exact rule on boundary maxima q * 2^k and their fp32 neighbours, powers of
    two, zero and subnormals."""
    ks = np.arange(-140, 128)
    q32 = np.float32(qmax if rule != binding.SCALE_OCP else 4.0)
    b = np.array([np.ldexp(np.float64(q32), int(k)) for k in ks if -149 <= k + 2 <= 126], dtype=np.float32)
    b = b[b > 0]
    amax = np.concatenate([b, np.nextafter(b, np.float32(0)), np.nextafter(b, np.float32(np.inf)),
                           np.ldexp(np.float32(1), np.arange(-149, 127)).astype(np.float32), np.float32([0.0])])
    got = _probe(binding.PROBE_SCALE_EXP, amax, binding.Opts(scale_rule=rule, qmax=qmax))
    ref = np.array([oracle.scale_exponent(float(a), rule, qmax) for a in amax])
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("op", [binding.PROBE_E2M1_STANDIN, binding.PROBE_E2M1_MUFU])
def test_e2m1_code_of_exp2_exact_at_integers(op):
    """A score equal to the running max gives 2^(0 - e) = 2^-e exactly in the oracle (exp(0) = 1
    scaled by a power of two); at e = 2 that is the E2M1 midpoint 0.25, which rounds to the even
    code 0.  Both exponential paths must give the exact code at every integer argument."""
    u = np.arange(-12, 5, dtype=np.float32)
    got = _probe(op, u)
    assert np.array_equal(got, e2m1_code_exact(np.exp2(u.astype(np.float64))))
    assert got[u == -2][0] == 0 and got[u == -1][0] == 1
