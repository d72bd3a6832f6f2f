"""Fused MXFP4 PNQ attention on the GPU vs the oracle on the same seeded inputs.

Tolerance (outputs in units of V ~ N(0, 1)): relative L2 <= 2e-3 and
max-abs <= 2e-2 over the compared rows.  The oracle uses the kernel's key
tile (64 or 128, opts.key_tile) and lazy-max threshold, so running maxima and
quantization points match; remaining differences come from exp2/accumulation
rounding flipping an occasional P~ code."""
import numpy as np
import pytest

from mxfp4_bit_attention_b200 import binding, inputs
from helpers import MAX_ABS_TOL, REL_L2_TOL, oracle_rows, out_to_numpy, rel_l2, to_device

pytestmark = pytest.mark.gpu


def run(g, w, opts, rows=None, scale=None):
    import torch
    BH = len(g["heads"])
    q, k, v = (to_device(g[n], w.dtype, (1, BH, w.N, w.d)) for n in "qkv")
    s = scale if scale is not None else float(np.float32(w.d ** -0.5))
    ws = binding.new_workspace(1, BH, w.N, w.d, opts)
    out = binding.mxattn_forward(q, k, v, s, opts, workspace=ws)
    torch.cuda.synchronize()
    assert binding.mxattn_get_device_error(ws) == 0
    got = out_to_numpy(out)[0]
    rows = np.arange(w.N) if rows is None else rows
    ref, _ = oracle_rows(g, w, rows, opts, s)
    return got[:, rows], ref


def check(got, ref, label=""):
    e = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref)))
    assert np.isfinite(got).all(), label
    assert e <= REL_L2_TOL and m <= MAX_ABS_TOL, f"{label}: rel_l2={e:.3e} max_abs={m:.3e}"
    return e, m


KEY_TILES = [64, 128]


@pytest.mark.parametrize("kt", KEY_TILES)
def test_tiny_full(kt):
    w = inputs.WORKLOADS["tiny"]
    g = inputs.generate(w)
    got, ref = run(g, w, binding.Opts(key_tile=kt))
    check(got, ref, f"tiny kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
@pytest.mark.parametrize("pnq", [True, False])
@pytest.mark.parametrize("rule", [binding.SCALE_UOS, binding.SCALE_QMAX6, binding.SCALE_OCP])
def test_tiny_modes(pnq, rule, kt):
    w = inputs.WORKLOADS["tiny"]
    g = inputs.generate(w)
    got, ref = run(g, w, binding.Opts(pnq=pnq, scale_rule=rule, key_tile=kt))
    check(got, ref, f"pnq={pnq} rule={rule} kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
@pytest.mark.parametrize("q", [7.0, 7.5])  # 7.0: the OAS rule of Appendix G (Eq. 96); 7.5: above UOS
@pytest.mark.parametrize("pnq", [True, False])
def test_tiny_custom_boundary(q, pnq, kt):
    w = inputs.WORKLOADS["tiny"]
    g = inputs.generate(w)
    got, ref = run(g, w, binding.Opts(scale_rule=binding.SCALE_CEIL_CUSTOM, qmax=q, pnq=pnq, key_tile=kt))
    check(got, ref, f"q={q} pnq={pnq} kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
@pytest.mark.parametrize("tau", [0.0, 8.0])
@pytest.mark.parametrize("rotate", [True, False])
def test_tiny_tau_rotate(tau, rotate, kt):
    w = inputs.WORKLOADS["tiny"]
    g = inputs.generate(w)
    got, ref = run(g, w, binding.Opts(rescale_tau=tau, rotate=rotate, key_tile=kt))
    check(got, ref, f"tau={tau} rotate={rotate} kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
@pytest.mark.parametrize("N,d,dtype", [(1, 64, "fp32"), (33, 128, "bf16"), (100, 64, "bf16"), (129, 128, "fp32"),
                                       (255, 128, "bf16"), (1000, 64, "bf16"), (1100, 128, "bf16")])
def test_ragged(N, d, dtype, kt):
    w = inputs.Workload("mini", 1, 3, N, d, dtype, 100 + N)
    g = inputs.generate(w)
    got, ref = run(g, w, binding.Opts(key_tile=kt))
    check(got, ref, f"N={N} d={d} {dtype} kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
@pytest.mark.parametrize("pnq", [True, False])
@pytest.mark.parametrize("rule", [binding.SCALE_UOS, binding.SCALE_OCP])
def test_outlier_workload(pnq, rule, kt):
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w)
    rows = inputs.sample_rows(w.N, 96)
    got, ref = run(g, w, binding.Opts(pnq=pnq, scale_rule=rule, key_tile=kt), rows)
    check(got, ref, f"outlier pnq={pnq} rule={rule} kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
def test_outlier_workload_full(kt):
    """The outlier workload compared in full: all 4096 query rows of all 8 heads (Pith review page,
    Fig. 4 / Proposition 1: PNQ with the UOS rule, the method's default)."""
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w)
    got, ref = run(g, w, binding.Opts(key_tile=kt))
    check(got, ref, f"outlier full kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
def test_output_rows_past_n_untouched(kt):
    import torch
    w = inputs.Workload("mini", 1, 2, 70, 128, "bf16", 5)
    g = inputs.generate(w)
    q, k, v = (to_device(g[n], w.dtype, (1, 2, w.N, w.d)) for n in "qkv")
    big = torch.full((1 * 2 * 70 * 128 + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[:2 * 70 * 128].view(1, 2, 70, 128)
    binding.mxattn_forward(q, k, v, 128 ** -0.5, binding.Opts(key_tile=kt), out=out)
    torch.cuda.synchronize()
    assert torch.all(big[2 * 70 * 128:] == 7.0)


@pytest.mark.slow
@pytest.mark.parametrize("kt", KEY_TILES)
@pytest.mark.parametrize("name", ["480p", "720p", "joint"])
def test_full_size_sampled(name, kt):
    """Full-size launch (the configuration the bench times); all heads x 16 sampled rows,
    including the first row and the ragged last query tile."""
    w = inputs.WORKLOADS[name]
    g = inputs.generate(w)
    rows = inputs.sample_rows(w.N, 16)
    got, ref = run(g, w, binding.Opts(key_tile=kt), rows)
    check(got, ref, f"{name} kt={kt}")


@pytest.mark.parametrize("kt", KEY_TILES)
@pytest.mark.parametrize("d,pnq", [(128, True), (128, False), (64, True)])
def test_repeat_calls_bit_identical(d, pnq, kt):
    """The pipeline hands the P~ buffers, scale-factor slots and the O~ accumulator between
    warps through barriers only: a missing hand-off shows up as output that changes from call
    to call on identical inputs, so repeated calls must agree bit for bit."""
    import torch
    w = inputs.Workload("repeat", 1, 8, 4000, d, "bf16", 11)
    g = inputs.generate(w)
    q, k, v = (to_device(g[n], w.dtype, (1, 8, w.N, w.d)) for n in "qkv")
    opts = binding.Opts(pnq=pnq, key_tile=kt)
    ws = binding.new_workspace(1, 8, w.N, w.d, opts)
    first = binding.mxattn_forward(q, k, v, float(np.float32(d ** -0.5)), opts, workspace=ws).clone()
    for _ in range(6):
        again = binding.mxattn_forward(q, k, v, float(np.float32(d ** -0.5)), opts, workspace=ws)
        torch.cuda.synchronize()
        assert binding.mxattn_get_device_error(ws) == 0
        assert torch.equal(again.view(torch.int16), first.view(torch.int16))
