"""GPU quantizers vs the oracle: codes and scales bit-exact, padding zero.

Covers the Q/K rotate+quantize kernel and the V (along keys) kernel in the
packed operand layouts, the plain generic quantizer, every scale rule, both
head dims, both input dtypes, ragged N and the full-size workloads (every head
and token)."""
import numpy as np
import pytest

import oracle
from oracle import layout
from mxfp4_bit_attention_b200 import binding, inputs
from helpers import to_device

pytestmark = pytest.mark.gpu

RULES = [(binding.SCALE_UOS, 7.25), (binding.SCALE_QMAX6, 6.0), (binding.SCALE_OCP, 7.25),
         (binding.SCALE_CEIL_CUSTOM, 7.0)]


def _mini(N, d, dtype, seed, H=2, name="mini"):
    return inputs.Workload(name, 1, H, N, d, dtype, seed)


def _check_qk(g, w, opts):
    q, k, v = (to_device(g[n], w.dtype, (1, len(g["heads"]), w.N, w.d)) for n in "qkv")
    ops = binding.mxattn_hadamard_quant_qk(q, k, opts)
    ops = binding.mxattn_quant_v(v, opts, out=ops)
    import torch
    torch.cuda.synchronize()
    BH = len(g["heads"])
    for name in "qk":
        codes, scales = layout.read_qk_operand(ops[f"{name}_codes"].cpu().numpy(), ops[f"{name}_scales"].cpu().numpy(),
                                               BH, w.N, w.d)
        x = inputs.as_fp32(g[name], w.dtype).reshape(-1, w.d)
        rc, rs = oracle.rotate_quantize_rows(x, opts.rotate, opts.scale_rule, opts.qmax)
        assert np.array_equal(scales.reshape(rs.shape), rs), f"{name} scales"
        mism = np.argwhere(codes.reshape(rc.shape) != rc)
        assert mism.size == 0, f"{name} codes differ at {mism[:5]} gpu={codes.reshape(rc.shape)[tuple(mism[0])]} ref={rc[tuple(mism[0])]}"
        pc, ps = layout.read_qk_padding(ops[f"{name}_codes"].cpu().numpy(), ops[f"{name}_scales"].cpu().numpy(),
                                        BH, w.N, w.d)
        assert not pc.any() and not ps.any(), f"{name} padding"
    vc, vs = layout.read_v_operand(ops["v_codes"].cpu().numpy(), ops["v_scales"].cpu().numpy(), BH, w.N, w.d)
    xv = inputs.as_fp32(g["v"], w.dtype)
    for h in range(BH):
        rc, rs = oracle.quantize(xv[h], axis=1, rule=opts.scale_rule, qmax=opts.qmax)   # [d, ceil(N/32)*32]
        ng = rs.shape[1]
        assert np.array_equal(vs[h][:, :ng], rs), f"v scales head {h}"
        assert not vs[h][:, ng:].any()
        assert np.array_equal(vc[h][:, :ng * 32], rc), f"v codes head {h}"
        assert not vc[h][:, ng * 32:].any()


@pytest.mark.parametrize("rule,qmax", RULES)
@pytest.mark.parametrize("rotate", [True, False])
def test_tiny_all_rules(rule, qmax, rotate):
    w = inputs.WORKLOADS["tiny"]
    g = inputs.generate(w)
    _check_qk(g, w, binding.Opts(scale_rule=rule, qmax=qmax, rotate=rotate))


@pytest.mark.parametrize("N,d,dtype", [(1, 64, "fp32"), (33, 64, "bf16"), (97, 128, "bf16"), (200, 128, "fp32"),
                                       (255, 64, "bf16"), (4096 + 16, 128, "bf16")])
def test_ragged(N, d, dtype):
    w = _mini(N, d, dtype, seed=N)
    g = inputs.generate(w)
    _check_qk(g, w, binding.Opts())


@pytest.mark.parametrize("rule,qmax", RULES)
def test_outlier_workload(rule, qmax):
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w, heads=[0, 5])
    _check_qk(g, w, binding.Opts(scale_rule=rule, qmax=qmax))


def test_extreme_magnitudes():
    """Blocks near the fp32 range ends, zeros, -0.0, subnormals and exact boundaries."""
    w = _mini(256, 128, "fp32", seed=7, H=1)
    g = inputs.generate(w)
    x = g["q"][0]
    x[0] = 0.0
    x[1] = -0.0
    x[2, :] = 3.0e38 * np.sign(np.random.default_rng(0).standard_normal(128))
    x[3, :] = 1e-39
    x[4, :] = np.float32(7.25 * 2.0 ** -5)
    x[5, ::2] = -1e-45
    x[6, :] = np.float32(2.0 ** -126)
    g["k"][0][:] = x
    g["v"][0][:8] = x[:8]
    _check_qk(g, w, binding.Opts(rotate=False))


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("shape", [(70, 45), (128, 256), (1, 33), (300, 1)])
def test_plain_quantizer(axis, dtype, shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    x = (rng.standard_normal(shape) * np.exp(rng.standard_normal(shape[1]))).astype(np.float32)
    bits = inputs.fp32_to_bf16_bits(x) if dtype == "bf16" else x
    xt = to_device(bits, dtype)
    codes, scales = binding.mxattn_quantize_mxfp4(xt, axis)
    outer, inner = (shape[0], shape[1]) if axis == 0 else (shape[1], shape[0])
    c, s = layout.read_plain(codes.cpu().numpy(), scales.cpu().numpy(), outer, inner)
    rc, rs = oracle.quantize(inputs.as_fp32(bits, dtype), axis, oracle.RULE_UOS)
    assert np.array_equal(s, rs) and np.array_equal(c, rc)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["480p", "720p", "joint"])
def test_full_size_workloads_full_tensors(name):
    """Full-size quantization on the GPU (the launch configuration the bench times), compared bit
    for bit with the oracle on every head and every token of Q, K and V (codes and scales), and
    the padding of the last 128-token tile zero.  MXFP4 format: Pith review page, axioms ledger
    (32-element E2M1 groups sharing one E8M0 scale); UOS interval (3.625, 7.25]: Fig. 3 caption."""
    import torch
    w = inputs.WORKLOADS[name]
    g = inputs.generate(w)
    q, k, v = (to_device(g[n], w.dtype, (1, w.H, w.N, w.d)) for n in "qkv")
    opts = binding.Opts()
    ops = binding.mxattn_hadamard_quant_qk(q, k, opts)
    ops = binding.mxattn_quant_v(v, opts, out=ops)
    torch.cuda.synchronize()
    del q, k, v
    T = (w.N + 127) // 128
    for name_ in "qk":
        cod = ops[f"{name_}_codes"].cpu().numpy().reshape(w.BH, T, 128, w.d // 2)
        sca = ops[f"{name_}_scales"].cpu().numpy().reshape(w.BH, T, 512)
        for h in range(w.BH):
            c, s = layout.read_qk_operand(cod[h], sca[h], 1, w.N, w.d)
            rc, rs = oracle.rotate_quantize_rows(inputs.as_fp32(g[name_][h], w.dtype), True)
            assert np.array_equal(s[0], rs), (name_, h, "scales")
            assert np.array_equal(c[0], rc), (name_, h, "codes")
            pc, ps = layout.read_qk_padding(cod[h], sca[h], 1, w.N, w.d)
            assert not pc.any() and not ps.any(), (name_, h, "padding")
    vc, vs = layout.read_v_operand(ops["v_codes"].cpu().numpy(), ops["v_scales"].cpu().numpy(), w.BH, w.N, w.d)
    for h in range(w.BH):
        rc, rs = oracle.quantize(inputs.as_fp32(g["v"][h], w.dtype), axis=1)
        ng = rs.shape[1]
        assert np.array_equal(vs[h][:, :ng], rs) and np.array_equal(vc[h][:, :ng * 32], rc), ("v", h)
        assert not vs[h][:, ng:].any() and not vc[h][:, ng * 32:].any(), ("v", h, "padding")
