"""The NVFP4 comparison format on the GPU (opts.format = FMT_NVFP4): 16-element blocks with E4M3
scales, against the oracle's NVFP4 functions.

1. Quantizers bit-exact: the plain quantizer (both axes, both dtypes, ragged shapes, zeros and
   extreme magnitudes), the rotated Q/K operands and the key-major V operand.  Both sides divide
   by the scale in fp32 with one rounding and round the quotient to E2M1 the same way.
2. The attention kernel (tcgen05 kind::mxf4nvf4, block16, UE4M3 scales) against the oracle's NVFP4
   attention: rel-L2 <= 2e-3 and max-abs <= 2e-2 (units of V ~ N(0, 1)), each case's largest
   deviation printed as a DIAG line.
3. Error against exact fp32 attention of NVFP4 beside MXFP4 (UOS) on the outlier workload: printed
   as DIAG lines (run with -s)."""
import json

import numpy as np
import pytest

import oracle
from oracle import layout
from mxfp4_bit_attention_b200 import binding, inputs
from helpers import MAX_ABS_TOL, REL_L2_TOL, out_to_numpy, rel_l2, to_device

pytestmark = pytest.mark.gpu

NV = binding.Opts(format=binding.FMT_NVFP4, key_tile=64)  # NVFP4 runs with 64-key tiles


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("shape", [(70, 45), (128, 256), (1, 17), (300, 1)])
def test_plain_quantizer(axis, dtype, shape):
    rng = np.random.default_rng(shape[0] * 5 + shape[1])
    x = (rng.standard_normal(shape) * np.exp(rng.standard_normal(shape[1]) * 2)).astype(np.float32)
    x.flat[::7] = 0.0
    x.flat[3::11] = -0.0
    if x.size > 40:
        x.flat[20] = 1e-7        # a block whose scale is subnormal or zero
        x.flat[21] = 5000.0      # a scale that saturates at 448
    bits = inputs.fp32_to_bf16_bits(x) if dtype == "bf16" else x
    codes, scales = binding.mxattn_quantize_mxfp4(to_device(bits, dtype), axis, NV)
    outer, inner = (shape[0], shape[1]) if axis == 0 else (shape[1], shape[0])
    c, s = layout.read_plain(codes.cpu().numpy(), scales.cpu().numpy(), outer, inner, group=16)
    rc, rs = oracle.quantize(inputs.as_fp32(bits, dtype), axis, fmt=oracle.FMT_NVFP4)
    assert np.array_equal(s, rs), "scales"
    assert np.array_equal(c, rc), f"codes differ at {np.argwhere(c != rc)[:5]}"


@pytest.mark.parametrize("N,d,dtype", [(1, 64, "fp32"), (97, 128, "bf16"), (200, 64, "bf16"), (1000, 128, "fp32")])
def test_operand_quantizers(N, d, dtype):
    import torch
    w = inputs.Workload("mini", 1, 2, N, d, dtype, N + d)
    g = inputs.generate(w)
    q, k, v = (to_device(g[n], w.dtype, (1, 2, N, d)) for n in "qkv")
    ops = binding.mxattn_quant_v(v, NV, out=binding.mxattn_hadamard_quant_qk(q, k, NV))
    torch.cuda.synchronize()
    for name in "qk":
        codes, scales = layout.read_qk_operand(ops[f"{name}_codes"].cpu().numpy(),
                                               ops[f"{name}_scales"].cpu().numpy(), 2, N, d, nvfp4=True)
        rc, rs = oracle.rotate_quantize_rows(inputs.as_fp32(g[name], dtype).reshape(-1, d), True,
                                             fmt=oracle.FMT_NVFP4)
        assert np.array_equal(scales.reshape(rs.shape), rs), f"{name} scales"
        assert np.array_equal(codes.reshape(rc.shape), rc), f"{name} codes"
    vc, vs = layout.read_v_operand(ops["v_codes"].cpu().numpy(), ops["v_scales"].cpu().numpy(), 2, N, d, nvfp4=True)
    xv = inputs.as_fp32(g["v"], dtype)
    for h in range(2):
        rc, rs = oracle.quantize(xv[h], axis=1, fmt=oracle.FMT_NVFP4)   # [d, ceil(N/16)*16]
        nb = rs.shape[1]
        assert np.array_equal(vs[h][:, :nb], rs), f"v scales head {h}"
        assert not vs[h][:, nb:].any()
        assert np.array_equal(vc[h][:, :nb * 16], rc), f"v codes head {h}"


def _draw(BH, N, d, dtype, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((BH, N, d), dtype=np.float32)
    k = rng.standard_normal((BH, N, d), dtype=np.float32) * np.float32(1.5)
    v = rng.standard_normal((BH, N, d), dtype=np.float32)
    if dtype == "bf16":
        q, k, v = (inputs.bf16_bits_to_fp32(inputs.fp32_to_bf16_bits(x)) for x in (q, k, v))
    return q, k, v


def _dev(x, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return (t.to(torch.bfloat16) if dtype == "bf16" else t)[None]


@pytest.mark.parametrize("BH,N,d,dtype", [(1, 256, 64, "fp32"), (2, 200, 128, "bf16"), (2, 1000, 128, "bf16"),
                                         (1, 4097, 64, "bf16")])
@pytest.mark.parametrize("pnq", [True, False])
@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_attention_matches_the_oracle(BH, N, d, dtype, pnq, tau):
    import torch
    q, k, v = _draw(BH, N, d, dtype, seed=900 + N + d)
    scale = float(np.float32(d ** -0.5))
    opts = binding.Opts(format=binding.FMT_NVFP4, pnq=pnq, rescale_tau=tau, key_tile=64)
    out = binding.mxattn_forward(_dev(q, dtype), _dev(k, dtype), _dev(v, dtype), scale, opts)
    torch.cuda.synchronize()
    got = out_to_numpy(out)[0]
    rows = np.arange(N) if N <= 1000 else inputs.sample_rows(N, 64)
    res = oracle.forward_rows(q, k, v, rows, scale, pnq=pnq, tau=tau, fmt=oracle.FMT_NVFP4)
    ref = oracle.round_to_bf16(res["out"]) if dtype == "bf16" else res["out"].astype(np.float32).astype(np.float64)
    got = got[:, rows]
    e = rel_l2(got, ref)
    dev = np.abs(got - ref)
    print("DIAG " + json.dumps({"diag": "nvfp4_parity", "BH": BH, "N": N, "d": d, "dtype": dtype, "pnq": pnq,
                                "tau": tau, "rel_l2": e, "max_abs": float(dev.max()),
                                "elements_over_2e-2": int((dev > MAX_ABS_TOL).sum())}))
    assert np.isfinite(got).all()
    assert e <= REL_L2_TOL and float(dev.max()) <= MAX_ABS_TOL, f"rel_l2={e:.3e} max_abs={float(dev.max()):.3e}"


def test_error_against_exact_attention_nvfp4_vs_mxfp4():
    import torch
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w)
    q, k, v = (to_device(g[n], w.dtype, (1, w.H, w.N, w.d)) for n in "qkv")
    scale = float(np.float32(w.d ** -0.5))
    torch.backends.cuda.matmul.allow_tf32 = False
    exact = torch.stack([torch.softmax((q[0, h].float() @ k[0, h].float().T) * scale, -1) @ v[0, h].float()
                         for h in range(w.H)])[None]
    table = {}
    for label, fmt in (("MXFP4 UOS", binding.FMT_MXFP4), ("NVFP4", binding.FMT_NVFP4)):
        for tau in (0.0, 8.0):
            for pnq in (True, False):
                opts = binding.Opts(format=fmt, pnq=pnq, rescale_tau=tau, key_tile=64)
                out = binding.mxattn_forward(q, k, v, scale, opts).float()
                err = (out - exact).double()
                rel = float(err.norm() / exact.double().norm())
                table[(label, tau, pnq)] = rel
                print("DIAG " + json.dumps({"diag": "error_vs_exact_fp32", "workload": "outlier", "format": label,
                                            "tau": tau, "pnq": pnq, "rel_l2": rel,
                                            "max_abs": float(err.abs().max())}))
    assert all(np.isfinite(list(table.values())))


def test_nvfp4_cross_and_host_paths():
    """The comparison format through cross-attention (keys of another length) against the oracle, and
    through the host-buffer call against the device call, bit for bit."""
    import torch
    q, _, _ = _draw(2, 300, 128, "bf16", seed=41)
    _, k, v = _draw(2, 1000, 128, "bf16", seed=42)
    scale = float(np.float32(128 ** -0.5))
    out = binding.mxattn_forward_cross(_dev(q, "bf16"), _dev(k, "bf16"), _dev(v, "bf16"), scale, NV)
    torch.cuda.synchronize()
    res = oracle.forward_rows(q, k, v, np.arange(300), scale, tau=8.0, fmt=oracle.FMT_NVFP4)
    ref = oracle.round_to_bf16(res["out"])
    got = out_to_numpy(out)[0]
    dev_abs = float(np.max(np.abs(got - ref)))
    print("DIAG " + json.dumps({"diag": "nvfp4_parity", "case": "cross 300 x 1000", "rel_l2": rel_l2(got, ref),
                                "max_abs": dev_abs}))
    assert rel_l2(got, ref) <= REL_L2_TOL and dev_abs <= MAX_ABS_TOL

    qs, ks, vs = (_dev(x, "bf16") for x in _draw(6, 1000, 128, "bf16", seed=43))
    dev = binding.mxattn_forward(qs, ks, vs, 0.088, NV)
    hq, hk, hv = (t.cpu().pin_memory() for t in (qs, ks, vs))
    host = torch.empty_like(hq).pin_memory()
    binding.mxattn_forward_host(hq, hk, hv, 0.088, NV, out=host)
    torch.cuda.synchronize()
    assert torch.equal(dev.cpu().view(torch.int16), host.view(torch.int16))


def test_nvfp4_rejects_masking():
    q, k, v = (_dev(x, "fp32") for x in _draw(1, 128, 64, "fp32", seed=2))
    with pytest.raises(binding.MXAttnError):
        binding.mxattn_forward(q, k, v, 0.125, binding.Opts(format=binding.FMT_NVFP4, causal=True, key_tile=64))
