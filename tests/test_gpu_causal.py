"""Causal self-attention (opts.causal = 1): query row i sees keys 0..i.

The oracle masks the scores of the keys after each row's own position; the kernel skips the key
tiles above its query tile's diagonal and masks, per row, the two tiles that cross it.  Both
quantize V over all N keys (its 32-key groups run across the diagonal), so the comparison is
element by element with the tolerance of full attention (rel-L2 <= 2e-3, max-abs <= 2e-2 in units of
V ~ N(0, 1)).  Sizes cover one row, a partial tile, exact tiles, a ragged tail past several tiles
and both head dimensions; large workloads are checked on sampled rows that include the first and
last rows of query tiles, where the diagonal tile holds one or 128 keys."""
import numpy as np
import pytest

import oracle
from mxfp4_bit_attention_b200 import binding, inputs
from helpers import MAX_ABS_TOL, REL_L2_TOL, out_to_numpy, rel_l2, to_device

pytestmark = pytest.mark.gpu


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
    return (t.to(torch.bfloat16) if dtype == "bf16" else t)[None]  # exact: the values are bf16 already


def _ref(q, k, v, rows, scale, dtype, pnq=True, tau=8.0, kt=128):
    ref = oracle.forward_rows(q, k, v, rows, scale, pnq=pnq, tau=tau, causal=True, key_tile=kt)["out"]
    return oracle.round_to_bf16(ref) if dtype == "bf16" else ref.astype(np.float32).astype(np.float64)


def _check(got, ref):
    assert np.isfinite(got).all()
    e, m = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    assert e <= REL_L2_TOL and m <= MAX_ABS_TOL, f"rel_l2={e:.3e} max_abs={m:.3e}"


@pytest.mark.parametrize("BH,N,d,dtype", [
    (1, 1, 64, "fp32"),       # one row, one key
    (2, 63, 128, "bf16"),     # inside one key tile
    (1, 128, 64, "fp32"),     # exactly one query tile, both key tiles on its diagonal
    (2, 129, 128, "bf16"),    # one row past a tile
    (2, 1000, 128, "bf16"),   # several tiles and a ragged tail
    (1, 777, 64, "bf16"),     # ragged, d = 64
])
@pytest.mark.parametrize("pnq", [True, False])
@pytest.mark.parametrize("kt", [64, 128])
def test_causal_matches_the_oracle(BH, N, d, dtype, pnq, kt):
    import torch
    q, k, v = _draw(BH, N, d, dtype, seed=500 + N + d)
    scale = float(np.float32(d ** -0.5))
    out = binding.mxattn_forward(_dev(q, dtype), _dev(k, dtype), _dev(v, dtype), scale,
                                 binding.Opts(pnq=pnq, causal=True, key_tile=kt))
    torch.cuda.synchronize()
    _check(out_to_numpy(out)[0], _ref(q, k, v, np.arange(N), scale, dtype, pnq=pnq, kt=kt))


def test_causal_first_row_is_the_quantized_first_value_row():
    """Row 0 sees key 0 alone: P~ = 1 is exact in E2M1 (4 x 2^-2), l = 1, so the output row is
    V^[0], V's MXFP4 value (its group of 32 keys quantized together along the key axis)."""
    import torch
    q, k, v = _draw(1, 300, 128, "fp32", seed=3)
    out = binding.mxattn_forward(_dev(q, "fp32"), _dev(k, "fp32"), _dev(v, "fp32"), 0.125,
                                 binding.Opts(causal=True))
    torch.cuda.synchronize()
    vhat = oracle.dequantize(*oracle.quantize(v[0], axis=1))  # [d, keys]: groups run along the keys
    np.testing.assert_array_equal(out_to_numpy(out)[0, 0, 0], vhat[:, 0])


@pytest.mark.parametrize("kt", [64, 128])
def test_causal_outlier_sampled_rows_and_repeat(kt):
    import torch
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w, heads=[0, 5])
    q, k, v = (to_device(g[n], w.dtype, (1, 2, w.N, w.d)) for n in "qkv")
    scale = float(np.float32(w.d ** -0.5))
    opts = binding.Opts(causal=True, key_tile=kt)
    out = binding.mxattn_forward(q, k, v, scale, opts)
    again = binding.mxattn_forward(q, k, v, scale, opts)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))
    rows = np.unique(np.concatenate([inputs.sample_rows(w.N, 24), [127, 128, 255, 256, 2047, 2048, 4095]]))
    qf, kf, vf = (inputs.as_fp32(g[n], w.dtype) for n in "qkv")
    _check(out_to_numpy(out)[0][:, rows], _ref(qf, kf, vf, rows, scale, "bf16", kt=kt))


def test_causal_720p_sampled_rows():
    """The 720p video shape (75,600 tokens, d = 128) under causal masking: two heads, sampled rows."""
    import torch
    w = inputs.WORKLOADS["720p"]
    g = inputs.generate(w, heads=[4, 31])
    q, k, v = (to_device(g[n], w.dtype, (1, 2, w.N, w.d)) for n in "qkv")
    scale = float(np.float32(w.d ** -0.5))
    out = binding.mxattn_forward(q, k, v, scale, binding.Opts(causal=True))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([inputs.sample_rows(w.N, 16), [75519, 75520, 75599]]))
    qf, kf, vf = (inputs.as_fp32(g[n], w.dtype) for n in "qkv")
    _check(out_to_numpy(out)[0][:, rows], _ref(qf, kf, vf, rows, scale, "bf16"))


def test_causal_host_path_matches_the_device_path():
    import torch
    q, k, v = _draw(6, 1000, 128, "bf16", seed=21)
    dq, dk, dv = (_dev(x, "bf16") for x in (q, k, v))
    opts = binding.Opts(causal=True)
    dev = binding.mxattn_forward(dq, dk, dv, 0.088, opts)
    hq, hk, hv = (t.cpu().pin_memory() for t in (dq, dk, dv))
    host = torch.empty_like(hq).pin_memory()
    binding.mxattn_forward_host(hq, hk, hv, 0.088, opts, out=host)
    torch.cuda.synchronize()
    assert torch.equal(dev.cpu().view(torch.int16), host.view(torch.int16))


def test_causal_cross_attention_is_rejected():
    q, k, v = _draw(1, 128, 64, "fp32", seed=1)
    with pytest.raises(binding.MXAttnError):
        binding.mxattn_forward_cross(_dev(q, "fp32"), _dev(k, "fp32"), _dev(v, "fp32"), 0.125,
                                     binding.Opts(causal=True))
