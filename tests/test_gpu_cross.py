"""Cross-attention (mxattn_forward_cross): queries and keys of different lengths, e.g. video tokens
attending to text tokens.  The oracle's attention takes any number of keys for its query rows, so
the comparison and the tolerance are those of self-attention (rel-L2 <= 2e-3, max-abs <= 2e-2 in
units of V ~ N(0, 1)).  Inputs are seeded draws of the stated shapes (bf16 by round to nearest
even where the case says bf16)."""
import numpy as np
import pytest

import oracle
from mxfp4_bit_attention_b200 import binding, inputs
from helpers import MAX_ABS_TOL, REL_L2_TOL, out_to_numpy, rel_l2

pytestmark = pytest.mark.gpu


def _draw(BH, Nq, Nk, d, dtype, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((BH, Nq, d), dtype=np.float32)
    k = rng.standard_normal((BH, Nk, d), dtype=np.float32) * np.float32(1.5)
    v = rng.standard_normal((BH, Nk, d), dtype=np.float32)
    if dtype == "bf16":
        q, k, v = (inputs.bf16_bits_to_fp32(inputs.fp32_to_bf16_bits(x)) for x in (q, k, v))
    return q, k, v


def _dev(x, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return (t.to(torch.bfloat16) if dtype == "bf16" else t)[None]  # exact: the values are bf16 already


@pytest.mark.parametrize("BH,Nq,Nk,d,dtype", [
    (2, 300, 1000, 128, "bf16"),   # more keys than queries, ragged key tile
    (2, 1000, 256, 128, "bf16"),   # a text-length key set
    (1, 129, 77, 64, "fp32"),      # both ragged, one key tile
    (1, 64, 4097, 128, "bf16"),    # one partial query tile, keys one past a tile
    (3, 200, 64, 64, "bf16"),      # exactly one key tile
])
@pytest.mark.parametrize("pnq", [True, False])
@pytest.mark.parametrize("kt", [64, 128])
def test_cross_attention_matches_the_oracle(BH, Nq, Nk, d, dtype, pnq, kt):
    import torch
    q, k, v = _draw(BH, Nq, Nk, d, dtype, seed=1000 + Nq + Nk + d)
    scale = float(np.float32(d ** -0.5))
    opts = binding.Opts(pnq=pnq, key_tile=kt)
    out = binding.mxattn_forward_cross(_dev(q, dtype), _dev(k, dtype), _dev(v, dtype), scale, opts)
    torch.cuda.synchronize()
    got = out_to_numpy(out)[0]
    ref = oracle.forward_rows(q, k, v, np.arange(Nq), scale, pnq=pnq, tau=8.0, key_tile=kt)["out"]
    ref = oracle.round_to_bf16(ref) if dtype == "bf16" else ref.astype(np.float32).astype(np.float64)
    assert np.isfinite(got).all()
    e, m = rel_l2(got, ref), float(np.max(np.abs(got - ref)))
    assert e <= REL_L2_TOL and m <= MAX_ABS_TOL, f"rel_l2={e:.3e} max_abs={m:.3e}"


def test_cross_with_equal_lengths_is_self_attention():
    import torch
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w, heads=[0, 1])
    q, k, v = (_dev(inputs.as_fp32(g[n], w.dtype), w.dtype) for n in "qkv")
    scale = float(np.float32(w.d ** -0.5))
    a = binding.mxattn_forward(q, k, v, scale)
    b = binding.mxattn_forward_cross(q, k, v, scale)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_video_to_text_cross_attention_sampled():
    """Video-DiT text cross-attention shape: 16,384 video queries x 512 text keys, 8 heads."""
    import torch
    BH, Nq, Nk, d = 8, 16384, 512, 128
    q, k, v = _draw(BH, Nq, Nk, d, "bf16", seed=77)
    scale = float(np.float32(d ** -0.5))
    out = binding.mxattn_forward_cross(_dev(q, "bf16"), _dev(k, "bf16"), _dev(v, "bf16"), scale)
    torch.cuda.synchronize()
    rows = inputs.sample_rows(Nq, 32)
    got = out_to_numpy(out)[0][:, rows]
    ref = oracle.round_to_bf16(oracle.forward_rows(q, k, v, rows, scale, tau=8.0, key_tile=128)["out"])
    assert rel_l2(got, ref) <= REL_L2_TOL and float(np.max(np.abs(got - ref))) <= MAX_ABS_TOL
