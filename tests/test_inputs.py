"""The seeded input generator: deterministic, head-subset consistent, bf16 RNE."""
import numpy as np
import torch

from mxfp4_bit_attention_b200 import inputs


def test_tiny_shapes_and_determinism():
    a = inputs.generate("tiny")
    b = inputs.generate("tiny")
    for n in "qkv":
        assert a[n].shape == (1, 256, 64) and a[n].dtype == np.float32
        assert np.array_equal(a[n], b[n])
    assert not np.array_equal(a["q"], a["k"])


def test_head_subset_matches_full_draw():
    w = inputs.Workload("mini", 1, 4, 300, 128, "bf16", 9)
    full = inputs.generate(w)
    sub = inputs.generate(w, heads=[2, 3])
    for n in "qkv":
        assert np.array_equal(full[n][2:], sub[n])


def test_bf16_rounding_is_rne():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 1e3
    x[:4] = [1.00390625, 1.01171875, -1.00390625, 3.0e38]   # exact ties and a large value
    ours = inputs.fp32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(inputs.bf16_bits_to_fp32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_outlier_structure():
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w, heads=[0])
    k = inputs.as_fp32(g["k"], "bf16")[0]
    q = inputs.as_fp32(g["q"], "bf16")[0]
    big = np.sort(np.abs(k).mean(axis=0))[-4:]
    assert big.min() > 8 * np.median(np.abs(k).mean(axis=0))
    assert np.abs(q).mean() < 1.0


def test_sample_rows_cover_edges():
    r = inputs.sample_rows(75600, 64)
    assert r[0] == 0 and r[-1] == 75599 and (75599 // 128) * 128 in r and len(r) == 64
