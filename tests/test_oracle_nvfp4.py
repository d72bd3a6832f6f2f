"""Pins of the oracle's NVFP4 comparison format (blocks of 16 E2M1 codes with an FP8 E4M3 scale).

The pages compare MXAttention with NVFP4-based baselines without defining the format; the oracle
follows the public one (E4M3: 4 exponent bits with bias 7, 3 mantissa bits, subnormals, largest
finite 448).  The pins: published E4M3 landmarks, torch's own float8_e4m3fn rounding (a library
routine) for the scale encoder, a brute-force nearest-code search for the block quantizer, and
the attention identities that hold for any element format (row sums, quantization off, one key)."""
import numpy as np
import pytest

import oracle

NV = oracle.FMT_NVFP4
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e4m3_landmarks():
    """Largest finite 448, smallest normal 2^-6, smallest subnormal 2^-9, 1.0 at byte 0x38, NaN at
    0x7F, and 126 distinct positive finite values in increasing byte order."""
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x38) == 1.0
    assert np.isnan(oracle.e4m3_decode(0x7F))
    vals = np.array([oracle.e4m3_decode(b) for b in range(0x7F)])
    assert (np.diff(vals) > 0).all() and len(vals) == 127
    assert oracle.e4m3_decode(0x80 | 0x38) == -1.0


def test_e4m3_encode_matches_torch_float8():
    """Round to nearest, ties to even, as torch's float8_e4m3fn conversion does (in range)."""
    import torch
    rng = np.random.default_rng(3)
    grid = np.array([oracle.e4m3_decode(b) for b in range(0x7F)])
    mids = (grid[1:] + grid[:-1]) / 2                      # every tie
    x = np.concatenate([mids, np.exp(rng.uniform(np.log(1e-4), np.log(440.0), 3000)), [0.0, 2.0 ** -11]])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    np.testing.assert_array_equal(got, ref)
    assert oracle.e4m3_encode(1000.0) == 0x7E            # saturating
    assert oracle.e4m3_encode(-3.0) == 0x80 | oracle.e4m3_encode(3.0)


def _nearest_e2m1(y):
    """Brute force: nearest E2M1 magnitude (ties to the even-mantissa code), saturating at 6."""
    a = np.abs(y)
    d = np.abs(a[..., None] - E2M1)
    best = np.argmin(d, axis=-1)
    # ties: argmin takes the lower index; the even-mantissa code is the even index
    tie = np.isclose(np.take_along_axis(d, np.minimum(best + 1, 7)[..., None], -1)[..., 0],
                     np.take_along_axis(d, best[..., None], -1)[..., 0], rtol=0, atol=0) & (best < 7)
    best = np.where(tie & (best % 2 == 1), best + 1, best)
    best = np.where(a >= 6.0, 7, best)
    return np.where(np.signbit(y), 8, 0) + best


@pytest.mark.parametrize("axis", [0, 1])
def test_block_quantizer_brute_force(axis):
    rng = np.random.default_rng(4 + axis)
    x = (rng.standard_normal((37, 50)) * np.exp(rng.standard_normal((37, 1)) * 2)).astype(np.float32)
    x[3, :] = 0.0
    x[5, 7] = -0.0
    codes, scales = oracle.quantize(x, axis=axis, fmt=NV)
    xt = x if axis == 0 else x.T
    outer, inner = xt.shape
    nb = (inner + 15) // 16
    assert codes.shape == (outer, nb * 16) and scales.shape == (outer, nb)
    pad = np.zeros((outer, nb * 16), np.float32)
    pad[:, :inner] = xt
    blocks = pad.reshape(outer, nb, 16)
    amax = np.abs(blocks).max(axis=-1)
    # scale: the E4M3 value nearest to fl32(amax / 6), computed by torch
    import torch
    sref = torch.from_numpy((amax / np.float32(6)).astype(np.float32)).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(scales, sref.view(torch.uint8).numpy())
    s = sref.float().numpy()
    y = np.where(s[..., None] > 0, blocks / np.where(s > 0, s, 1)[..., None], 0).astype(np.float32)
    want = np.where(s[..., None] > 0, _nearest_e2m1(y), 0).reshape(outer, -1)
    np.testing.assert_array_equal(codes, want)
    # the block maximum lands on 6 up to the scale's rounding: a normal E4M3 value is within a
    # relative 2^-4 (half of its 3-bit mantissa step) of what it rounds
    nz = amax / 6 >= 2.0 ** -6
    ratio = amax[nz] / s[nz]
    assert (ratio >= 6 / (1 + 2 ** -4)).all() and (ratio <= 6 / (1 - 2 ** -4)).all()


def test_rotate_quantize_rows_agrees_with_the_generic_quantizer():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((9, 128)).astype(np.float32)
    c1, s1 = oracle.rotate_quantize_rows(x, rotate=True, fmt=NV)
    c2, s2 = oracle.quantize(oracle.rotate_rows(x), axis=0, fmt=NV)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)


@pytest.fixture(scope="module")
def head():
    rng = np.random.default_rng(7)
    N, d = 300, 64
    q = rng.standard_normal((N, d)).astype(np.float32)
    k = (rng.standard_normal((N, d)) * 1.5).astype(np.float32)
    v = rng.standard_normal((N, d)).astype(np.float32)
    return q, k, v


def test_nvfp4_pnq_weights_sum_to_one(head):
    q, k, v = head
    qd, kd, vd = oracle.prepare_head(q[:40], k, v, fmt=NV)
    r = oracle.attention_rows(qd, kd, vd, 0.125, tau=8.0, weights=True, fmt=NV)
    np.testing.assert_allclose(r["wsum"], 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["ocheck"], r["out"], rtol=0, atol=1e-12)


def test_nvfp4_quant_off_is_the_format_free_softmax(head):
    q, k, v = head
    a = oracle.forward_rows(q[None], k[None], v[None], np.arange(10), 0.125, quant=False, fmt=NV)["out"]
    b = oracle.forward_rows(q[None], k[None], v[None], np.arange(10), 0.125, quant=False)["out"]
    np.testing.assert_array_equal(a, b)


def test_nvfp4_single_key_row_is_the_quantized_value_row(head):
    """Causal row 0 sees one key: P~ = 1, times 2688 is 448 * 6, so the scale is 448, the code 6 and
    P^ = 6 * 448 / 2688 = 1 exactly; the output is V's NVFP4 value row 0."""
    q, k, v = head
    out = oracle.forward_rows(q[None], k[None], v[None], np.array([0]), 0.125, causal=True, fmt=NV)["out"][0, 0]
    vc, vs = oracle.quantize(v, axis=1, fmt=NV)
    np.testing.assert_array_equal(out, oracle.dequantize(vc, vs, NV)[:, 0])


def test_nvfp4_p_codes_rebuild_the_tile(head):
    """The recorded P codes and E4M3 bytes, dequantized and divided by 2688, give back l (PNQ)."""
    q, k, v = head
    qd, kd, vd = oracle.prepare_head(q[:8], k, v, fmt=NV)
    r = oracle.attention_rows(qd, kd, vd, 0.125, tau=0.0, codes=True, fmt=NV)
    vals = oracle.dequantize(r["p_codes"], r["p_scales"], NV) / 2688.0
    ntiles = (300 + 63) // 64
    assert r["p_scales"].shape == (8, ntiles * 4)
    # with tau = 0 every tile is rescaled to the final max only through alpha; the last tile alone
    # is in final units, so check the row sums of single-tile problems instead
    qd1, kd1, vd1 = oracle.prepare_head(q[:8], k[:64], v[:64], fmt=NV)
    r1 = oracle.attention_rows(qd1, kd1, vd1, 0.125, codes=True, fmt=NV)
    v1 = oracle.dequantize(r1["p_codes"], r1["p_scales"], NV) / 2688.0
    np.testing.assert_allclose(v1.sum(axis=1), r1["l"], rtol=1e-15, atol=0)
    assert np.isfinite(vals).all()
