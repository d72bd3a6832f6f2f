"""Packed batches of variable-length sequences (mxattn_forward_varlen): token-major [T, H, d] inputs,
device cu_seqlens.  Every sequence is an attention problem of its own, so the oracle runs each one
alone (oracle.forward_varlen) and the comparison is element by element at the plain bound:
rel-L2 <= 2e-3 over the batch and max-abs <= 2e-2 per element, in units of V ~ N(0, 1), short
sequences (rows of a few keys, where one flipped P^ code would be visible) included.  Each case
prints a DIAG line with its largest deviation (run with -s).
Bit-exact checks tie the packing to the fixed-length kernels: every sequence equals mxattn_forward
run on it alone, a single sequence equals mxattn_forward on [1, H, N, d], and equal-length
sequences equal mxattn_forward with B = nseq."""
import json

import numpy as np
import pytest

import oracle
from mxfp4_bit_attention_b200 import binding, inputs
from helpers import MAX_ABS_TOL, REL_L2_TOL, out_to_numpy, rel_l2

pytestmark = pytest.mark.gpu


def _draw(T, H, d, dtype, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, d), dtype=np.float32)
    k = rng.standard_normal((T, H, d), dtype=np.float32) * np.float32(1.5)
    v = rng.standard_normal((T, H, d), dtype=np.float32)
    if dtype == "bf16":
        q, k, v = (inputs.bf16_bits_to_fp32(inputs.fp32_to_bf16_bits(x)) for x in (q, k, v))
    return q, k, v


def _dev(x, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _cu(lengths):
    import torch
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return cu, torch.from_numpy(cu).cuda()


def _check(got, ref, case):
    assert np.isfinite(got).all()
    e = rel_l2(got, ref)
    dev = np.abs(got - ref)
    print("DIAG " + json.dumps({"diag": "varlen_parity", "case": case, "rel_l2": e, "max_abs": float(dev.max()),
                                "elements_over_2e-2": int((dev > MAX_ABS_TOL).sum())}))
    assert e <= REL_L2_TOL and float(dev.max()) <= MAX_ABS_TOL, f"rel_l2={e:.3e} max_abs={float(dev.max()):.3e}"


@pytest.mark.parametrize("lengths,H,d,dtype", [
    ([1], 1, 64, "fp32"),                        # one token
    ([5, 0, 70, 1, 130], 2, 128, "bf16"),        # an empty sequence, ragged tails, one past a tile
    ([128, 128, 64], 3, 64, "fp32"),             # whole tiles and a half tile
    ([1000, 37, 300], 2, 128, "bf16"),           # several tiles per sequence
    ([0, 0, 257], 1, 128, "bf16"),               # leading empty sequences
])
@pytest.mark.parametrize("pnq", [True, False])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("kt", [64, 128])
def test_varlen_matches_the_oracle(lengths, H, d, dtype, pnq, causal, kt):
    import torch
    cu, cu_dev = _cu(lengths)
    T = int(cu[-1])
    q, k, v = _draw(T, H, d, dtype, seed=700 + T + d)
    scale = float(np.float32(d ** -0.5))
    opts = binding.Opts(pnq=pnq, causal=causal, key_tile=kt)
    ws = torch.zeros(binding.load().mxattn_workspace_bytes_varlen(
        len(lengths), H, T, d, binding.ctypes.byref(binding._copts(opts, binding._dtype_code(_dev(q[:1], dtype))))),
        dtype=torch.uint8, device="cuda")
    out = binding.mxattn_forward_varlen(_dev(q, dtype), _dev(k, dtype), _dev(v, dtype), cu_dev, scale, opts,
                                        workspace=ws)
    torch.cuda.synchronize()
    assert binding.mxattn_get_device_error(ws) == 0
    ref = oracle.forward_varlen(q, k, v, cu, np.arange(T), scale, pnq=pnq, tau=8.0, causal=causal, key_tile=kt)
    ref = oracle.round_to_bf16(ref) if dtype == "bf16" else ref.astype(np.float32).astype(np.float64)
    _check(out_to_numpy(out), ref, f"lengths={lengths} H={H} d={d} {dtype} pnq={pnq} causal={causal} kt={kt}")

    # each sequence on its own through the fixed-length pass: the same bits
    got = out.view(torch.int16 if dtype == "bf16" else torch.int32)
    for s, n in enumerate(lengths):
        if n == 0:
            continue
        lo = int(cu[s])
        one = [x[lo:lo + n].transpose(0, 1).contiguous()[None] for x in (_dev(q, dtype), _dev(k, dtype), _dev(v, dtype))]
        b = binding.mxattn_forward(*one, scale, opts)[0].transpose(0, 1).contiguous()
        torch.cuda.synchronize()
        assert torch.equal(got[lo:lo + n], b.view(got.dtype)), f"sequence {s} (length {n})"


@pytest.mark.parametrize("causal", [False, True])
def test_single_sequence_equals_the_fixed_length_pass(causal):
    import torch
    T, H, d = 1000, 4, 128
    q, k, v = (_dev(x, "bf16") for x in _draw(T, H, d, "bf16", seed=5))
    _, cu_dev = _cu([T])
    opts = binding.Opts(causal=causal)
    a = binding.mxattn_forward_varlen(q, k, v, cu_dev, 0.088, opts)
    b = binding.mxattn_forward(*(x.transpose(0, 1).contiguous()[None] for x in (q, k, v)), 0.088, opts)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b[0].transpose(0, 1).contiguous().view(torch.int16))


def test_equal_lengths_equal_the_batched_pass():
    import torch
    nseq, N, H, d = 3, 777, 2, 64
    q, k, v = (_dev(x, "bf16") for x in _draw(nseq * N, H, d, "bf16", seed=6))
    _, cu_dev = _cu([N] * nseq)
    a = binding.mxattn_forward_varlen(q, k, v, cu_dev, 0.125)
    bhnd = [x.view(nseq, N, H, d).transpose(1, 2).contiguous() for x in (q, k, v)]
    b = binding.mxattn_forward(*bhnd, 0.125)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.transpose(1, 2).reshape(nseq * N, H, d).contiguous().view(torch.int16))


def test_video_mix_sampled_rows():
    """Three clips of different durations at 480p/720p-like token counts, 4 heads, sampled rows of
    each sequence (first rows, tile edges, ragged tails) against the oracle."""
    import torch
    lengths = [32760, 4097, 20000]
    cu, cu_dev = _cu(lengths)
    T, H, d = int(cu[-1]), 4, 128
    q, k, v = _draw(T, H, d, "bf16", seed=9)
    out = binding.mxattn_forward_varlen(_dev(q, "bf16"), _dev(k, "bf16"), _dev(v, "bf16"), cu_dev, 0.088)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([cu[s] + inputs.sample_rows(n, 8) for s, n in enumerate(lengths)]))
    ref = oracle.round_to_bf16(oracle.forward_varlen(q, k, v, cu, rows, 0.088, tau=8.0, key_tile=128))
    _check(out_to_numpy(out)[rows], ref, "video mix sampled rows")


@pytest.mark.parametrize("table", [[0, 50, 40, 100], [0, 50, 100, 120], [3, 50, 80, 100]])
def test_invalid_offsets_write_nothing_and_report(table):
    """A cu_seqlens table that decreases, overshoots T or does not start at 0 is caught on the
    device: the tile table is all zero, no later kernel writes, and the status reads as
    MXATTN_ERR_INVALID_ARG."""
    import torch
    T, H, d = 100, 2, 64
    q, k, v = (_dev(x, "fp32") for x in _draw(T, H, d, "fp32", seed=1))
    cu_dev = torch.tensor(table, dtype=torch.int32, device="cuda")
    opts = binding.Opts()
    ws = torch.zeros(binding.load().mxattn_workspace_bytes_varlen(
        3, H, T, d, binding.ctypes.byref(binding._copts(opts, binding.FP32))), dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, 7.0)
    binding.mxattn_forward_varlen(q, k, v, cu_dev, 0.125, opts, out=out, workspace=ws)
    assert binding.mxattn_get_device_error(ws) == 1
    assert bool((out == 7.0).all())
