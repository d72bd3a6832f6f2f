"""Scale-rule diagnostics on the GPU.

1. The per-block Qmax sweep (mxattn_qmax_sweep, boundaries 6.00..8.00 step 0.05) against the
   oracle's on the same values: Hadamard-rotated Q and K, key-major V, the P~ tiles of one CTA
   (from the diagnostic dump) and a ragged fp32 matrix.  Counts of groups for which each boundary
   is optimal must agree exactly (both sides decide on the same fp64 error sums); the summed
   errors to 1e-12 relative (the GPU adds them atomically).
2. The row-sum error of direct placement, split into zeroing, saturation, down- and up-rounding,
   computed from the kernel's own dumped tiles; PNQ's row sum (the ones row of the PV MMA) must
   equal the sum of its quantized tiles.

Lines starting with "DIAG" carry the measured values (run with -s to see them)."""
import json

import numpy as np
import pytest

import oracle
from mxfp4_bit_attention_b200 import binding, inputs
from helpers import to_device

pytestmark = pytest.mark.gpu

QS = oracle.qmax_grid()
I725 = int(np.argmin(np.abs(QS - 7.25)))
I700 = int(np.argmin(np.abs(QS - 7.0)))
I750 = int(np.argmin(np.abs(QS - 7.5)))


def _sweep_both(x_dev, x_host, rotate, label):
    counts, sums = binding.mxattn_qmax_sweep(x_dev, QS, rotate=rotate)
    got_c = counts.cpu().numpy().astype(np.uint64)
    got_s = sums.cpu().numpy()
    ref_c, ref_s = oracle.qmax_sweep(x_host, QS, rotate=rotate)
    np.testing.assert_array_equal(got_c, ref_c, err_msg=label)
    np.testing.assert_allclose(got_s, ref_s, rtol=1e-12, err_msg=label)
    groups = x_host.shape[0] * ((x_host.shape[1] + 31) // 32)
    print("DIAG " + json.dumps({"diag": "qmax_sweep", "tensor": label, "groups": groups,
                                "mode_q": float(QS[int(np.argmax(got_c))]),
                                "fraction_optimal_at_7.00": float(got_c[I700]) / groups,
                                "fraction_optimal_at_7.25": float(got_c[I725]) / groups,
                                "fraction_optimal_at_7.50": float(got_c[I750]) / groups,
                                "fraction_optimal_at_6.00": float(got_c[0]) / groups,
                                "fraction_optimal_at_8.00": float(got_c[-1]) / groups,
                                "argmin_mean_sse_q": float(QS[int(np.argmin(got_s))])}))
    return got_c, got_s


@pytest.fixture(scope="module")
def outlier():
    w = inputs.WORKLOADS["outlier"]
    g = inputs.generate(w)
    return w, g


def test_sweep_rotated_q_and_k_match_the_oracle(outlier):
    w, g = outlier
    for name in "qk":
        dev = to_device(g[name], w.dtype, (w.H * w.N, w.d))
        host = inputs.as_fp32(g[name], w.dtype).reshape(w.H * w.N, w.d)
        _sweep_both(dev, host, True, f"outlier {name.upper()} (rotated)")


def test_sweep_key_major_v_matches_the_oracle(outlier):
    w, g = outlier
    v = to_device(g["v"], w.dtype, (w.H, w.N, w.d)).transpose(1, 2).contiguous().view(w.H * w.d, w.N)
    host = inputs.as_fp32(g["v"], w.dtype).transpose(0, 2, 1).reshape(w.H * w.d, w.N)
    _sweep_both(v, np.ascontiguousarray(host), False, "outlier V (key-major)")


def test_sweep_ragged_fp32_matches_the_oracle():
    import torch
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((37, 70)) * np.exp(rng.standard_normal((37, 1)) * 3)).astype(np.float32)
    _sweep_both(torch.from_numpy(x).cuda(), x, False, "ragged fp32 37x70")


def _dump(w, g, head, qtile, pnq=True):
    import torch
    q, k, v = (to_device(g[n], w.dtype, (1, w.H, w.N, w.d)) for n in "qkv")
    opts = binding.Opts(pnq=pnq, key_tile=64)  # the tile arithmetic below is written for 64-key tiles
    ops = binding.mxattn_quant_v(v, opts, out=binding.mxattn_hadamard_quant_qk(q, k, opts))
    out = torch.empty_like(q)
    return binding.mxattn_attention_mxfp4_dump(ops, 1, w.H, w.N, w.d, float(np.float32(w.d ** -0.5)), out,
                                               dump_bh=head, dump_qt=qtile, opts=opts)


def test_sweep_of_p_tiles_and_rowsum_decomposition(outlier):
    import torch
    w, g = outlier
    d = _dump(w, g, head=2, qtile=7)
    T64 = d["p_tilde"].shape[0]
    pt = np.ascontiguousarray(d["p_tilde"].reshape(T64 * 128, 64))
    _sweep_both(torch.from_numpy(pt).cuda(), pt, False, "outlier P~ tiles (head 2, query tile 7)")

    # the dumped P~, quantized by the oracle, gives the kernel's codes (up to exp2 rounding)
    codes, scales = oracle.quantize(pt, axis=0)
    kc = d["p_codes"].reshape(T64 * 128, 64)
    assert np.mean(codes != kc) < 1e-3
    assert np.mean(scales != d["p_scales"].reshape(T64 * 128, 2)) < 1e-3

    r = oracle.rowsum_decomposition(d["p_tilde"], d["p_codes"], d["p_scales"], d["m_tiles"])
    # PNQ: the kernel's row sum (ones row of the PV MMA, fp32) is the sum of its quantized tiles
    pnq_l = r["rowsum_direct"] * (np.asarray(d["p_tilde"], np.float64)
                                  * np.exp2(d["m_tiles"] - d["m_tiles"][-1])[:, :, None]).sum(axis=(0, 2))
    np.testing.assert_allclose(d["l"], pnq_l, rtol=2e-5)
    print("DIAG " + json.dumps({"diag": "rowsum_decomposition", "workload": "outlier", "rows": 128,
                                "mean_rowsum_direct": float(r["rowsum_direct"].mean()),
                                "mean_rowsum_pnq": 1.0,
                                **{f"mean_{k}": float(r[k].mean()) for k in ("zeroing", "saturation", "down", "up")}}))
    assert np.allclose(r["rowsum_direct"], 1 + r["zeroing"] + r["saturation"] + r["down"] + r["up"], atol=1e-12)


def test_sweep_720p_full_tensors_report():
    """The whole 720p Q, K (rotated) and V (key-major) on the GPU; the oracle checks two heads."""
    import torch
    w = inputs.WORKLOADS["720p"]
    g = inputs.generate(w)
    q, k, v = (to_device(g[n], w.dtype, (w.H, w.N, w.d)) for n in "qkv")
    for name, t, rot in (("Q", q, True), ("K", k, True)):
        counts, sums = binding.mxattn_qmax_sweep(t.view(w.H * w.N, w.d), QS, rotate=rot)
        c = counts.cpu().numpy().astype(np.uint64)
        groups = w.H * w.N * w.d // 32
        print("DIAG " + json.dumps({"diag": "qmax_sweep", "tensor": f"720p {name} (rotated, all heads)",
                                    "groups": groups, "mode_q": float(QS[int(np.argmax(c))]),
                                    "fraction_optimal_at_7.25": float(c[I725]) / groups,
                                    "fraction_optimal_at_6.00": float(c[0]) / groups,
                                    "argmin_mean_sse_q": float(QS[int(np.argmin(sums.cpu().numpy()))])}))
    vt = v.transpose(1, 2).contiguous().view(w.H * w.d, w.N)
    counts, sums = binding.mxattn_qmax_sweep(vt, QS)
    c = counts.cpu().numpy().astype(np.uint64)
    groups = w.H * w.d * ((w.N + 31) // 32)
    print("DIAG " + json.dumps({"diag": "qmax_sweep", "tensor": "720p V (key-major, all heads)", "groups": groups,
                                "mode_q": float(QS[int(np.argmax(c))]),
                                "fraction_optimal_at_7.25": float(c[I725]) / groups,
                                "fraction_optimal_at_6.00": float(c[0]) / groups,
                                "argmin_mean_sse_q": float(QS[int(np.argmin(sums.cpu().numpy()))])}))
    # parity on two heads of K
    host = inputs.as_fp32(g["k"], w.dtype)[:2].reshape(2 * w.N, w.d)
    _sweep_both(k[:2].reshape(2 * w.N, w.d), host, True, "720p K heads 0-1 (rotated)")
