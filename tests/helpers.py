"""Shared test plumbing: device tensors from the seeded inputs, oracle calls
on the same inputs, and the error metrics the parity tests use."""
from __future__ import annotations

import numpy as np

import oracle
from oracle import layout
from mxfp4_bit_attention_b200 import inputs

# Attention tolerance (outputs in units of V ~ N(0, 1)): relative L2 and max-abs.
REL_L2_TOL = 2e-3
MAX_ABS_TOL = 2e-2

RULE_NAMES = {0: "uos", 1: "qmax6", 2: "ocp", 3: "custom"}


def to_device(arr: np.ndarray, dtype: str, shape=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    if shape is not None:
        t = t.reshape(shape)
    return t.cuda()


def qkv_device(g, w):
    shape = (w.B, len(g["heads"]) // w.B if w.B == 1 else w.H, w.N, w.d)
    return [to_device(g[n], w.dtype, (1, len(g["heads"]), w.N, w.d)) for n in "qkv"]


def out_to_numpy(t) -> np.ndarray:
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def oracle_rows(g, w, rows, opts, softmax_scale=None, tau=None):
    """Oracle output (rounded to the output dtype) for the given query rows of every head."""
    s = softmax_scale if softmax_scale is not None else float(np.float32(w.d ** -0.5))
    q, k, v = (inputs.as_fp32(g[n], w.dtype) for n in "qkv")
    res = oracle.forward_rows(q, k, v, rows, s, rotate=opts.rotate, rule=opts.scale_rule, qmax=opts.qmax,
                              pnq=opts.pnq, key_tile=opts.key_tile,
                              tau=opts.rescale_tau if tau is None else tau)
    out = res["out"]
    if w.dtype == "bf16":
        return oracle.round_to_bf16(out), res
    return out.astype(np.float32).astype(np.float64), res
