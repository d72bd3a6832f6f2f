"""CPU oracle for MXAttention's MXFP4 forward attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does, and this package imports nothing from it.

``mxref.c`` holds the arithmetic (plain C, fp64 accumulation, fp32 where the
method rounds to fp32); this module compiles it with gcc, loads it through
ctypes and marshals numpy arrays.  ``uos_theory`` holds the data-free UOS
objective, ``layout`` reads the CUDA library's packed operand layouts back into
plain row-major arrays.

Sources: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
Quantization for MXFP4 Attention" -- Pith review page (axioms ledger; Figs. 1,
3, 4; Eq. (96)) and the 10100.com article (MXFP4 format, UOS, PNQ).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mxref.c")
LIB = os.path.join(HERE, "libmxref.so")

RULE_UOS, RULE_QMAX6, RULE_OCP, RULE_CUSTOM = 0, 1, 2, 3
FMT_MXFP4, FMT_NVFP4 = 0, 1   # 32-element groups with an E8M0 scale; 16-element blocks with an E4M3 scale
RULES = {"uos": RULE_UOS, "qmax6": RULE_QMAX6, "ocp": RULE_OCP, "custom": RULE_CUSTOM}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile mxref.c into libmxref.so next to it (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-std=gnu11", "-o", LIB, SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB


class AttnCfg(ctypes.Structure):
    _fields_ = [("key_tile", ctypes.c_int), ("pnq", ctypes.c_int), ("quant_p", ctypes.c_int),
                ("rule", ctypes.c_int), ("qmax", ctypes.c_double), ("tau", ctypes.c_double),
                ("qpos", ctypes.c_void_p), ("fmt", ctypes.c_int)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(LIB)
            P = ctypes.c_void_p
            i64, i32, f64, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
            L.mxref_e2m1_decode.argtypes = [i32]
            L.mxref_e2m1_decode.restype = f64
            L.mxref_e2m1_encode.argtypes = [f64]
            L.mxref_e2m1_encode.restype = i32
            L.mxref_scale_exponent.argtypes = [f64, i32, f64]
            L.mxref_scale_exponent.restype = i32
            L.mxref_quantize.argtypes = [P, i64, i64, i32, i32, f64, P, P]
            L.mxref_quantize.restype = None
            L.mxref_fwht_row.argtypes = [P, i32]
            L.mxref_fwht_row.restype = None
            L.mxref_rotate_rows.argtypes = [P, i64, i32]
            L.mxref_rotate_rows.restype = None
            L.mxref_rotate_quantize_rows.argtypes = [P, i64, i32, i32, i32, f64, P, P]
            L.mxref_rotate_quantize_rows.restype = None
            L.mxref_dequantize.argtypes = [P, P, i64, P]
            L.mxref_dequantize.restype = None
            L.mxref_attention_rows.argtypes = [P, i64, P, P, i32, i32, f32, ctypes.POINTER(AttnCfg),
                                               P, P, P, P, P, P, P]
            L.mxref_attention_rows.restype = None
            L.mxref_qmax_sweep.argtypes = [P, i64, i64, i32, P, i32, P, P]
            L.mxref_qmax_sweep.restype = None
            L.mxref_e4m3_decode.argtypes = [i32]
            L.mxref_e4m3_decode.restype = f64
            L.mxref_e4m3_encode.argtypes = [f64]
            L.mxref_e4m3_encode.restype = i32
            L.mxref_quantize_nvfp4.argtypes = [P, i64, i64, i32, P, P]
            L.mxref_quantize_nvfp4.restype = None
            L.mxref_dequantize_nvfp4.argtypes = [P, P, i64, P]
            L.mxref_dequantize_nvfp4.restype = None
            L.mxref_rotate_quantize_rows_nvfp4.argtypes = [P, i64, i32, i32, P, P]
            L.mxref_rotate_quantize_rows_nvfp4.restype = None
            L.mxref_num_threads.argtypes = []
            L.mxref_num_threads.restype = i32
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def num_threads() -> int:
    return int(lib().mxref_num_threads())


# ----------------------------------------------------------------------------------------------
# Element format and scale rule
# ----------------------------------------------------------------------------------------------

def e2m1_encode(v: float) -> int:
    return int(lib().mxref_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(lib().mxref_e2m1_decode(int(code)))


def scale_exponent(amax: float, rule: int = RULE_UOS, qmax: float = 7.25) -> int:
    return int(lib().mxref_scale_exponent(float(amax), int(rule), float(qmax)))


def e4m3_encode(v: float) -> int:
    """E4M3 byte nearest to v (ties to even, saturating at 448): the NVFP4 block scale."""
    return int(lib().mxref_e4m3_encode(float(v)))


def e4m3_decode(byte: int) -> float:
    return float(lib().mxref_e4m3_decode(int(byte)))


def block_size(fmt: int) -> int:
    return 16 if fmt == FMT_NVFP4 else 32


# ----------------------------------------------------------------------------------------------
# Quantization
# ----------------------------------------------------------------------------------------------

def quantize(x: np.ndarray, axis: int = 0, rule: int = RULE_UOS, qmax: float = 7.25, fmt: int = FMT_MXFP4):
    """MXFP4-quantize a 2-D fp32 matrix in groups of 32 along columns (axis 0)
    or along rows (axis 1, output transposed).  Returns (codes, scales) with
    codes unpacked, one 4-bit code per byte: [outer, ceil(inner/32)*32].
    fmt = FMT_NVFP4: blocks of 16 with E4M3 scale bytes (rule and qmax unused)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    outer, inner = (rows, cols) if axis == 0 else (cols, rows)
    bs = block_size(fmt)
    ng = (inner + bs - 1) // bs
    codes = np.zeros((outer, ng * bs), np.uint8)
    scales = np.zeros((outer, ng), np.uint8)
    if fmt == FMT_NVFP4:
        lib().mxref_quantize_nvfp4(_ptr(x), rows, cols, axis, _ptr(codes), _ptr(scales))
    else:
        lib().mxref_quantize(_ptr(x), rows, cols, axis, rule, qmax, _ptr(codes), _ptr(scales))
    return codes, scales


def rotate_rows(x: np.ndarray) -> np.ndarray:
    """Hadamard-rotate each row (fp32, normalized by fl32(1/sqrt(d)))."""
    y = np.array(x, dtype=np.float32, copy=True, order="C")
    rows, d = y.reshape(-1, y.shape[-1]).shape
    lib().mxref_rotate_rows(_ptr(y), rows, d)
    return y


def rotate_quantize_rows(x: np.ndarray, rotate: bool = True, rule: int = RULE_UOS, qmax: float = 7.25,
                         fmt: int = FMT_MXFP4):
    """Q/K operand: optional rotation then groups of 32 along d (NVFP4: blocks of 16).
    Returns unpacked codes [rows, d] and scales [rows, d/32] (NVFP4: [rows, d/16])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    d = x.shape[-1]
    x2 = x.reshape(-1, d)
    rows = x2.shape[0]
    codes = np.zeros((rows, d), np.uint8)
    scales = np.zeros((rows, d // block_size(fmt)), np.uint8)
    if fmt == FMT_NVFP4:
        lib().mxref_rotate_quantize_rows_nvfp4(_ptr(x2), rows, d, int(bool(rotate)), _ptr(codes), _ptr(scales))
    else:
        lib().mxref_rotate_quantize_rows(_ptr(x2), rows, d, int(bool(rotate)), rule, qmax, _ptr(codes),
                                         _ptr(scales))
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: int = FMT_MXFP4) -> np.ndarray:
    """Exact values of unpacked codes with one scale byte per 32 codes (NVFP4: per 16) (fp64)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    assert codes.size == scales.size * block_size(fmt)
    out = np.empty(codes.shape, np.float64)
    if fmt == FMT_NVFP4:
        lib().mxref_dequantize_nvfp4(_ptr(codes), _ptr(scales), scales.size, _ptr(out))
    else:
        lib().mxref_dequantize(_ptr(codes), _ptr(scales), scales.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------------------------

def attention_rows(qd, kd, vd, softmax_scale, key_tile=64, pnq=True, quant_p=True, rule=RULE_UOS,
                   qmax=7.25, tau=0.0, weights=False, codes=False, qpos=None, fmt=FMT_MXFP4):
    """Online-softmax attention with PNQ for query rows qd [n, d] against
    kd, vd [N, d] (fp64 values).  Returns dict(out, m, l[, wsum, ocheck]
    [, p_codes [n, ntiles*key_tile], p_scales [n, ntiles*key_tile/32]]).  qpos: causal masking,
    row i sees keys 0..qpos[i] (None: all keys).  fmt = FMT_NVFP4: P~ in NVFP4 blocks of 16
    (p_scales [n, ntiles*key_tile/16], E4M3 bytes)."""
    qd = np.ascontiguousarray(qd, dtype=np.float64)
    kd = np.ascontiguousarray(kd, dtype=np.float64)
    vd = np.ascontiguousarray(vd, dtype=np.float64)
    n, d = qd.shape
    N = kd.shape[0]
    assert kd.shape == (N, d) and vd.shape == (N, d) and key_tile % 32 == 0
    qp = None if qpos is None else np.ascontiguousarray(qpos, dtype=np.int64)
    cfg = AttnCfg(int(key_tile), int(bool(pnq)), int(bool(quant_p)), int(rule), float(qmax), float(tau),
                  None if qp is None else qp.ctypes.data, int(fmt))
    out = np.empty((n, d), np.float64)
    m = np.empty(n, np.float64)
    l = np.empty(n, np.float64)
    wsum = np.empty(n, np.float64) if weights else None
    ocheck = np.empty((n, d), np.float64) if weights else None
    ntiles = (N + key_tile - 1) // key_tile
    pc = np.zeros((n, ntiles * key_tile), np.uint8) if codes else None
    ps = np.zeros((n, ntiles * key_tile // block_size(fmt)), np.uint8) if codes else None
    lib().mxref_attention_rows(_ptr(qd), n, _ptr(kd), _ptr(vd), N, d, float(np.float32(softmax_scale)),
                               ctypes.byref(cfg), _ptr(out), _ptr(m), _ptr(l), _ptr(wsum), _ptr(ocheck),
                               _ptr(pc), _ptr(ps))
    res = {"out": out, "m": m, "l": l}
    if codes:
        res["p_codes"] = pc
        res["p_scales"] = ps
    if weights:
        res["wsum"] = wsum
        res["ocheck"] = ocheck
    return res


def prepare_head(q, k, v, rotate=True, rule=RULE_UOS, qmax=7.25, quant=True, fmt=FMT_MXFP4):
    """Rotate/quantize one head's Q [nq, d], K [N, d], V [N, d] (fp32) and
    return their exact dequantized values (fp64): Q, K groups along d, V
    groups of 32 consecutive keys per channel (NVFP4: blocks of 16)."""
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    if not quant:
        qr = rotate_rows(q) if rotate else q
        kr = rotate_rows(k) if rotate else k
        return qr.astype(np.float64), kr.astype(np.float64), v.astype(np.float64)
    qc, qs = rotate_quantize_rows(q, rotate, rule, qmax, fmt)
    kc, ks = rotate_quantize_rows(k, rotate, rule, qmax, fmt)
    vc, vs = quantize(v, axis=1, rule=rule, qmax=qmax, fmt=fmt)  # [d, ceil(N/bs)*bs]
    N = v.shape[0]
    vd = dequantize(vc, vs, fmt)[:, :N].T                           # [N, d]
    return dequantize(qc, qs, fmt), dequantize(kc, ks, fmt), np.ascontiguousarray(vd)


def forward_rows(q, k, v, rows, softmax_scale, rotate=True, rule=RULE_UOS, qmax=7.25, pnq=True,
                 key_tile=64, tau=0.0, quant=True, weights=False, causal=False, fmt=FMT_MXFP4):
    """MXAttention forward for selected query rows of every head.

    q, k, v: fp32 arrays [BH, N, d] (exact upcasts of the inputs).
    rows:    int array of query indices (same rows for every head).
    causal:  each row sees only the keys up to its own index (self-attention, top-left aligned).
    fmt:     FMT_MXFP4 (the method) or FMT_NVFP4 (the comparison format) for Q, K, V and P~.
    Returns dict with out [BH, len(rows), d] (fp64) and m, l [BH, len(rows)].
    """
    BH, N, d = q.shape
    rows = np.asarray(rows, dtype=np.int64)
    outs, ms, ls, ws, ocs = [], [], [], [], []
    for h in range(BH):
        qd, kd, vd = prepare_head(q[h][rows], k[h], v[h], rotate, rule, qmax, quant, fmt)
        r = attention_rows(qd, kd, vd, softmax_scale, key_tile, pnq, quant, rule, qmax, tau, weights,
                           qpos=rows if causal else None, fmt=fmt)
        outs.append(r["out"])
        ms.append(r["m"])
        ls.append(r["l"])
        if weights:
            ws.append(r["wsum"])
            ocs.append(r["ocheck"])
    res = {"out": np.stack(outs), "m": np.stack(ms), "l": np.stack(ls)}
    if weights:
        res["wsum"] = np.stack(ws)
        res["ocheck"] = np.stack(ocs)
    return res


def forward_varlen(q, k, v, cu_seqlens, rows, softmax_scale, causal=False, with_l=False, **kw):
    """Attention over a packed batch of variable-length sequences: sequence s holds tokens
    cu_seqlens[s] .. cu_seqlens[s+1]-1 and attends only to its own tokens, as an attention problem
    of its own (its V groups of 32 keys start at its first token).  This is the definition of a
    packed batch: each sequence is handed to forward_rows on its own.

    q, k, v: fp32 arrays [T, H, d] (token-major packing).  rows: global token indices.
    Keyword arguments go to forward_rows.  Returns out [len(rows), H, d] (fp64), and with with_l
    also the row sums l [len(rows), H] (in units of the row's running maximum).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    T, H, d = q.shape
    assert cu[0] == 0 and cu[-1] == T and (np.diff(cu) >= 0).all()
    out = np.zeros((len(rows), H, d))
    ls = np.zeros((len(rows), H))
    seq = np.searchsorted(cu, rows, side="right") - 1
    for s in np.unique(seq):
        lo, hi = int(cu[s]), int(cu[s + 1])
        sel = np.nonzero(seq == s)[0]
        per_head = lambda x: np.ascontiguousarray(x[lo:hi].transpose(1, 0, 2))
        res = forward_rows(per_head(q), per_head(k), per_head(v), rows[sel] - lo, softmax_scale,
                           causal=causal, **kw)
        out[sel] = res["out"].transpose(1, 0, 2)
        ls[sel] = res["l"].T
    return (out, ls) if with_l else out


# ----------------------------------------------------------------------------------------------
# Scale-rule diagnostic: per-block Qmax sweep
# ----------------------------------------------------------------------------------------------

def qmax_grid(lo: float = 6.0, hi: float = 8.0, step: float = 0.05) -> np.ndarray:
    """The swept boundaries as fp32 values: lo, lo + step, ..., hi (rounded to fp32 once)."""
    n = int(round((hi - lo) / step)) + 1
    return np.array([lo + k * step for k in range(n)], dtype=np.float32)


def qmax_sweep(x: np.ndarray, qs: np.ndarray, rotate: bool = False):
    """Per-block Qmax sweep of the rows of x [rows, cols] (groups of 32 along each row; rows
    Hadamard-rotated first when rotate).  Returns (counts [nq] uint64: groups for which each q is
    SSE-optimal, sse_sums [nq] fp64: summed squared error at each q)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    qs = np.ascontiguousarray(qs, dtype=np.float32)
    rows, cols = x.shape
    counts = np.zeros(qs.size, np.uint64)
    sums = np.zeros(qs.size, np.float64)
    lib().mxref_qmax_sweep(_ptr(x), rows, cols, int(bool(rotate)), _ptr(qs), qs.size, _ptr(counts), _ptr(sums))
    return counts, sums


def rowsum_decomposition(p_tilde, p_codes, p_scales, m_tiles):
    """Row-sum error of direct placement, split by what quantization did to each P~ value.

    p_tilde [T, rows, K]  unquantized exponential tiles (each relative to its tile's running max)
    p_codes [T, rows, K]  their E2M1 codes (one per byte), p_scales [T, rows, K/32] E8M0 bytes
    m_tiles [T, rows]     the running max of each tile, log2 units
    Every value is brought to the final running max (weight 2^(m_t - m_final)).  With direct
    placement the normalized weights of a row sum to sum(P^) / sum(P~) = 1 + sum of the four
    contributions below, each the summed (P^ - P~) of its class over sum(P~):
      zeroing       P~ > 0 quantized to 0
      saturation    P~ above 6 * 2^e, clipped to the largest code
      down          other values rounded down, up: values rounded up.
    Under PNQ the row sum is 1 by construction (Proposition 1).  Returns a dict of per-row arrays
    (zeroing, saturation, down, up, rowsum_direct)."""
    pt = np.asarray(p_tilde, dtype=np.float64)
    T, R, K = pt.shape
    sc = np.repeat(np.asarray(p_scales, dtype=np.int64), 32, axis=2)
    codes = np.asarray(p_codes, dtype=np.uint8)
    mag = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    ph = np.where(codes & 8, -1.0, 1.0) * mag[codes & 7] * np.ldexp(1.0, sc - 127)
    w = np.exp2(np.asarray(m_tiles, dtype=np.float64) - np.asarray(m_tiles, dtype=np.float64)[-1])[:, :, None]
    d = (ph - pt) * w
    top = np.ldexp(6.0, sc - 127)
    zero = (ph == 0) & (pt > 0)
    sat = ((codes & 7) == 7) & (pt > top)
    down = (ph < pt) & ~zero & ~sat
    up = ph > pt
    total = (pt * w).sum(axis=(0, 2))
    res = {name: (d * mask).sum(axis=(0, 2)) / total
           for name, mask in (("zeroing", zero), ("saturation", sat), ("down", down), ("up", up))}
    res["rowsum_direct"] = (ph * w).sum(axis=(0, 2)) / total
    return res


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to fp32 and then to bf16 (round to nearest, ties to
    even), returned as fp64 values; finite inputs only."""
    f = np.asarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)
