"""ctypes binding of libmxattn.so (declared in include/mxattn.h).

Argument marshalling only: torch tensors become device pointers and sizes,
the stream is torch's current CUDA stream, and every step of the method runs
in the library's kernels.  There is no fallback: if the library cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))

SCALE_UOS, SCALE_QMAX6, SCALE_OCP, SCALE_CEIL_CUSTOM = 0, 1, 2, 3
BF16, FP32 = 0, 1
FMT_MXFP4, FMT_NVFP4 = 0, 1

STATUS = {0: "MXATTN_OK", 1: "MXATTN_ERR_INVALID_ARG", 2: "MXATTN_ERR_UNSUPPORTED",
          3: "MXATTN_ERR_WORKSPACE", 4: "MXATTN_ERR_CUDA", 5: "MXATTN_ERR_TIMEOUT"}

EXPORTS = (
    "mxattn_opts_default", "mxattn_workspace_bytes", "mxattn_qk_codes_bytes",
    "mxattn_qk_scales_bytes", "mxattn_v_codes_bytes", "mxattn_v_scales_bytes",
    "mxattn_workspace_init", "mxattn_quantize_mxfp4", "mxattn_hadamard_quant_qk",
    "mxattn_quant_v", "mxattn_attention_mxfp4", "mxattn_forward", "mxattn_get_device_error",
    "mxattn_status_string", "mxattn_fp4_mma_probe", "mxattn_attention_dump_bytes",
    "mxattn_attention_mxfp4_dump", "mxattn_forward_noalloc", "mxattn_qmax_sweep",
    "mxattn_workspace_bytes_cross", "mxattn_forward_cross", "mxattn_workspace_bytes_host",
    "mxattn_forward_host", "mxattn_workspace_bytes_varlen", "mxattn_forward_varlen", "mxattn_operand_bytes",
    "mxattn_arith_probe",
)


class MXAttnError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} failed: {STATUS.get(status, status)}")
        self.status = status


class COpts(ctypes.Structure):
    _fields_ = [("scale_rule", ctypes.c_int), ("qmax", ctypes.c_float), ("pnq", ctypes.c_int),
                ("rotate", ctypes.c_int), ("dtype", ctypes.c_int), ("key_tile", ctypes.c_int),
                ("rescale_tau", ctypes.c_float), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("wait_budget_cycles", ctypes.c_longlong),
                ("causal", ctypes.c_int), ("format", ctypes.c_int)]


@dataclass
class Opts:
    scale_rule: int = SCALE_UOS
    qmax: float = 7.25
    pnq: bool = True
    rotate: bool = True
    key_tile: int = 128  # 64 for the NVFP4 comparison format
    rescale_tau: float = 8.0
    wait_budget_cycles: int = 0  # 0: the library's default (about one second)
    causal: bool = False  # self-attention: query row i sees keys 0..i
    format: int = 0       # FMT_MXFP4 (the method) or FMT_NVFP4 (the comparison format)


def lib_path() -> str:
    return os.path.join(HERE, "libmxattn.so")


_lib = None


def load():
    """Load libmxattn.so once; raise if it is missing or lacks a symbol."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m mxfp4_bit_attention_b200.build`")
    L = ctypes.CDLL(path)
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    PO = ctypes.POINTER(COpts)
    sig = {
        "mxattn_opts_default": ([PO], None),
        "mxattn_workspace_bytes": ([i32, i32, i32, i32, PO], sz),
        "mxattn_qk_codes_bytes": ([i32, i32, i32, i32], sz),
        "mxattn_qk_scales_bytes": ([i32, i32, i32, i32], sz),
        "mxattn_v_codes_bytes": ([i32, i32, i32, i32], sz),
        "mxattn_v_scales_bytes": ([i32, i32, i32, i32], sz),
        "mxattn_workspace_init": ([PO, P], i32),
        "mxattn_quantize_mxfp4": ([P, i64, i64, i32, PO, P, P, P], i32),
        "mxattn_hadamard_quant_qk": ([P, P, i32, i32, i32, i32, PO, P, P, P, P, P], i32),
        "mxattn_quant_v": ([P, i32, i32, i32, i32, PO, P, P, P], i32),
        "mxattn_attention_mxfp4": ([P, P, P, P, P, P, i32, i32, i32, i32, f32, PO, P, P], i32),
        "mxattn_forward": ([P, P, P, i32, i32, i32, i32, f32, PO, P, P], i32),
        "mxattn_get_device_error": ([PO, P], i32),
        "mxattn_status_string": ([i32], ctypes.c_char_p),
        "mxattn_fp4_mma_probe": ([i32, i32, i32, P], i32),
        "mxattn_attention_dump_bytes": ([i32, i32], sz),
        "mxattn_attention_mxfp4_dump": ([P, P, P, P, P, P, i32, i32, i32, i32, f32, PO, P, i32, i32, P, P], i32),
        "mxattn_forward_noalloc": ([P, P, P, i32, i32, i32, i32, f32, PO, P, P], i32),
        "mxattn_qmax_sweep": ([P, i64, i64, i32, i32, P, i32, P, P, P], i32),
        "mxattn_workspace_bytes_cross": ([i32, i32, i32, i32, i32, PO], sz),
        "mxattn_forward_cross": ([P, P, P, i32, i32, i32, i32, i32, f32, PO, P, P], i32),
        "mxattn_workspace_bytes_host": ([i32, i32, i32, i32, PO], sz),
        "mxattn_forward_host": ([P, P, P, i32, i32, i32, i32, f32, PO, P, P], i32),
        "mxattn_workspace_bytes_varlen": ([i32, i32, i32, i32, PO], sz),
        "mxattn_forward_varlen": ([P, P, P, P, i32, i32, i32, i32, f32, PO, P, P], i32),
        "mxattn_operand_bytes": ([i32, i32, i32, i32, PO, P], i32),
        "mxattn_arith_probe": ([i32, P, i64, PO, P, P], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(call, status):
    if status != 0:
        raise MXAttnError(call, status)


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _copts(o: Opts | None, dtype: int, workspace=None) -> COpts:
    o = o or Opts()
    c = COpts()
    load().mxattn_opts_default(ctypes.byref(c))
    c.scale_rule, c.qmax, c.pnq, c.rotate = int(o.scale_rule), float(o.qmax), int(bool(o.pnq)), int(bool(o.rotate))
    c.dtype, c.key_tile, c.rescale_tau = dtype, int(o.key_tile), float(o.rescale_tau)
    c.wait_budget_cycles = int(o.wait_budget_cycles)
    c.causal = int(bool(o.causal))
    c.format = int(o.format)
    if workspace is not None:
        c.workspace = ctypes.c_void_p(workspace.data_ptr())
        c.workspace_bytes = workspace.numel() * workspace.element_size()
    return c


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def operand_sizes(B: int, H: int, N: int, d: int, fmt: int = FMT_MXFP4) -> dict:
    """Bytes of the packed operands for the element format (the library's mxattn_operand_bytes)."""
    c = _copts(Opts(format=fmt), BF16)
    sizes = (ctypes.c_size_t * 6)()
    _check("mxattn_operand_bytes", load().mxattn_operand_bytes(B, H, N, d, ctypes.byref(c), sizes))
    return dict(zip(("q_codes", "q_scales", "k_codes", "k_scales", "v_codes", "v_scales"), (int(x) for x in sizes)))


def mxattn_workspace_bytes(B: int, H: int, N: int, d: int, opts: Opts | None = None) -> int:
    c = _copts(opts, BF16)
    return int(load().mxattn_workspace_bytes(B, H, N, d, ctypes.byref(c)))


def new_workspace(B, H, N, d, opts=None, device="cuda"):
    """A zeroed workspace tensor (uint8) of the size mxattn_forward needs."""
    import torch
    return torch.zeros(mxattn_workspace_bytes(B, H, N, d, opts), dtype=torch.uint8, device=device)


def mxattn_quantize_mxfp4(x, group_axis=0, opts: Opts | None = None, codes=None, scales=None, stream=None):
    """Plain MXFP4 quantization of a 2-D bf16/fp32 tensor; returns (codes, scales) uint8."""
    import torch
    rows, cols = x.shape
    outer, inner = (rows, cols) if group_axis == 0 else (cols, rows)
    gs = 16 if (opts is not None and opts.format == FMT_NVFP4) else 32
    ng = (inner + gs - 1) // gs
    codes = codes if codes is not None else torch.empty((outer, ng * gs // 2), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else torch.empty((outer, ng), dtype=torch.uint8, device=x.device)
    c = _copts(opts, _dtype_code(x))
    _check("mxattn_quantize_mxfp4", load().mxattn_quantize_mxfp4(
        _ptr(x), rows, cols, group_axis, ctypes.byref(c), _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def _alloc_operands(B, H, N, d, device, fmt=FMT_MXFP4):
    import torch
    s = operand_sizes(B, H, N, d, fmt)
    return {k: torch.empty(v, dtype=torch.uint8, device=device) for k, v in s.items()}


def mxattn_hadamard_quant_qk(q, k, opts: Opts | None = None, out=None, stream=None):
    """Rotate + quantize Q and K ([B, H, N, d]) into the packed QK operand layout."""
    B, H, N, d = q.shape
    out = out or _alloc_operands(B, H, N, d, q.device, (opts or Opts()).format)
    c = _copts(opts, _dtype_code(q))
    _check("mxattn_hadamard_quant_qk", load().mxattn_hadamard_quant_qk(
        _ptr(q), _ptr(k), B, H, N, d, ctypes.byref(c), _ptr(out["q_codes"]), _ptr(out["q_scales"]),
        _ptr(out["k_codes"]), _ptr(out["k_scales"]), _stream(stream)))
    return out


def mxattn_quant_v(v, opts: Opts | None = None, out=None, stream=None):
    """Quantize V ([B, H, N, d]) along keys into the packed V operand layout."""
    B, H, N, d = v.shape
    out = out or _alloc_operands(B, H, N, d, v.device, (opts or Opts()).format)
    c = _copts(opts, _dtype_code(v))
    _check("mxattn_quant_v", load().mxattn_quant_v(
        _ptr(v), B, H, N, d, ctypes.byref(c), _ptr(out["v_codes"]), _ptr(out["v_scales"]), _stream(stream)))
    return out


def mxattn_attention_mxfp4(ops, B, H, N, d, softmax_scale, out, opts: Opts | None = None, workspace=None,
                           stream=None):
    """Fused MXFP4 attention on packed operands (dict from the two quantizers)."""
    import torch
    ws = workspace if workspace is not None else torch.zeros(256, dtype=torch.uint8, device=out.device)
    c = _copts(opts, _dtype_code(out), ws)
    _check("mxattn_attention_mxfp4", load().mxattn_attention_mxfp4(
        _ptr(ops["q_codes"]), _ptr(ops["q_scales"]), _ptr(ops["k_codes"]), _ptr(ops["k_scales"]),
        _ptr(ops["v_codes"]), _ptr(ops["v_scales"]), B, H, N, d, float(softmax_scale), ctypes.byref(c),
        _ptr(out), _stream(stream)))
    return out


def dump_layout(N: int, d: int, key_tile: int = 128) -> dict:
    """Byte offsets of the diagnostic dump for key tiles of key_tile keys (mirrors the header)."""
    KT = key_tile
    T = (N + KT - 1) // KT
    p_codes = 2 * 128 * KT * 4
    p_scales = p_codes + T * 128 * (KT // 2)
    o = (p_scales + T * 128 * (KT // 32) + 15) // 16 * 16
    l = o + 128 * d * 4
    m = l + 128 * 4
    p_tilde = m + 128 * 4
    m_tiles = p_tilde + T * 128 * KT * 4
    return {"s": 0, "p_codes": p_codes, "p_scales": p_scales, "o": o, "l": l, "m": m, "p_tilde": p_tilde,
            "m_tiles": m_tiles, "total": m_tiles + T * 128 * 4}


def mxattn_attention_mxfp4_dump(ops, B, H, N, d, softmax_scale, out, dump_bh=0, dump_qt=0, opts=None,
                                workspace=None, stream=None):
    """mxattn_attention_mxfp4 plus the diagnostic dump of one CTA; returns the dump as a dict
    of numpy arrays (S tiles, P codes unpacked one per byte, P scales, O accumulator, l, m)."""
    import numpy as np
    import torch
    ws = workspace if workspace is not None else torch.zeros(256, dtype=torch.uint8, device=out.device)
    nbytes = int(load().mxattn_attention_dump_bytes(N, d))
    dump = torch.zeros(nbytes, dtype=torch.uint8, device=out.device)
    c = _copts(opts, _dtype_code(out), ws)
    _check("mxattn_attention_mxfp4_dump", load().mxattn_attention_mxfp4_dump(
        _ptr(ops["q_codes"]), _ptr(ops["q_scales"]), _ptr(ops["k_codes"]), _ptr(ops["k_scales"]),
        _ptr(ops["v_codes"]), _ptr(ops["v_scales"]), B, H, N, d, float(softmax_scale), ctypes.byref(c),
        _ptr(out), dump_bh, dump_qt, _ptr(dump), _stream(stream)))
    torch.cuda.synchronize()
    raw = dump.cpu().numpy()
    KT = int((opts or Opts()).key_tile)
    L = dump_layout(N, d, KT)
    T = (N + KT - 1) // KT
    pc = raw[L["p_codes"]:L["p_scales"]].reshape(T, 128, KT // 2)
    codes = np.empty((T, 128, KT), np.uint8)
    codes[..., 0::2] = pc & 0x0F
    codes[..., 1::2] = pc >> 4
    return {"s": raw[:L["p_codes"]].view(np.float32).reshape(2, 128, KT),
            "p_codes": codes,
            "p_scales": raw[L["p_scales"]:L["p_scales"] + T * 128 * (KT // 32)].reshape(T, 128, KT // 32),
            "o": raw[L["o"]:L["l"]].view(np.float32).reshape(128, d),
            "l": raw[L["l"]:L["m"]].view(np.float32).copy(),
            "m": raw[L["m"]:L["m"] + 512].view(np.float32).copy(),
            "p_tilde": raw[L["p_tilde"]:L["m_tiles"]].view(np.float32).reshape(T, 128, KT),
            "m_tiles": raw[L["m_tiles"]:L["total"]].view(np.float32).reshape(T, 128).copy()}


def mxattn_forward(q, k, v, softmax_scale=None, opts: Opts | None = None, out=None, workspace=None, stream=None):
    """MXAttention forward: O = MXFP4-PNQ-attention(Q, K, V) for [B, H, N, d] tensors."""
    import torch
    B, H, N, d = q.shape
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    out = out if out is not None else torch.empty_like(q)
    ws = workspace if workspace is not None else new_workspace(B, H, N, d, opts, q.device)
    c = _copts(opts, _dtype_code(q), ws)
    _check("mxattn_forward", load().mxattn_forward(
        _ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(softmax_scale), ctypes.byref(c), _ptr(out),
        _stream(stream)))
    return out


def mxattn_forward_host(q, k, v, softmax_scale=None, opts: Opts | None = None, out=None, workspace=None,
                        stream=None):
    """The forward pass from host tensors q, k, v [B, H, N, d] (page-locked for the transfers to
    overlap the kernels) into the host tensor `out`; chunks of heads pipeline their copies with
    the computation.  Synchronize the stream before reading `out`."""
    import torch
    B, H, N, d = q.shape
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    out = out if out is not None else torch.empty_like(q).pin_memory()
    dev = torch.device("cuda", torch.cuda.current_device())
    if workspace is None:
        nbytes = load().mxattn_workspace_bytes_host(B, H, N, d, ctypes.byref(_copts(opts, _dtype_code(q))))
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    c = _copts(opts, _dtype_code(q), workspace)
    _check("mxattn_forward_host", load().mxattn_forward_host(
        _ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(softmax_scale), ctypes.byref(c), _ptr(out), _stream(stream)))
    return out


def mxattn_forward_cross(q, k, v, softmax_scale=None, opts: Opts | None = None, out=None, workspace=None,
                         stream=None):
    """Cross-attention: q [B, H, Nq, d] attends to k, v [B, H, Nk, d]; out [B, H, Nq, d]."""
    import torch
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    out = out if out is not None else torch.empty_like(q)
    if workspace is None:
        nbytes = load().mxattn_workspace_bytes_cross(B, H, Nq, Nk, d, ctypes.byref(_copts(opts, _dtype_code(q))))
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=q.device)
    c = _copts(opts, _dtype_code(q), workspace)
    _check("mxattn_forward_cross", load().mxattn_forward_cross(
        _ptr(q), _ptr(k), _ptr(v), B, H, Nq, Nk, d, float(softmax_scale), ctypes.byref(c), _ptr(out),
        _stream(stream)))
    return out


def mxattn_forward_varlen(q, k, v, cu_seqlens, softmax_scale=None, opts: Opts | None = None, out=None,
                          workspace=None, stream=None):
    """Packed batch of variable-length sequences: q, k, v, out token-major [T, H, d]; cu_seqlens an
    int32 device tensor [nseq + 1] (sequence s = tokens cu_seqlens[s] .. cu_seqlens[s+1]-1).  An
    invalid cu_seqlens is reported by mxattn_get_device_error (MXATTN_ERR_INVALID_ARG)."""
    import torch
    T, H, d = q.shape
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
        raise TypeError("cu_seqlens must be a contiguous 1-D int32 tensor")
    nseq = cu_seqlens.numel() - 1
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    out = out if out is not None else torch.empty_like(q)
    if workspace is None:
        nbytes = load().mxattn_workspace_bytes_varlen(nseq, H, T, d, ctypes.byref(_copts(opts, _dtype_code(q))))
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=q.device)
    c = _copts(opts, _dtype_code(q), workspace)
    _check("mxattn_forward_varlen", load().mxattn_forward_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, H, T, d, float(softmax_scale), ctypes.byref(c),
        _ptr(out), _stream(stream)))
    return out


def mxattn_forward_noalloc(q, k, v, softmax_scale=None, opts: Opts | None = None, out=None, stream=None):
    """mxattn_forward with the library's fixed internal scratch instead of a workspace: for
    callers that cannot allocate device memory.  Problems needing more than the fixed scratch
    raise MXAttnError(MXATTN_ERR_WORKSPACE); concurrent calls on one device race."""
    import torch
    B, H, N, d = q.shape
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    out = out if out is not None else torch.empty_like(q)
    c = _copts(opts, _dtype_code(q))
    _check("mxattn_forward_noalloc", load().mxattn_forward_noalloc(
        _ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(softmax_scale), ctypes.byref(c), _ptr(out),
        _stream(stream)))
    return out


def mxattn_qmax_sweep(x, qs, rotate: bool = False, counts=None, sse_sums=None, stream=None):
    """Per-block Qmax sweep of the rows of x ([rows, cols], bf16 or fp32, on the GPU) over the
    increasing boundaries qs (host values in [4, 8]): returns (counts, sse_sums), device tensors
    of len(qs) -- int64 storage of the unsigned counts of groups for which each q is optimal, and
    the fp64 summed squared errors.  Given tensors are accumulated into."""
    import numpy as np
    import torch
    rows, cols = x.shape
    q = np.ascontiguousarray(qs, dtype=np.float32)
    if counts is None:
        counts = torch.zeros(q.size, dtype=torch.int64, device=x.device)
    if sse_sums is None:
        sse_sums = torch.zeros(q.size, dtype=torch.float64, device=x.device)
    _check("mxattn_qmax_sweep", load().mxattn_qmax_sweep(
        _ptr(x), rows, cols, _dtype_code(x), int(bool(rotate)), q.ctypes.data_as(ctypes.c_void_p), q.size,
        _ptr(counts), _ptr(sse_sums), _stream(stream)))
    return counts, sse_sums


def mxattn_get_device_error(workspace, stream=None) -> int:
    """Synchronize, read and clear the workspace status block; returns the status code."""
    c = _copts(None, BF16, workspace)
    return int(load().mxattn_get_device_error(ctypes.byref(c), _stream(stream)))


def mxattn_fp4_mma_probe(ctas: int, iters: int, n: int, stream=None):
    _check("mxattn_fp4_mma_probe", load().mxattn_fp4_mma_probe(ctas, iters, n, _stream(stream)))


PROBE_EXP2_POLY, PROBE_EXP2_MUFU, PROBE_E2M1_STANDIN, PROBE_E2M1_MUFU, PROBE_SCALE_EXP_LOG2, PROBE_SCALE_EXP = range(6)


def mxattn_arith_probe(op: int, x, opts: Opts | None = None, stream=None):
    """Evaluate one of the kernels' arithmetic shortcuts on a device float32 tensor x (see the
    header's mxattn_arith_probe); returns a device tensor (float32, uint8 or int32 by op)."""
    import torch
    out_dtype = {PROBE_EXP2_POLY: torch.float32, PROBE_EXP2_MUFU: torch.float32, PROBE_E2M1_STANDIN: torch.uint8,
                 PROBE_E2M1_MUFU: torch.uint8}.get(op, torch.int32)
    x = x.contiguous()
    out = torch.empty(x.numel(), dtype=out_dtype, device=x.device)
    c = _copts(opts, BF16)
    _check("mxattn_arith_probe", load().mxattn_arith_probe(op, _ptr(x), x.numel(), ctypes.byref(c), _ptr(out),
                                                           _stream(stream)))
    return out
