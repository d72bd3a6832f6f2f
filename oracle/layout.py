"""Readers for the CUDA library's packed MXFP4 layouts -- TEST INFRASTRUCTURE.

Written from the layout description in the library's public header (the
packed QK / V attention-operand layouts and the plain layout of the generic
quantizer) so that tests can compare the library's bytes with the oracle's
unpacked codes and scales one element at a time.  Pure numpy index
arithmetic; no arithmetic of the method.
"""
from __future__ import annotations

import numpy as np


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Two codes per byte, element 2i in the low nibble -> one code per byte."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


def _atom_index(rows: np.ndarray, g: np.ndarray) -> np.ndarray:
    """Byte offset of (row within a 128-row tile, group 0..3) in a 512-byte scale atom."""
    return (rows % 32) * 16 + (rows // 32) * 4 + g


def read_qk_operand(codes: np.ndarray, scales: np.ndarray, BH: int, N: int, d: int, nvfp4: bool = False):
    """Packed QK operand -> (codes [BH, N, d] one per byte, scales [BH, N, d/32]); NVFP4: scales
    [BH, N, d/16] read from d/64 atoms per tile (block b in atom b // 4, slot b % 4)."""
    T = (N + 127) // 128
    c = np.asarray(codes, np.uint8).reshape(BH, T, 128, d // 32, 16)
    r = np.arange(128)
    if d == 128:
        s = (r >> 1) & 3
    elif d == 64:
        s = (r >> 2) & 1
    else:
        raise ValueError(d)
    chunk = np.arange(d // 32)[None, :] ^ s[:, None]          # [128, groups] stored position
    logical = c[:, :, r[:, None], chunk, :]                     # [BH, T, 128, groups, 16]
    logical = logical.reshape(BH, T * 128, d // 2)[:, :N]
    if nvfp4:
        sc = np.asarray(scales, np.uint8).reshape(BH, T, (d // 64) * 512)
        b = np.arange(d // 16)
        idx = (b // 4)[None, :] * 512 + _atom_index(r[:, None], (b % 4)[None, :])   # [128, blocks]
        sv = sc[:, :, idx].reshape(BH, T * 128, d // 16)[:, :N]
        return unpack_nibbles(logical), sv
    sc = np.asarray(scales, np.uint8).reshape(BH, T, 512)
    g = np.arange(d // 32)
    idx = _atom_index(r[:, None], g[None, :])                   # [128, groups]
    sv = sc[:, :, idx].reshape(BH, T * 128, d // 32)[:, :N]
    return unpack_nibbles(logical), sv


def read_qk_padding(codes: np.ndarray, scales: np.ndarray, BH: int, N: int, d: int):
    """Bytes the QK layout must hold as zero: rows past N and unused scale slots."""
    T = (N + 127) // 128
    c = np.asarray(codes, np.uint8).reshape(BH, T * 128, d // 2)[:, N:]
    sc = np.asarray(scales, np.uint8).reshape(BH, T, 512)
    r = np.arange(128)
    rows = (np.arange(T)[:, None] * 128 + r[None, :])
    mask = np.zeros((T, 512), bool)
    for g in range(4):
        idx = _atom_index(r, g)
        for t in range(T):
            mask[t, idx] = (rows[t] >= N) | (g >= d // 32)
    return c, sc[:, mask]


def read_v_operand(codes: np.ndarray, scales: np.ndarray, BH: int, N: int, d: int, nvfp4: bool = False):
    """Packed V operand -> (codes [BH, d, Npad] one per byte, keys along the
    last axis, Npad = 64*ceil(N/64); scales [BH, d, Npad/32]; NVFP4: [BH, d, Npad/16] from one
    atom per 64-key tile)."""
    T64 = (N + 63) // 64
    T128 = (N + 127) // 128
    c = np.asarray(codes, np.uint8).reshape(BH, T64, d, 2, 16)
    ch = np.arange(d)
    pos = np.arange(2)[None, :] ^ ((ch >> 2) & 1)[:, None]       # [d, 2]
    logical = c[:, :, ch[:, None], pos, :]                       # [BH, T64, d, 2, 16]
    logical = logical.transpose(0, 2, 1, 3, 4).reshape(BH, d, T64 * 32)
    if nvfp4:
        sc = np.asarray(scales, np.uint8).reshape(BH, T64, 512)
        b = np.arange(T64 * 4)
        idx = _atom_index(ch[:, None], (b % 4)[None, :])          # [d, blocks]
        return unpack_nibbles(logical), sc[:, (b // 4)[None, :], idx]
    sc = np.asarray(scales, np.uint8).reshape(BH, T128, 512)
    groups = T64 * 2
    gi = np.arange(groups)
    idx = _atom_index(ch[:, None], (gi % 4)[None, :])             # [d, groups]
    sv = sc[:, (gi // 4)[None, :], idx]                           # [BH, d, groups]
    return unpack_nibbles(logical), sv


def read_plain(codes: np.ndarray, scales: np.ndarray, outer: int, inner: int, group: int = 32):
    """Generic quantizer output -> (codes [outer, ng*group] one per byte, scales [outer, ng]);
    group 16 for NVFP4."""
    ng = (inner + group - 1) // group
    c = np.asarray(codes, np.uint8).reshape(outer, ng * group // 2)
    return unpack_nibbles(c), np.asarray(scales, np.uint8).reshape(outer, ng)
