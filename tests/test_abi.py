"""The C-ABI library loads without a GPU and exports every symbol the header declares."""
import ctypes
import os
import re

import pytest

from mxfp4_bit_attention_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "mxattn.h")).read()
    return sorted(set(re.findall(r"MXATTN_API\s+[\w\s\*]+?\b(mxattn_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    from mxfp4_bit_attention_b200 import build
    build.build()
    return binding.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.EXPORTS)


def test_host_only_calls(lib):
    o = binding.COpts()
    lib.mxattn_opts_default(ctypes.byref(o))
    assert (o.scale_rule, o.pnq, o.rotate, o.key_tile) == (0, 1, 1, 128)
    assert abs(o.qmax - 7.25) < 1e-7 and abs(o.rescale_tau - 8.0) < 1e-7
    assert o.wait_budget_cycles == 0  # the library's default budget
    assert o.causal == 0 and o.format == 0
    assert lib.mxattn_qk_codes_bytes(1, 2, 200, 128) == 2 * 2 * 128 * 64
    assert lib.mxattn_qk_scales_bytes(1, 2, 200, 128) == 2 * 2 * 512
    assert lib.mxattn_v_codes_bytes(1, 2, 200, 128) == 2 * 4 * 128 * 32
    assert lib.mxattn_v_scales_bytes(1, 2, 200, 64) == 2 * 2 * 512
    assert lib.mxattn_workspace_bytes(1, 1, 256, 96, ctypes.byref(o)) == 0
    assert lib.mxattn_workspace_bytes(1, 40, 75600, 128, ctypes.byref(o)) > 256
    assert lib.mxattn_workspace_bytes_cross(2, 3, 500, 500, 128, ctypes.byref(o)) == \
        lib.mxattn_workspace_bytes(2, 3, 500, 128, ctypes.byref(o))
    assert lib.mxattn_workspace_bytes_cross(1, 4, 75600, 512, 128, ctypes.byref(o)) < \
        lib.mxattn_workspace_bytes(1, 4, 75600, 128, ctypes.byref(o))
    assert lib.mxattn_workspace_bytes_cross(1, 4, 100, 0, 128, ctypes.byref(o)) == 0
    # staging for two chunks of 4 heads, far below the 2.3 GB of all 40 heads' bf16 inputs
    assert 0 < lib.mxattn_workspace_bytes_host(1, 40, 75600, 128, ctypes.byref(o)) < 3 * 40 * 75600 * 128 * 2 // 3
    assert lib.mxattn_workspace_bytes_host(1, 1, 0, 128, ctypes.byref(o)) == 0
    # varlen: (T + 127 nseq) / 128 tiles per head reserved; one sequence packs like B = 1
    one = lib.mxattn_workspace_bytes_varlen(1, 4, 1000, 128, ctypes.byref(o))
    assert one >= lib.mxattn_workspace_bytes(1, 4, 1000, 128, ctypes.byref(o))
    assert lib.mxattn_workspace_bytes_varlen(3, 4, 1000, 128, ctypes.byref(o)) > one
    assert lib.mxattn_workspace_bytes_varlen(0, 4, 1000, 128, ctypes.byref(o)) == 0
    assert lib.mxattn_workspace_bytes_varlen(2, 4, 1000, 96, ctypes.byref(o)) == 0
    # NVFP4: d/64 Q/K scale atoms per tile and one V atom per 64 keys
    nv = binding.COpts()
    lib.mxattn_opts_default(ctypes.byref(nv))
    nv.format = 1
    mx_b = lib.mxattn_workspace_bytes(1, 4, 1000, 128, ctypes.byref(o))
    nv_b = lib.mxattn_workspace_bytes(1, 4, 1000, 128, ctypes.byref(nv))
    assert nv_b - mx_b == 2 * 4 * 8 * 512 + 4 * (16 - 8) * 512
    assert lib.mxattn_status_string(5) == b"MXATTN_ERR_TIMEOUT"


def test_validation_rejects_before_enqueue(lib):
    """Invalid arguments return a status without touching the (fake) pointers."""
    o = binding.COpts()
    lib.mxattn_opts_default(ctypes.byref(o))
    fake = ctypes.c_void_p(0x1000)
    P = ctypes.byref(o)
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 96, 0.1, P, fake, None) == 1       # d
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 0, 64, 0.1, P, fake, None) == 1         # N
    assert lib.mxattn_forward(None, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1       # null
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, -1.0, P, fake, None) == 1      # scale
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 3       # no workspace
    assert lib.mxattn_forward_cross(fake, fake, fake, 1, 1, 256, 0, 64, 0.1, P, fake, None) == 1    # Nk
    assert lib.mxattn_forward_cross(fake, fake, fake, 1, 1, 256, 100, 96, 0.1, P, fake, None) == 1  # d
    assert lib.mxattn_forward_cross(fake, fake, fake, 1, 1, 256, 100, 64, 0.1, P, fake, None) == 3  # no workspace
    assert lib.mxattn_forward_host(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 3       # no workspace
    assert lib.mxattn_forward_host(None, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1       # null
    o.key_tile = 128  # supported: only the workspace is missing
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 3
    o.key_tile = 96
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1
    o.key_tile, o.format = 128, 1  # NVFP4 runs with 64-key tiles only
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 2
    o.key_tile, o.format = 64, 0
    o.wait_budget_cycles = -5
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1
    o.wait_budget_cycles = 0
    o.causal = 2
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1
    o.causal = 1  # causal masking needs a query/key position correspondence
    assert lib.mxattn_attention_mxfp4_dump(fake, fake, fake, fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, 0, 0,
                                           fake, None) == 2  # the dump runs full attention only
    assert lib.mxattn_forward_cross(fake, fake, fake, 1, 1, 256, 100, 64, 0.1, P, fake, None) == 2
    assert lib.mxattn_forward_cross(fake, fake, fake, 1, 1, 256, 256, 64, 0.1, P, fake, None) == 2
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 3  # no workspace
    o.causal = 0
    o.format = 2
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1
    o.format = 1  # NVFP4 runs full attention only
    o.causal = 1
    assert lib.mxattn_forward(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 2
    o.causal = 0
    assert lib.mxattn_forward_varlen(fake, fake, fake, fake, 2, 2, 100, 64, 0.1, P, fake, None) == 2
    o.format = 0
    V = lib.mxattn_forward_varlen
    assert V(fake, fake, fake, fake, 0, 2, 100, 64, 0.1, P, fake, None) == 1     # nseq
    assert V(fake, fake, fake, fake, 2, 2, 100, 96, 0.1, P, fake, None) == 1     # d
    assert V(fake, fake, fake, None, 2, 2, 100, 64, 0.1, P, fake, None) == 1     # cu_seqlens
    assert V(fake, fake, fake, fake, 2, 2, 100, 64, 0.1, P, fake, None) == 3     # no workspace
    o.workspace, o.workspace_bytes = ctypes.c_void_p(0x100000), 1 << 30
    assert V(fake, fake, fake, ctypes.c_void_p(0x1002), 2, 2, 100, 64, 0.1, P, fake, None) == 1  # unaligned
    o.workspace, o.workspace_bytes = None, 0
    o.scale_rule = 3
    o.qmax = 9.0
    assert lib.mxattn_quant_v(fake, 1, 1, 256, 64, P, fake, fake, None) == 1
    o.scale_rule = 7
    assert lib.mxattn_quant_v(fake, 1, 1, 256, 64, P, fake, fake, None) == 1
    o.scale_rule = 0
    assert lib.mxattn_quantize_mxfp4(fake, 10, 10, 2, P, fake, fake, None) == 1
    assert lib.mxattn_fp4_mma_probe(1, 1, 96, None) == 1
    qs = (ctypes.c_float * 3)(6.0, 7.25, 8.0)
    assert lib.mxattn_qmax_sweep(fake, 4, 96, 0, 1, qs, 3, fake, fake, None) == 1       # rotate needs d
    assert lib.mxattn_qmax_sweep(fake, 4, 128, 0, 0, qs, 0, fake, fake, None) == 1      # nq
    bad = (ctypes.c_float * 2)(7.25, 7.0)
    assert lib.mxattn_qmax_sweep(fake, 4, 128, 0, 0, bad, 2, fake, fake, None) == 1     # not increasing
    out = (ctypes.c_float * 2)(6.0, 9.0)
    assert lib.mxattn_qmax_sweep(fake, 4, 128, 0, 0, out, 2, fake, fake, None) == 1     # q > 8


def test_package_import_does_not_need_the_library(monkeypatch):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "lib_path", lambda: "/nonexistent/libmxattn.so")
    with pytest.raises(ImportError):
        binding.load()


def _align256(x):
    return (x + 255) // 256 * 256


def test_workspace_sizes_follow_the_header(lib):
    """The workspace sizes are the header's layouts added up: status block, then (varlen) the tile
    table, then each packed operand, every piece 256-byte aligned."""
    o = binding.COpts()
    lib.mxattn_opts_default(ctypes.byref(o))
    B, H, N, d = 2, 3, 1000, 128
    t128, t64 = (N + 127) // 128, (N + 63) // 64
    codes = B * H * t128 * 128 * d // 2
    pieces = [codes, B * H * t128 * 512, codes, B * H * t128 * 512, B * H * t64 * d * 32, B * H * t128 * 512]
    total = 256
    for p in pieces:
        total = _align256(total + p)
    assert lib.mxattn_workspace_bytes(B, H, N, d, ctypes.byref(o)) == total
    # NVFP4: d/64 Q/K scale atoms per tile, one V atom per 64 keys
    o.format = 1
    pieces = [codes, B * H * t128 * 512 * 2, codes, B * H * t128 * 512 * 2, B * H * t64 * d * 32, B * H * t64 * 512]
    total = 256
    for p in pieces:
        total = _align256(total + p)
    assert lib.mxattn_workspace_bytes(B, H, N, d, ctypes.byref(o)) == total
    o.format = 0
    # varlen: (T + 127 nseq) / 128 tiles per head, the tile table after the status block
    nseq, T = 5, 1000
    tph = (T + 127 * nseq) // 128
    vcodes = H * tph * 128 * d // 2
    pieces = [(nseq + 1) * 4, vcodes, H * tph * 512, vcodes, H * tph * 512, vcodes, H * tph * 512]
    total = 256
    for p in pieces:
        total = _align256(total + p)
    assert lib.mxattn_workspace_bytes_varlen(nseq, H, T, d, ctypes.byref(o)) == total
    # the per-operand sizes add up to the same layout
    sizes = (ctypes.c_size_t * 6)()
    o.format = 1
    assert lib.mxattn_operand_bytes(B, H, N, d, ctypes.byref(o), sizes) == 0
    assert list(sizes) == [codes, B * H * t128 * 1024, codes, B * H * t128 * 1024, B * H * t64 * d * 32,
                           B * H * t64 * 512]
    o.format = 3
    assert lib.mxattn_operand_bytes(B, H, N, d, ctypes.byref(o), sizes) == 1
    o.format = 0
    assert lib.mxattn_operand_bytes(B, H, N, 96, ctypes.byref(o), sizes) == 1
    assert lib.mxattn_operand_bytes(B, H, N, d, ctypes.byref(o), None) == 1
    # the host-buffer call stages two chunks and keeps two sets of packed operands (two compute streams)
    host = lib.mxattn_workspace_bytes_host(1, 40, 75600, 128, ctypes.byref(o))
    head = 75600 * 128 * 2
    one_set = lib.mxattn_workspace_bytes(1, 1, 75600, 128, ctypes.byref(o)) - 256
    assert host >= 256 + 2 * 3 * head + 2 * head + 2 * one_set


def test_noalloc_checks_arguments_before_enqueueing():
    """mxattn_forward_noalloc runs every argument check of mxattn_forward before it touches the
    device: on this CPU-only host any device call would fail with MXATTN_ERR_CUDA, so an argument
    error must come back as MXATTN_ERR_INVALID_ARG."""
    lib = binding.load()
    o = binding.COpts()
    lib.mxattn_opts_default(ctypes.byref(o))
    P = ctypes.byref(o)
    fake, odd = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1008)
    assert lib.mxattn_forward_noalloc(odd, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1      # misaligned q
    assert lib.mxattn_forward_noalloc(fake, fake, fake, 1, 1, 256, 64, -1.0, P, fake, None) == 1    # scale
    assert lib.mxattn_forward_noalloc(fake, fake, None, 1, 1, 256, 64, 0.1, P, fake, None) == 1     # null v
    o.pnq = 3
    assert lib.mxattn_forward_noalloc(fake, fake, fake, 1, 1, 256, 64, 0.1, P, fake, None) == 1     # options
