"""mxattn_forward_noalloc: the forward pass for callers that cannot allocate.

A process whose memory manager has already reserved the GPU's memory (or a
plain C caller with no allocator) cannot hand the library a workspace.  This
entry point takes its scratch from a fixed array inside the library instead,
so it must give the same output as mxattn_forward with a caller workspace,
call after call, and must refuse problems larger than that array.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process (the first call on the device does the one-time address lookup).
"""
import ctypes

import numpy as np
import pytest

from mxfp4_bit_attention_b200 import binding, inputs
from helpers import to_device

pytestmark = pytest.mark.gpu


def _inputs(workload, heads):
    w = inputs.WORKLOADS[workload]
    g = inputs.generate(w, heads=heads)
    return w, [to_device(g[n], w.dtype, (1, len(heads), w.N, w.d)) for n in "qkv"]


@pytest.mark.parametrize("kt", [64, 128])
@pytest.mark.parametrize("workload,heads", [("tiny", [0]), ("outlier", [0, 1, 2, 3, 4, 5, 6, 7])])
def test_noalloc_matches_workspace_forward_twice(workload, heads, kt):
    """The same kernels on the same inputs as mxattn_forward with a caller workspace: the output
    must agree bit for bit, on the first call and on a second one that finds the previous call's
    contents in the shared scratch."""
    import torch
    w, (q, k, v) = _inputs(workload, heads)
    scale = float(np.float32(w.d ** -0.5))
    opts = binding.Opts(key_tile=kt)
    ref = binding.mxattn_forward(q, k, v, scale, opts)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        binding.mxattn_forward_noalloc(q, k, v, scale, opts, out=out)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = binding.load()
    o = binding.COpts()
    lib.mxattn_opts_default(ctypes.byref(o))
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the size check comes first
    status = lib.mxattn_forward_noalloc(fake, fake, fake, 1, 40, 32760, 128, 0.088, ctypes.byref(o), fake, None)
    assert status == 3  # MXATTN_ERR_WORKSPACE
