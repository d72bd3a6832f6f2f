"""mxattn_forward_host: the forward pass from and to host memory with the transfers pipelined
against the kernels (chunks of heads on internal copy streams).  Each chunk is an independent
problem, so the output must equal mxattn_forward's on device copies bit for bit, with page-locked
and with pageable host buffers, for head counts that do not divide into the chunks evenly, and
call after call."""
import ctypes

import numpy as np
import pytest

from mxfp4_bit_attention_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _host(g, w, B, H, pin):
    import torch
    out = []
    for n in "qkv":
        t = torch.from_numpy(np.ascontiguousarray(g[n]))
        if w.dtype == "bf16":
            t = t.view(torch.int16).view(torch.bfloat16)
        t = t.reshape(B, H, w.N, w.d)
        out.append(t.pin_memory() if pin else t.clone())
    return out


@pytest.mark.parametrize("B,H,N,d,dtype,pin", [
    (1, 8, 4096, 128, "bf16", True),     # 8 chunks of one head
    (2, 23, 1000, 64, "fp32", True),     # 46 heads: 23 chunks of 2 heads
    (1, 3, 700, 128, "bf16", False),     # pageable buffers: same result, no overlap
])
def test_host_forward_equals_device_forward(B, H, N, d, dtype, pin):
    import torch
    w = inputs.Workload("host", B, H, N, d, dtype, 31)
    g = inputs.generate(w)
    hq, hk, hv = _host(g, w, B, H, pin)
    scale = float(np.float32(d ** -0.5))
    ref = binding.mxattn_forward(hq.cuda(), hk.cuda(), hv.cuda(), scale).cpu()
    out = torch.empty_like(hq)
    if pin:
        out = out.pin_memory()
    ws = None
    for _ in range(2):  # the same workspace, twice
        out.fill_(float("nan"))
        binding.mxattn_forward_host(hq, hk, hv, scale, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16) if dtype == "bf16" else out.view(torch.int32),
                           ref.view(torch.int16) if dtype == "bf16" else ref.view(torch.int32))
        if ws is None:
            c = binding._copts(None, binding._dtype_code(hq))
            nbytes = binding.load().mxattn_workspace_bytes_host(B, H, N, d, ctypes.byref(c))
            ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
