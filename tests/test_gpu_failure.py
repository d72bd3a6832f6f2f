"""Failure detection on the GPU without a fault: pipeline waits that run out.

Every mbarrier wait in the attention kernel is bounded.  With wait_budget_cycles = 1 a
pipeline wait gives up as soon as its first hardware try_wait returns without the phase (that
try_wait may itself sleep for a short hardware-defined time, so a problem of a few microseconds
can finish without any wait expiring; the cases here run long enough that some do): each CTA
that gives up raises its abort flag, lets the bulk copies it issued
land and its MMAs finish (those drains keep the full budget), frees its tensor memory and exits,
and the workspace status word reports MXATTN_ERR_TIMEOUT.  The context must stay usable: the
next call with the default budget gives the normal result, bit for bit.
"""
import numpy as np
import pytest

from mxfp4_bit_attention_b200 import binding, inputs
from helpers import to_device

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # MXATTN_ERR_TIMEOUT


@pytest.mark.parametrize("N", [1000, 4096])
def test_expired_waits_report_timeout_and_leave_the_context_usable(N):
    import torch
    w = inputs.Workload("expiry", 1, 4, N, 128, "bf16", 21)
    g = inputs.generate(w)
    q, k, v = (to_device(g[n], w.dtype, (1, w.H, w.N, w.d)) for n in "qkv")
    scale = float(np.float32(w.d ** -0.5))
    ws = binding.new_workspace(1, w.H, w.N, w.d)
    ref = binding.mxattn_forward(q, k, v, scale, binding.Opts(), workspace=ws).clone()
    assert binding.mxattn_get_device_error(ws) == 0

    binding.mxattn_forward(q, k, v, scale, binding.Opts(wait_budget_cycles=1), workspace=ws)
    torch.cuda.synchronize()
    assert binding.mxattn_get_device_error(ws) == TIMEOUT
    assert binding.mxattn_get_device_error(ws) == 0  # reading the status clears it

    again = binding.mxattn_forward(q, k, v, scale, binding.Opts(), workspace=ws)
    torch.cuda.synchronize()
    assert binding.mxattn_get_device_error(ws) == 0
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))
