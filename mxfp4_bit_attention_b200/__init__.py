"""MXAttention MXFP4 forward attention for NVIDIA B200 (sm_100a).

The compute lives in ``libmxattn.so`` (hand-written CUDA kernels behind a C
ABI, declared in ``include/mxattn.h``); ``binding`` marshals torch tensors into
those calls.  Importing this package does not load the library; the first
call does, and raises if the library is missing.
"""
from .binding import (  # noqa: F401
    Opts,
    MXAttnError,
    SCALE_UOS,
    SCALE_QMAX6,
    SCALE_OCP,
    SCALE_CEIL_CUSTOM,
    lib_path,
    load,
    mxattn_forward,
    mxattn_attention_mxfp4,
    mxattn_hadamard_quant_qk,
    mxattn_quant_v,
    mxattn_quantize_mxfp4,
    mxattn_workspace_bytes,
    mxattn_get_device_error,
    mxattn_fp4_mma_probe,
    operand_sizes,
)
