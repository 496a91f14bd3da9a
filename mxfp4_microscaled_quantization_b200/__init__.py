"""B200-native MXFP4 attention with Universal Optimal Scaling and
Pre-Normalization Quantization (MXAttention), behind a C-ABI CUDA library.

The compute runs in ``libmxattn.so`` (CUDA kernels for sm_100a); this package
only marshals arguments.  Importing it does not load the library; the first
call does, and fails loudly if the library was not built.
"""
from . import ulysses, workloads  # noqa: F401
from .mxattn import (  # noqa: F401
    MxattnError,
    attention_from_host,
    declared_symbols,
    forward_host_workspace_size,
    host_groups,
    mxattn_attend,
    mxattn_forward,
    mxattn_forward_noalloc,
    mxattn_forward_quantized,
    mxattn_nvfp4_attend,
    mxattn_nvfp4_forward,
    mxattn_nvfp4_prepare,
    mxattn_nvfp4_quantize,
    mxattn_mxf4_mma_loop,
    mxattn_p_selftest,
    mxattn_prepare,
    mxattn_quantize,
    mxattn_quantize_vt,
    mxattn_status_string,
    mxattn_wait_selftest,
    mxattn_workspace_size,
    mxattn_workspace_status,
    new_nvfp4_workspace,
    new_workspace,
    nvfp4_workspace_layout,
    nvfp4_workspace_size,
    workspace_layout,
)
