"""B200-native Sherry 1.25-bit ternary GEMV/GEMM (sm_100a CUDA kernels behind a C ABI).

The compute path lives in ``libsherry.so`` (``csrc/``, header ``include/sherry.h``);
``sherry`` is its thin Python binding.
"""
from .sherry import (  # noqa: F401
    GroupedGemv, GroupedGemvBf16, SherryError, codes_shape, device_error, gemm, gemm_acc, gemv, gemv_acc, gemv_grouped,
    gemv_static, quantize_act, gemv_bf16, gemv_bf16_grouped, gemv_bf16_workspace_bytes,
    gemv_workspace_bytes, lib, library_path, pack, packed_bytes, workspace,
    GroupedGemvF32, quantize_f32, quantize_swiglu, gemv_f32, gemv_swiglu, gemv_f32_grouped,
    gemv_f32_workspace_bytes,
)
