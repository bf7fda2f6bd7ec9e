"""Group-wise affine quantized matrix products on B200 (sm_100a).

The compute path is the C-ABI library ``libnvq.so`` (CUDA kernels, declared in
include/nvq.h); the functions exported here only marshal torch tensors and
streams into it. ``group_wise_affine_dequant_b200.workloads`` holds the seeded
synthetic inputs.
"""
from .binding import (  # noqa: F401
    NV_ROW_INDEPENDENT_ROWS,
    NvqError,
    lib,
    nv_gather_mm,
    nv_gather_qmm,
    nv_gather_qmm_flags,
    nv_gather_qmm_workspace_size,
    nv_dequantize_affine,
    nv_dequantize_fp,
    nv_moe_swiglu,
    nv_moe_swiglu_workspace_size,
    nv_pipeline_error,
    nv_pipeline_selftest,
    nv_qmm,
    nv_qmm_batched,
    nv_qmm_fp,
    nv_qmm_splits,
    nv_quantize_affine,
    nv_quantize_fp,
    nv_status_string,
)
