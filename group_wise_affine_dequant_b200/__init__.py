"""Group-wise affine quantized matrix products on B200 (sm_100a).

The compute path is the C-ABI library ``libnvq.so`` (CUDA kernels); the
Python functions here only marshal torch tensors and streams into it. Import
``group_wise_affine_dequant_b200.workloads`` for the seeded synthetic inputs.
"""
