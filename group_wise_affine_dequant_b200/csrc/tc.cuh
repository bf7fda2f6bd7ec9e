// Tensor-core (tcgen05 / TMEM / TMA) quantized GEMM for many rows: host side.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvq {

bool tc_supported(int64_t M, int64_t K, int64_t N, int bits, int gs);
cudaError_t launch_tc_qmm(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                          const void* scales, const void* biases, int gs, int bits, void* y,
                          cudaStream_t stream, int num_sms);

// Read and clear the error word of the tensor-core kernels (synchronous).
unsigned int tc_error_take();

}  // namespace nvq
