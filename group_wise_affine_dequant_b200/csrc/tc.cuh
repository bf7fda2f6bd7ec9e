// Tensor-core (tcgen05 / TMEM / TMA) quantized GEMM for many rows: host side.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvq {

bool tc_supported(int64_t M, int64_t K, int64_t N, int bits, int gs);
// item_rows: rows of one item of a batch (0: all M rows are one item); the
// tiling and the split-K partition count follow it.
// transpose = 0: weights stored [K, N] grouped along N (tc_supported_t0).
cudaError_t launch_tc_qmm(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                          const void* scales, const void* biases, int gs, int bits, void* y,
                          cudaStream_t stream, int num_sms, int64_t item_rows = 0,
                          int transpose = 1, int fmt = 0);
bool tc_supported_t0(int64_t M, int64_t K, int64_t N, int bits, int gs);
// K-partitions the tiled kernel uses for an item of m_rows rows (1: no split).
int tc_splits(int64_t m_rows, int64_t K, int64_t N, int num_sms, int bits, int transpose);

// Read and clear the error word of the tensor-core kernels (synchronous).
unsigned int tc_error_take();

// Mixture-of-experts product on the tensor cores (transposed: weights as the
// 128-row operand, each expert's gathered activation rows as N). perm/offsets
// come from the gather router.
bool tc_gather_supported(int64_t K, int64_t N, int bits, int gs);
// act_gate (nullable, bf16 [R, N]): store silu(act_gate) * product instead of
// the product, over act_gate in place when y == act_gate.
cudaError_t launch_tc_gather(const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs,
                             const uint32_t* perm, const uint32_t* offsets, int64_t E, int64_t N,
                             const uint32_t* codes, const void* scales, const void* biases, int gs,
                             int bits, void* y, cudaStream_t stream, int num_sms,
                             const void* act_gate = nullptr);
unsigned int tc_gather_error_take();

// The same grouped product with full-precision (bf16) experts [E, N, K].
bool tc_gather_mm_supported(int64_t K, int64_t N);
cudaError_t launch_tc_gather_mm(const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs,
                                const uint32_t* perm, const uint32_t* offsets, int64_t E, int64_t N,
                                const void* w, void* y, cudaStream_t stream, int num_sms);
unsigned int tc_gather_mm_error_take();

// The quantized grouped product with experts stored [E][K, N] (transpose = 0),
// grouped along N; N * bits a multiple of 128 and K of 64.
bool tc_gather_t0_supported(int64_t K, int64_t N, int bits, int gs);
cudaError_t launch_tc_gather_t0(const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs,
                                const uint32_t* perm, const uint32_t* offsets, int64_t E, int64_t N,
                                const uint32_t* codes, const void* scales, const void* biases, int gs,
                                int bits, void* y, cudaStream_t stream, int num_sms);
unsigned int tc_gather_t0_error_take();

}  // namespace nvq
