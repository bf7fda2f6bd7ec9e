// Internal launchers of the nvq kernels (host side). Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvq {

cudaError_t launch_quantize_affine(const void* w, int dt, int64_t rows, int64_t cols, int gs,
                                   int bits, uint32_t* codes, void* scales, void* biases,
                                   cudaStream_t stream, int num_sms);

// w_hat = scale * code + bias for every code, in the scales' dtype.
cudaError_t launch_dequantize_affine(const uint32_t* codes, const void* scales,
                                     const void* biases, int dt, int64_t rows, int64_t cols,
                                     int gs, int bits, void* out, cudaStream_t stream,
                                     int num_sms);

// Matrix-vector products for up to 8 rows, weights [N, K] (transpose = 1), bf16.
bool qmv_supported(int bits, int gs);
unsigned int qmv_error_take();  // read and clear the kernels' pipeline error word
cudaError_t launch_qmv(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                       const void* scales, const void* biases, int gs, int bits, void* y,
                       cudaStream_t stream, int num_sms);

// Grouped form for gather: problems (expert, first sorted pair, count <= 8) come
// from the routing kernel; max_problems bounds the grid.
cudaError_t launch_qmv_gather(const void* x, int64_t K, int64_t N, const uint32_t* codes,
                              const void* scales, const void* biases, int gs, int bits,
                              const uint32_t* lhs, const uint32_t* perm,
                              const uint32_t* problems, const uint32_t* num_problems,
                              int64_t max_problems, int64_t E, void* y, cudaStream_t stream,
                              int num_sms);

// Matrix-vector products for up to 8 rows, weights [K, N] (transpose = 0), bf16.
bool qmvt_supported(int bits, int gs);
bool qmvt_supported_m(int bits, int gs, int64_t M);
cudaError_t launch_qmvt(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                        const void* scales, const void* biases, int gs, int bits, void* y,
                        cudaStream_t stream, int num_sms);

// Plain per-output kernel: any M, either layout, fp32 or bf16.
cudaError_t launch_qmm_simt(const void* x, int dt, int64_t M, int64_t K, int64_t N,
                            const uint32_t* codes, const void* scales, const void* biases,
                            int gs, int bits, int transpose, void* y, cudaStream_t stream);

// Gather through the plain per-output kernel (fp32, or shapes the fast kernels lack).
cudaError_t launch_gather_simt(const void* x, int dt, int64_t x_rows, int64_t K,
                               const uint32_t* lhs, const uint32_t* rhs, int64_t R, int64_t E,
                               int64_t N, const uint32_t* codes, const void* scales,
                               const void* biases, int gs, int bits, int transpose, void* y,
                               cudaStream_t stream);

// Self-test of the bounded pipeline waits: one wait on a barrier nothing
// completes gives up after limit_ns and records kSelftestWaitCode in the error
// word that selftest_error_take() reads and clears.
constexpr unsigned int kSelftestWaitCode = 0x5E;
cudaError_t launch_pipeline_selftest(uint64_t limit_ns, cudaStream_t stream);
unsigned int selftest_error_take();

// Largest expert count the single-CTA router handles (its histograms live in
// shared memory).
constexpr int64_t kMaxExperts = 1023;

// Routing for gather: flags, expert offsets, stable expert order, problem list.
struct GatherWorkspace {
    uint32_t* flags;         // [1]
    uint32_t* num_problems;  // [1]
    uint32_t* offsets;       // [E + 2]
    uint32_t* perm;          // [R]
    uint32_t* problems;      // [max_problems * 4]
    int64_t max_problems;
};
size_t gather_workspace_bytes(int64_t R, int64_t E);
GatherWorkspace gather_workspace_carve(void* base, int64_t R, int64_t E);
// want_problems: also write the (expert, first, count <= 8) work items of the
// matrix-vector route (the tensor-core routes read only offsets and perm).
cudaError_t launch_gather_route(const uint32_t* lhs, const uint32_t* rhs, int64_t R, int64_t E,
                                int64_t x_rows, int sorted, const GatherWorkspace& ws,
                                cudaStream_t stream, bool want_problems);

}  // namespace nvq
