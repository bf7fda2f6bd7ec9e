// Plain per-output kernels: one thread computes one output element with a
// sequential k loop, dequantizing each weight as scale * code + bias
// ("Docs / Quantization", section "Affine") and accumulating in fp64. They
// serve fp32 activations (fp32 scales and biases) and the shapes the
// matrix-vector and tensor-core kernels do not cover. Every output is
// independent of every other one, so they are row-exact by construction.
#include "common.cuh"
#include "kernels.cuh"

namespace nvq {
namespace {

template <int DT>
__device__ __forceinline__ double dot_one(const void* x_row, int64_t K, int64_t N, int64_t n,
                                          const uint32_t* codes, const void* scales,
                                          const void* biases, int gs, int bits, int transpose) {
    const uint32_t mask = (1u << bits) - 1u;
    const int per = 32 / bits;
    double acc = 0.0;
    if (transpose) {  // weights [N, K], grouped along K
        const int64_t wpr = K * bits / 32, gpr = K / gs;
        for (int64_t k = 0; k < K; ++k) {
            const uint32_t word = __ldg(codes + n * wpr + k / per);
            const float c = static_cast<float>((word >> ((k % per) * bits)) & mask);
            const float s = load_elem<DT>(scales, n * gpr + k / gs);
            const float b = load_elem<DT>(biases, n * gpr + k / gs);
            acc += static_cast<double>(load_elem<DT>(x_row, k)) *
                   (static_cast<double>(s) * c + static_cast<double>(b));
        }
    } else {  // weights [K, N], grouped along N
        const int64_t wpr = N * bits / 32, gpr = N / gs;
        for (int64_t k = 0; k < K; ++k) {
            const uint32_t word = __ldg(codes + k * wpr + n / per);
            const float c = static_cast<float>((word >> ((n % per) * bits)) & mask);
            const float s = load_elem<DT>(scales, k * gpr + n / gs);
            const float b = load_elem<DT>(biases, k * gpr + n / gs);
            acc += static_cast<double>(load_elem<DT>(x_row, k)) *
                   (static_cast<double>(s) * c + static_cast<double>(b));
        }
    }
    return acc;
}

template <int DT>
__global__ void __launch_bounds__(256) qmm_simt_kernel(const void* x, int64_t M, int64_t K,
                                                       int64_t N, const uint32_t* codes,
                                                       const void* scales, const void* biases,
                                                       int gs, int bits, int transpose, void* y) {
    const size_t esz = DT == NV_F32 ? 4 : 2;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < M * N;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = i / N, n = i % N;
        const void* xr = static_cast<const char*>(x) + static_cast<size_t>(m * K) * esz;
        const double v = dot_one<DT>(xr, K, N, n, codes, scales, biases, gs, bits, transpose);
        store_elem<DT>(y, i, static_cast<float>(v));
    }
}

template <int DT>
__global__ void __launch_bounds__(256) gather_simt_kernel(
    const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs, const uint32_t* rhs, int64_t R,
    int64_t E, int64_t N, const uint32_t* codes, const void* scales, const void* biases, int gs,
    int bits, int transpose, void* y) {
    const size_t esz = DT == NV_F32 ? 4 : 2;
    const int64_t words_e = N * K * bits / 32, groups_e = N * K / gs;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < R * N;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / N, n = i % N;
        const int64_t t = lhs ? static_cast<int64_t>(__ldg(lhs + r)) : r;
        const int64_t e = __ldg(rhs + r);
        double v = 0.0;
        if (t < x_rows && e < E) {  // out-of-range pairs are flagged by the router; output 0
            const void* xr = static_cast<const char*>(x) + static_cast<size_t>(t * K) * esz;
            v = dot_one<DT>(xr, K, N, n, codes + e * words_e,
                            static_cast<const char*>(scales) + static_cast<size_t>(e * groups_e) * esz,
                            static_cast<const char*>(biases) + static_cast<size_t>(e * groups_e) * esz,
                            gs, bits, transpose);
        }
        store_elem<DT>(y, i, static_cast<float>(v));
    }
}

unsigned grid_for(int64_t total) {
    int64_t b = (total + 255) / 256;
    if (b > 65535) b = 65535;
    return static_cast<unsigned>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_qmm_simt(const void* x, int dt, int64_t M, int64_t K, int64_t N,
                            const uint32_t* codes, const void* scales, const void* biases,
                            int gs, int bits, int transpose, void* y, cudaStream_t stream) {
    if (M * N == 0) return cudaSuccess;
    if (dt == NV_F32)
        qmm_simt_kernel<NV_F32><<<grid_for(M * N), 256, 0, stream>>>(x, M, K, N, codes, scales,
                                                                     biases, gs, bits, transpose, y);
    else
        qmm_simt_kernel<NV_BF16><<<grid_for(M * N), 256, 0, stream>>>(x, M, K, N, codes, scales,
                                                                      biases, gs, bits, transpose, y);
    return cudaGetLastError();
}

cudaError_t launch_gather_simt(const void* x, int dt, int64_t x_rows, int64_t K,
                               const uint32_t* lhs, const uint32_t* rhs, int64_t R, int64_t E,
                               int64_t N, const uint32_t* codes, const void* scales,
                               const void* biases, int gs, int bits, int transpose, void* y,
                               cudaStream_t stream) {
    if (R * N == 0) return cudaSuccess;
    if (dt == NV_F32)
        gather_simt_kernel<NV_F32><<<grid_for(R * N), 256, 0, stream>>>(
            x, x_rows, K, lhs, rhs, R, E, N, codes, scales, biases, gs, bits, transpose, y);
    else
        gather_simt_kernel<NV_BF16><<<grid_for(R * N), 256, 0, stream>>>(
            x, x_rows, K, lhs, rhs, R, E, N, codes, scales, biases, gs, bits, transpose, y);
    return cudaGetLastError();
}

}  // namespace nvq
