// Affine quantizer kernel ("Docs / Quantization", section "Affine").
//
// One warp per group: the lanes find the group's minimum and maximum, every
// lane derives the same fp32 scale and bias, then lane j builds packed word j
// of the group (code i of a word at bits [i*bits, (i+1)*bits)). Every fp32 step
// is an explicitly rounded IEEE operation (__fsub_rn, __fdiv_rn, rintf), so the
// result does not depend on contraction or fast-math settings. A one-off,
// load-time kernel: it is written for exactness, not speed.
#include "common.cuh"
#include "kernels.cuh"

namespace nvq {

// Total order with -0 < +0, so a group's extremes do not depend on visiting order.
__device__ __forceinline__ float min_signed(float a, float b) {
    return (b < a || (b == a && signbit(b))) ? b : a;
}
__device__ __forceinline__ float max_signed(float a, float b) {
    return (b > a || (b == a && !signbit(b))) ? b : a;
}

template <int DT>
__global__ void __launch_bounds__(256) quantize_affine_kernel(const void* __restrict__ w,
                                                              int64_t total_groups, int gs,
                                                              int bits, uint32_t* __restrict__ codes,
                                                              void* __restrict__ scales,
                                                              void* __restrict__ biases) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const float levels = static_cast<float>((1u << bits) - 1u);
    const int per_word = 32 / bits;
    const int words_per_group = gs * bits / 32;

    for (int64_t grp = warp; grp < total_groups; grp += nwarps) {
        // Groups tile each row contiguously, so group grp starts at element grp * gs.
        const int64_t base = grp * gs;
        float mn = load_elem<DT>(w, base + lane), mx = mn;
        for (int i = lane + 32; i < gs; i += 32) {
            float v = load_elem<DT>(w, base + i);
            mn = min_signed(mn, v);
            mx = max_signed(mx, v);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = min_signed(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = max_signed(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        const float scale = __fdiv_rn(__fsub_rn(mx, mn), levels);
        const float bias = mn;
        if (lane < words_per_group) {
            uint32_t word = 0;
            for (int j = 0; j < per_word; ++j) {
                uint32_t q = 0;
                if (scale != 0.0f) {
                    const float v = load_elem<DT>(w, base + lane * per_word + j);
                    float r = rintf(__fdiv_rn(__fsub_rn(v, bias), scale));
                    r = fminf(fmaxf(r, 0.0f), levels);
                    q = static_cast<uint32_t>(r);
                }
                word |= q << (j * bits);
            }
            codes[grp * words_per_group + lane] = word;
        }
        if (lane == 0) {
            store_elem<DT>(scales, grp, scale);
            store_elem<DT>(biases, grp, bias);
        }
    }
}

cudaError_t launch_quantize_affine(const void* w, int dt, int64_t rows, int64_t cols, int gs,
                                   int bits, uint32_t* codes, void* scales, void* biases,
                                   cudaStream_t stream, int num_sms) {
    const int64_t total_groups = rows * (cols / gs);
    if (total_groups == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total_groups + 7) / 8;  // one warp per group
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    if (dt == NV_F32) {
        quantize_affine_kernel<NV_F32><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
            w, total_groups, gs, bits, codes, scales, biases);
    } else {
        quantize_affine_kernel<NV_BF16><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
            w, total_groups, gs, bits, codes, scales, biases);
    }
    return cudaGetLastError();
}

}  // namespace nvq
