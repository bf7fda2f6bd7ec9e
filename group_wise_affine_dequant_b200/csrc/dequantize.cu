// Dequantizer ("Docs / Quantization", section "Affine": every value is stored
// as a small unsigned code with a scale and a bias per group, w ~ scale *
// code + bias; the nuvec crate docs list `dequantize` beside the quantizer).
//
// The codes of every row are one flat run of words, and a group never crosses
// a row (cols is a multiple of the group size, and a word's 32 / bits codes
// never cross a group), so word i of the whole array holds the values
// [i * per_word, (i + 1) * per_word) of the flat output and belongs to group
// (i * per_word) / group_size of the flat scale and bias arrays. The kernel is
// therefore a flat map over words: a warp takes 128 consecutive words per
// step, lane l the words 32 q + l (q < 4), so that every load and store
// instruction of the warp covers one contiguous run; it writes each word's
// values with 8- to 16-byte stores and strides over the array. Every value is
// the exact scale * code + bias rounded once to the output dtype: one fp32
// fused multiply-add for fp32 outputs, one bf16 fused multiply-add (on codes
// held exactly as bf16, every integer below 256 being a bf16 number) for bf16
// outputs. HBM-bound: bytes moved per weight are bits / 8 (codes) +
// 4 / group_size or 8 / group_size (scale and bias) + the output element size.
#include "common.cuh"
#include "kernels.cuh"

namespace nvq {
namespace {

// Exact fp32 value of a code below 2^23: its bits under the mantissa of 2^23,
// minus 2^23.
__device__ __forceinline__ float code_f32(uint32_t c) {
    return __uint_as_float(0x4B000000u | c) - 8388608.0f;
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t f2_to_bf2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Values of one word, stored at out (16-byte aligned for bf16 at 4 bits and
// wider outputs, 8-byte for 8-bit codes to bf16). s2, b2: (s, s) and (b, b)
// as bf16 pairs (bf16 outputs only).
template <int DT, int BITS>
__device__ __forceinline__ void word_out(uint32_t w, float s, float b, uint32_t s2, uint32_t b2,
                                         void* out) {
    constexpr int PER = 32 / BITS;
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    if constexpr (DT == NV_BF16) {
        uint32_t v[PER / 2];
#pragma unroll
        for (int j = 0; j < PER / 2; ++j) {
            const uint32_t lo = (w >> (2 * j * BITS)) & MASK;
            const uint32_t hi = (w >> ((2 * j + 1) * BITS)) & MASK;
            uint32_t c2;  // (lo, hi) as exact bf16
            if constexpr (BITS == 8) {
                c2 = f2_to_bf2(code_f32(lo), code_f32(hi));
            } else {  // 128 + c for c < 128 (bf16's unit at 128 is 1), minus 128
                c2 = bf2_sub(lo | (hi << 16) | 0x43004300u, 0x43004300u);
            }
            v[j] = bf2_fma(s2, c2, b2);
        }
        if constexpr (PER / 2 >= 4) {
            uint4* o = reinterpret_cast<uint4*>(out);
#pragma unroll
            for (int q = 0; q < PER / 8; ++q) o[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
            *reinterpret_cast<uint2*>(out) = make_uint2(v[0], v[1]);
        }
    } else {
        float v[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) v[j] = fmaf(s, code_f32((w >> (j * BITS)) & MASK), b);
        float4* o = reinterpret_cast<float4*>(out);
#pragma unroll
        for (int q = 0; q < PER / 4; ++q) o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
}

template <int DT, int BITS>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t* __restrict__ codes,
                                                         const void* __restrict__ scales,
                                                         const void* __restrict__ biases,
                                                         int64_t words, int lg_gs,
                                                         void* __restrict__ out) {
    // launched as the programmatic dependent of the previous kernel: the next
    // call may launch at once; this one waits for the previous grid before its
    // first read or write
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int PER = 32 / BITS;
    constexpr int ESZ = DT == NV_F32 ? 4 : 2;
    char* o = static_cast<char*>(out);
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    // A warp takes 128 consecutive words per step, lane l the words 32 q + l:
    // each load and each store instruction of the warp covers one contiguous
    // run (128 code bytes in; 32 words' outputs out).
    for (int64_t base = warp * 128; base < words; base += nwarps * 128) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t i = base + 32 * q + lane;
            w[q] = i < words ? __ldg(codes + i) : 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t i = base + 32 * q + lane;
            if (i < words) {
                const int64_t g = (i * PER) >> lg_gs;
                const float s = load_elem<DT>(scales, g), b = load_elem<DT>(biases, g);
                const uint32_t s2 = (__float_as_uint(s) >> 16) * 0x00010001u;
                const uint32_t b2 = (__float_as_uint(b) >> 16) * 0x00010001u;
                word_out<DT, BITS>(w[q], s, b, s2, b2, o + i * PER * ESZ);
            }
        }
    }
}

template <int DT>
cudaError_t launch_dt(const uint32_t* codes, const void* scales, const void* biases,
                      int64_t words, int gs, int bits, void* out, cudaStream_t stream,
                      int num_sms) {
    const int lg_gs = gs == 32 ? 5 : gs == 64 ? 6 : 7;
    const int threads = 256;
    int64_t blocks = (words / 4 + threads - 1) / threads;  // four words per thread
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    void (*k)(const uint32_t*, const void*, const void*, int64_t, int, void*);
    switch (bits) {
        case 1: k = dequantize_kernel<DT, 1>; break;
        case 2: k = dequantize_kernel<DT, 2>; break;
        case 4: k = dequantize_kernel<DT, 4>; break;
        case 8: k = dequantize_kernel<DT, 8>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, codes, scales, biases, words, lg_gs, out);
}

}  // namespace

cudaError_t launch_dequantize_affine(const uint32_t* codes, const void* scales,
                                     const void* biases, int dt, int64_t rows, int64_t cols,
                                     int gs, int bits, void* out, cudaStream_t stream,
                                     int num_sms) {
    const int64_t words = rows * (cols * bits / 32);
    if (words == 0) return cudaSuccess;
    return dt == NV_F32 ? launch_dt<NV_F32>(codes, scales, biases, words, gs, bits, out, stream, num_sms)
                        : launch_dt<NV_BF16>(codes, scales, biases, words, gs, bits, out, stream, num_sms);
}

}  // namespace nvq
