// The floating-point quantization modes ("Docs / Quantization", section
// "Floating-point formats": every value a small float, one shared scale per
// group stored as a uint8 code, no biases; dequantization gives bfloat16; the
// product quantized_matmul(q, transpose = true) returns x's dtype). The
// pages' table of the formats did not survive extraction; the formats are the
// published definitions of the three names:
//   MXFP4: E2M1 values, one E8M0 scale (2^(s - 127)) per 32 values;
//   MXFP8: E4M3 values (no infinities), one E8M0 scale per 32 values;
//   NVFP4: E2M1 values, one E4M3 scale per 16 values.
// Codes pack like the affine codes: code j of a word at bits [j*b, (j+1)*b).
//
// Quantizer (one thread per group): amax = max |w|; MX: X = 2^(floor(log2
// amax) - emax) with emax 2 (E2M1) or 8 (E4M3), the scale code clamped to
// 0..254 (0 for an all-zero group); NVFP4: S = fl32(amax / 6) rounded to E4M3.
// Each code is w / X (exact: a power of two) or fl32(w / S) rounded to the
// element grid by the hardware conversion (nearest, ties to the even
// mantissa, saturated at the largest finite value), which equals the oracle's
// brute-force rounding on every finite input.
//
// Products: every element decodes exactly to f16 by the hardware conversion
// (two codes per instruction), widens to fp32 and meets x in fp32 fused
// multiply-adds; the sum over a group (or the part of it in one 16-byte chunk
// of codes) is then multiplied by the group's scale. There is no bias, so
// nothing can cancel between the two factors; with an E8M0 scale the result
// is exactly that of multiplying each dequantized weight first. A warp owns
// one output row of W (every activation row), its lanes stride over 16-byte
// chunks of the row, and lane partial sums are reduced in a fixed order: the
// same operations for every activation row whatever M is (row exactness).
#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"

namespace nvq {
namespace {

constexpr int kMx4 = 1, kMx8 = 2, kNv4 = 3;

template <int MODE>
struct FpFormat {
    static constexpr int GS = MODE == kNv4 ? 16 : 32;  // values per scale
    static constexpr int BITS = MODE == kMx8 ? 8 : 4;
    static constexpr int PER = 32 / BITS;               // codes per word
    static constexpr int CPC = 4 * PER;                 // codes per 16-byte chunk
};

// Two E2M1 codes (one byte, first code in the low nibble) -> f16x2 (first in
// the low half), exact.
__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t byte) {
    uint32_t h;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h) : "r"(byte));
    return h;
}
// Two E4M3 codes (16 bits, first in the low byte) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t pair) {
    uint32_t h;
    asm("{\n\t.reg .b16 s;\n\tcvt.u16.u32 s, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, s;\n\t}" : "=r"(h) : "r"(pair));
    return h;
}
__device__ __forceinline__ void f16x2_f32(uint32_t h, float& lo, float& hi) {
    asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h));
}
// fp32 pair -> bf16x2 (`lo` in the low half), round to nearest even.
__device__ __forceinline__ uint32_t f2_to_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
// fp32 pair -> two E2M1 codes (byte, `lo` in the low nibble) / two E4M3 codes.
__device__ __forceinline__ uint32_t f32x2_e2m1x2(float lo, float hi) {
    uint16_t b;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
        : "=h"(b) : "f"(hi), "f"(lo));
    return b;
}
__device__ __forceinline__ uint32_t f32x2_e4m3x2(float lo, float hi) {
    uint16_t b;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(b) : "f"(hi), "f"(lo));
    return b;
}
__device__ __forceinline__ float e8m0_f32(uint32_t s) {
    return s == 0 ? __uint_as_float(0x00400000u)            // 2^-127
                  : s == 255 ? __uint_as_float(0x7FC00000u)  // NaN
                             : __uint_as_float(s << 23);
}
__device__ __forceinline__ float e4m3_f32(uint32_t s) {
    float lo, hi;
    f16x2_f32(e4m3x2_f16x2(s & 255u), lo, hi);
    return lo;
}
template <int MODE>
__device__ __forceinline__ float scale_f32(uint32_t s) {
    if constexpr (MODE == kNv4) return e4m3_f32(s);
    else return e8m0_f32(s);
}

// ------------------------------------------------------------------ quantize
template <int MODE>
__global__ void quantize_fp_kernel(const void* __restrict__ w, int dt, int64_t rows, int64_t cols,
                                   uint32_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    using F = FpFormat<MODE>;
    const int64_t groups = cols / F::GS;
    const int64_t total = rows * groups;
    const int64_t wpr = cols * F::BITS / 32;
    for (int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; gi < total;
         gi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = gi / groups, g = gi - r * groups;
        const int64_t base = r * cols + g * F::GS;
        float v[F::GS];
#pragma unroll
        for (int i = 0; i < F::GS; ++i)
            v[i] = dt == NV_F32 ? static_cast<const float*>(w)[base + i]
                                : bf16_bits_to_f32(static_cast<const uint16_t*>(w)[base + i]);
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < F::GS; ++i) amax = fmaxf(amax, fabsf(v[i]));
        uint32_t sc = 0;
        if constexpr (MODE == kNv4) {
            sc = f32x2_e4m3x2(__fdiv_rn(amax, 6.0f), 0.f) & 127u;
        } else if (amax > 0.f) {
            int e = ilogbf(amax) - (MODE == kMx8 ? 8 : 2) + 127;
            sc = static_cast<uint32_t>(e < 0 ? 0 : e > 254 ? 254 : e);
        }
        scales[gi] = static_cast<uint8_t>(sc);
        const float X = scale_f32<MODE>(sc);
        uint32_t* out = codes + r * wpr + g * (F::GS * F::BITS / 32);
        const bool zero = MODE == kNv4 && X == 0.f;  // NVFP4 scale 0: every code 0
#pragma unroll
        for (int wd = 0; wd < F::GS * F::BITS / 32; ++wd) {
            uint32_t word = 0;
            if (!zero) {
#pragma unroll
                for (int p = 0; p < F::PER / 2; ++p) {
                    const int i = wd * F::PER + 2 * p;
                    const float t0 = __fdiv_rn(v[i], X), t1 = __fdiv_rn(v[i + 1], X);
                    if constexpr (F::BITS == 4) word |= f32x2_e2m1x2(t0, t1) << (8 * p);
                    else word |= f32x2_e4m3x2(t0, t1) << (16 * p);
                }
            }
            out[wd] = word;
        }
    }
}

// ---------------------------------------------------------------- dequantize
template <int MODE>
__global__ void dequantize_fp_kernel(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                     int64_t rows, int64_t cols, uint16_t* __restrict__ out) {
    using F = FpFormat<MODE>;
    const int64_t wpr = cols * F::BITS / 32;
    const int64_t groups = cols / F::GS;
    const int64_t total = rows * wpr;
    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; wi < total;
         wi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = wi / wpr, j = wi - r * wpr;
        const int64_t k0 = j * F::PER;
        const float S = scale_f32<MODE>(__ldg(scales + r * groups + k0 / F::GS));
        const uint32_t word = __ldg(codes + wi);
        uint32_t o[F::PER / 2];
#pragma unroll
        for (int p = 0; p < F::PER / 2; ++p) {
            const uint32_t h = F::BITS == 4 ? e2m1x2_f16x2((word >> (8 * p)) & 255u)
                                            : e4m3x2_f16x2((word >> (16 * p)) & 0xFFFFu);
            float lo, hi;
            f16x2_f32(h, lo, hi);
            o[p] = f2_to_bf16x2(lo * S, hi * S);
        }
        uint16_t* dst = out + r * cols + k0;
        if constexpr (F::PER == 8) {
            *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
        } else {
            *reinterpret_cast<uint2*>(dst) = make_uint2(o[0], o[1]);
        }
    }
}

// ------------------------------------------------- products of 1 .. 8 rows
__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

constexpr int kFpRowsPerBlock = 8;  // one warp per output row

template <int MODE, int MT>
__global__ void __launch_bounds__(kFpRowsPerBlock * 32)
qmv_fp_kernel(const uint16_t* __restrict__ x, int M, int64_t K, int64_t N, const uint32_t* __restrict__ codes,
              const uint8_t* __restrict__ scales, uint16_t* __restrict__ y) {
    using F = FpFormat<MODE>;
    // launched as the programmatic dependent of the previous kernel: the next
    // product may launch at once; this one waits for the previous grid (which
    // may have written x or the weights) before its first read
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int64_t n = static_cast<int64_t>(blockIdx.x) * kFpRowsPerBlock + (threadIdx.x >> 5);
    if (n >= N) return;
    const int64_t wpr = K * F::BITS / 32;
    const int64_t chunks = wpr / 4;
    const int64_t groups = K / F::GS;
    constexpr int PARTS = F::CPC / F::GS > 0 ? F::CPC / F::GS : 1;  // scale groups per chunk
    constexpr int CODES_PART = F::CPC / PARTS;                      // codes per part
    const uint4* crow = reinterpret_cast<const uint4*>(codes + n * wpr);
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    for (int64_t c = lane; c < chunks; c += 32) {
        const uint4 q4 = ldg_stream(crow + c);
        const uint32_t q[4] = {q4.x, q4.y, q4.z, q4.w};
        const int64_t k0 = c * F::CPC;
        // the chunk's activations, 16 bytes at a time: xr[m][i] = x[m, k0 + 2i .. 2i + 1]
        uint32_t xr[MT][F::CPC / 2];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
#pragma unroll
            for (int v = 0; v < F::CPC / 8; ++v) {
                uint4 xv = make_uint4(0u, 0u, 0u, 0u);
                if (m < M) xv = __ldg(reinterpret_cast<const uint4*>(x + m * K + k0) + v);
                xr[m][4 * v] = xv.x; xr[m][4 * v + 1] = xv.y; xr[m][4 * v + 2] = xv.z; xr[m][4 * v + 3] = xv.w;
            }
        }
#pragma unroll
        for (int part = 0; part < PARTS; ++part) {
            const float S = scale_f32<MODE>(__ldg(scales + n * groups + (k0 + part * CODES_PART) / F::GS));
            float partial[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) partial[m] = 0.f;
            // the part's codes, two at a time, in k order
#pragma unroll
            for (int pr = 0; pr < CODES_PART / 2; ++pr) {
                const int ci = part * CODES_PART + 2 * pr;  // first code of the pair in the chunk
                const uint32_t word = q[ci / F::PER];
                const int jp = (ci % F::PER) / 2;
                const uint32_t h = F::BITS == 4 ? e2m1x2_f16x2((word >> (8 * jp)) & 255u)
                                                : e4m3x2_f16x2((word >> (16 * jp)) & 0xFFFFu);
                float e0, e1;
                f16x2_f32(h, e0, e1);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint32_t xv = xr[m][ci / 2];
                    partial[m] = fmaf(__uint_as_float(xv << 16), e0, partial[m]);
                    partial[m] = fmaf(__uint_as_float(xv & 0xFFFF0000u), e1, partial[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = fmaf(S, partial[m], acc[m]);
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
            if (m < M) y[m * N + n] = f32_to_bf16_bits(acc[m]);
    }
}

template <int MODE>
cudaError_t launch_qmv_fp(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                          const uint8_t* scales, void* y, cudaStream_t s) {
    const unsigned blocks = static_cast<unsigned>((N + kFpRowsPerBlock - 1) / kFpRowsPerBlock);
    const auto* xp = static_cast<const uint16_t*>(x);
    auto* yp = static_cast<uint16_t*>(y);
    const int m = static_cast<int>(M);
    void (*k)(const uint16_t*, int, int64_t, int64_t, const uint32_t*, const uint8_t*, uint16_t*) =
        M <= 1 ? qmv_fp_kernel<MODE, 1> : M <= 2 ? qmv_fp_kernel<MODE, 2> : M <= 4 ? qmv_fp_kernel<MODE, 4>
                                                                              : qmv_fp_kernel<MODE, 8>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3(kFpRowsPerBlock * 32, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, xp, m, K, N, codes, scales, yp);
}

int fp_group(int mode) { return mode == kNv4 ? 16 : 32; }
bool valid_mode(int mode) { return mode == kMx4 || mode == kMx8 || mode == kNv4; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int grid_for(int64_t items, int threads) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t b = (items + threads - 1) / threads;
    return static_cast<int>(b < 8 * sms ? (b > 0 ? b : 1) : 8 * sms);
}

}  // namespace

bool qmm_fp_tiled_supported(int64_t K, int mode);
cudaError_t launch_tc_qmm_fp(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                             const uint8_t* scales, int mode, void* y, cudaStream_t stream, int num_sms);

}  // namespace nvq

extern "C" {

nv_status nv_quantize_fp(const void* w, nv_dtype dt, int64_t rows, int64_t cols, nv_fp_mode mode,
                         uint32_t* codes, uint8_t* scales, nv_stream_t stream) {
    if (!nvq::valid_mode(mode)) return NV_ERR_INVALID_ARG;
    if (dt != NV_F32 && dt != NV_BF16) return NV_ERR_UNSUPPORTED;
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return NV_ERR_INVALID_ARG;
    if (rows == 0) return NV_OK;
    if (!w || !codes || !scales) return NV_ERR_INVALID_ARG;
    if (!nvq::aligned16(w) || !nvq::aligned16(codes)) return NV_ERR_INVALID_ARG;
    const int64_t groups = rows * (cols / nvq::fp_group(mode));
    const int grid = nvq::grid_for(groups, 128);
    cudaStream_t s = stream;
    switch (mode) {
        case NV_MXFP4: nvq::quantize_fp_kernel<nvq::kMx4><<<grid, 128, 0, s>>>(w, dt, rows, cols, codes, scales); break;
        case NV_MXFP8: nvq::quantize_fp_kernel<nvq::kMx8><<<grid, 128, 0, s>>>(w, dt, rows, cols, codes, scales); break;
        case NV_NVFP4: nvq::quantize_fp_kernel<nvq::kNv4><<<grid, 128, 0, s>>>(w, dt, rows, cols, codes, scales); break;
    }
    return cudaGetLastError() == cudaSuccess ? NV_OK : NV_ERR_CUDA;
}

nv_status nv_dequantize_fp(const uint32_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                           nv_fp_mode mode, void* out, nv_stream_t stream) {
    if (!nvq::valid_mode(mode)) return NV_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return NV_ERR_INVALID_ARG;
    if (rows == 0) return NV_OK;
    if (!codes || !scales || !out) return NV_ERR_INVALID_ARG;
    if (!nvq::aligned16(codes) || !nvq::aligned16(out)) return NV_ERR_INVALID_ARG;
    const int64_t words = rows * cols * (mode == NV_MXFP8 ? 8 : 4) / 32;
    const int grid = nvq::grid_for(words, 256);
    cudaStream_t s = stream;
    auto* o = static_cast<uint16_t*>(out);
    switch (mode) {
        case NV_MXFP4: nvq::dequantize_fp_kernel<nvq::kMx4><<<grid, 256, 0, s>>>(codes, scales, rows, cols, o); break;
        case NV_MXFP8: nvq::dequantize_fp_kernel<nvq::kMx8><<<grid, 256, 0, s>>>(codes, scales, rows, cols, o); break;
        case NV_NVFP4: nvq::dequantize_fp_kernel<nvq::kNv4><<<grid, 256, 0, s>>>(codes, scales, rows, cols, o); break;
    }
    return cudaGetLastError() == cudaSuccess ? NV_OK : NV_ERR_CUDA;
}

nv_status nv_qmm_fp(const void* x, nv_dtype dt, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                    const uint8_t* scales, nv_fp_mode mode, void* y, nv_stream_t stream) {
    if (!nvq::valid_mode(mode)) return NV_ERR_INVALID_ARG;
    if (dt != NV_BF16) return NV_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return NV_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return NV_OK;
    if (!x || !codes || !scales || !y) return NV_ERR_INVALID_ARG;
    if (!nvq::aligned16(x) || !nvq::aligned16(codes) || !nvq::aligned16(y)) return NV_ERR_INVALID_ARG;
    cudaStream_t s = stream;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (M > NV_ROW_INDEPENDENT_ROWS && nvq::qmm_fp_tiled_supported(K, mode)) {
        const cudaError_t e = nvq::launch_tc_qmm_fp(x, M, K, N, codes, scales, mode, y, s, sms);
        return e == cudaSuccess ? NV_OK : NV_ERR_CUDA;
    }
    // rows in chunks of up to 8 (each row's arithmetic is the same in any chunk)
    for (int64_t m0 = 0; m0 < M; m0 += NV_ROW_INDEPENDENT_ROWS) {
        const int64_t mc = M - m0 < NV_ROW_INDEPENDENT_ROWS ? M - m0 : NV_ROW_INDEPENDENT_ROWS;
        const void* xm = static_cast<const uint16_t*>(x) + m0 * K;
        void* ym = static_cast<uint16_t*>(y) + m0 * N;
        cudaError_t e = cudaSuccess;
        switch (mode) {
            case NV_MXFP4: e = nvq::launch_qmv_fp<nvq::kMx4>(xm, mc, K, N, codes, scales, ym, s); break;
            case NV_MXFP8: e = nvq::launch_qmv_fp<nvq::kMx8>(xm, mc, K, N, codes, scales, ym, s); break;
            case NV_NVFP4: e = nvq::launch_qmv_fp<nvq::kNv4>(xm, mc, K, N, codes, scales, ym, s); break;
        }
        if (e != cudaSuccess) return NV_ERR_CUDA;
    }
    return NV_OK;
}

}  // extern "C"
