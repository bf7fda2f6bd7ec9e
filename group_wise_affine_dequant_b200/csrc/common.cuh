// Shared device helpers of the nvq library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/nvq.h"

namespace nvq {

constexpr int kRowIndependentRows = NV_ROW_INDEPENDENT_ROWS;

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h16) {
    return __uint_as_float(h16 << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int64_t i) {
    if constexpr (DT == NV_F32) {
        return __ldg(reinterpret_cast<const float*>(p) + i);
    } else {
        return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short*>(p) + i));
    }
}

template <int DT>
__device__ __forceinline__ void store_elem(void* p, int64_t i, float v) {
    if constexpr (DT == NV_F32) {
        reinterpret_cast<float*>(p)[i] = v;
    } else {
        reinterpret_cast<unsigned short*>(p)[i] = f32_to_bf16_bits(v);
    }
}

// Warp-level mma m16n8k16, bf16 inputs, fp32 accumulate: d = a . b + d.
// Fragment ownership (lane = 4 * g + t): a0 (row g, k 2t..2t+1), a1 (row g+8,
// k 2t..2t+1), a2 (row g, k 2t+8..2t+9), a3 (row g+8, k 2t+8..2t+9); b0 (k
// 2t..2t+1, col g), b1 (k 2t+8..2t+9, col g); d0 (g, 2t), d1 (g, 2t+1),
// d2 (g+8, 2t), d3 (g+8, 2t+1).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with fp16 inputs.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two bf16 values (lo, hi) from halves of two 32-bit words.
__device__ __forceinline__ uint32_t pair_lo(uint32_t a, uint32_t b) {
    return __byte_perm(a, b, 0x5410);  // (a.lo, b.lo)
}
__device__ __forceinline__ uint32_t pair_hi(uint32_t a, uint32_t b) {
    return __byte_perm(a, b, 0x7632);  // (a.hi, b.hi)
}

// bf16x2 (128 + c_lo, 128 + c_hi) from two code fields at bits [0, n) and
// [16, 16 + n) of v: OR-ing an integer below 128 into the mantissa of 128.0
// (0x4300) gives exactly 128 + c, since bf16's unit in the last place at 128 is 1.
__device__ __forceinline__ uint32_t codes_to_bf16x2(uint32_t v, uint32_t mask) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(mask), "r"(0x43004300u));
    return r;  // (v & mask) | 0x43004300
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace nvq
