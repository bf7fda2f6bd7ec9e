// Device helpers shared by the tcgen05 kernels (sm_100a): tensor-core fences,
// MMA issue and commit, shared-memory / instruction descriptors, bf16 pair
// arithmetic, and the code -> bf16 weight dequantizers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "tma.cuh"

namespace nvq {

// A bounded wait (as mbar_wait) for waits expected to be long (an epilogue waiting
// for a whole tile's accumulation, a producer waiting for a free stage): after
// the first failed poll the thread sleeps between polls, doubling the sleep up
// to max_ns, so that it takes almost no issue slots from the working warps.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, unsigned code,
                                                  uint32_t max_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    uint32_t ns = 32;
    for (;;) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        ns = ns * 2 < max_ns ? ns * 2 : max_ns;
        if (globaltimer() - t0 > kWaitLimitNs) {
            atomicCAS(&g_pipeline_error, 0u, code);
            return false;
        }
    }
}

namespace tc {

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same MMA with A read from tensor memory (M rows = TMEM lanes, two 16-bit
// K elements per 32-bit column, the lower K in the low half).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Store 8 consecutive 32-bit columns of this thread's TMEM lane (warp w may
// address lanes 32 (w % 4) .. 32 (w % 4) + 31), then wait for the store.
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// tcgen05.st without the wait: complete it (with any other stores of the
// thread) by tmem_st_wait before the stored columns are read.
__device__ __forceinline__ void tmem_st_x16_async(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes stacked along M/N (stride 1024), Blackwell descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(const void* p) {
    const uint64_t addr = smem_u32(p);
    return ((addr & 0x3FFFFull) >> 4) | (1ull << 16) | (static_cast<uint64_t>(1024 >> 4) << 32) |
           (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

// Block of 8 groups that k-step ks starts in (sgk k-steps per block).
__device__ __forceinline__ int blk_in_tile(int ks, int sgk) { return ks / sgk; }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
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

// ---------------------------------------------------------------- dequantizer
__device__ __forceinline__ uint32_t shr(uint32_t w, uint32_t bits) { return w >> bits; }

// One word of codes -> bf16 weights w = s * c + b for consecutive k, written
// as 32-bit pairs out[0..PAIRS). s2 / b2: bf16x2 (s, s) and (b, b); m2/m4/m6:
// the shift counts 2, 4, 6.
template <int BITS>
struct Dequant;

// run_fast (s a normal number below 2^-5, see dq_fast_ok): a 16-bit pattern
// below 0x100 read as a bf16 is exactly pattern * 2^-133 (subnormals and the
// lowest binade form one linear scale), so a code field masked in place at
// bits p .. p + bits - 1 of a half is c * 2^(p - 133), and the bf16 fma takes
// s * 2^(133 - p) for that half, formed by adding 133 - p to s's exponent
// (exact, finite since s < 2^-5). The product is the same real number s * c
// as in run, so both round to the same bf16 w = s * c + b.
__device__ __forceinline__ bool dq_fast_ok(uint32_t s2) {
    return ((s2 >> 7) & 0xFFu) - 1u < 121u;  // biased exponent 1 .. 121
}

template <>
struct Dequant<4> {  // word: 8 codes -> 4 pairs
    static constexpr int PAIRS = 4;
    __device__ static __forceinline__ void run_fast(uint32_t w, uint32_t s2, uint32_t b2, uint32_t* out) {
        const uint32_t m = s2 + 0x40804280u;  // (s * 2^133, s * 2^129)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // byte i into bytes 0 and 2: code 2i at bits 0-3, code 2i+1 at bits 20-23
            const uint32_t r = prmt(w, w, i | (i << 8)) & 0x00F0000Fu;
            out[i] = bf2_fma(m, r, b2);
        }
    }
    __device__ static __forceinline__ void run(uint32_t w, uint32_t s2, uint32_t b2, float,
                                               float, uint32_t, uint32_t m4, uint32_t,
                                               uint32_t* out) {
        const uint32_t v = shr(w, m4);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // bytes (w.byte_i, -, v.byte_i, -): low nibbles are codes 2i and 2i+1
            const uint32_t sel = i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12);
            const uint32_t r = codes_to_bf16x2(prmt(w, v, sel), 0x000F000Fu);  // 128 + c
            out[i] = bf2_fma(s2, bf2_sub(r, 0x43004300u), b2);
        }
    }
};

template <>
struct Dequant<2> {  // word: 16 codes -> 8 pairs
    static constexpr int PAIRS = 8;
    __device__ static __forceinline__ void run_fast(uint32_t w, uint32_t s2, uint32_t b2, uint32_t* out) {
        const uint32_t m01 = s2 + 0x41804280u;  // fields at bits 0-1 / 2-3: (s * 2^133, s * 2^131)
        const uint32_t m23 = s2 + 0x3F804080u;  // fields at bits 4-5 / 6-7: (s * 2^129, s * 2^127)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t r = prmt(w, w, i | (i << 8));  // byte i in both halves
            out[2 * i] = bf2_fma(m01, r & 0x000C0003u, b2);      // codes 4i, 4i+1
            out[2 * i + 1] = bf2_fma(m23, r & 0x00C00030u, b2);  // codes 4i+2, 4i+3
        }
    }
    __device__ static __forceinline__ void run(uint32_t w, uint32_t s2, uint32_t b2, float,
                                               float, uint32_t m2, uint32_t m4, uint32_t m6,
                                               uint32_t* out) {
        const uint32_t v1 = shr(w, m2), v2 = shr(w, m4), v3 = shr(w, m6);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t sel = i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12);
            const uint32_t r0 = codes_to_bf16x2(prmt(w, v1, sel), 0x00030003u);   // codes 4i, 4i+1
            const uint32_t r1 = codes_to_bf16x2(prmt(v2, v3, sel), 0x00030003u);  // codes 4i+2, 4i+3
            out[2 * i] = bf2_fma(s2, bf2_sub(r0, 0x43004300u), b2);
            out[2 * i + 1] = bf2_fma(s2, bf2_sub(r1, 0x43004300u), b2);
        }
    }
};

// Packed fp32 pairs (sm_100a): d = a * b + c on both halves, one rounding each.
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_pack(uint32_t lo, uint32_t hi) {
    return (static_cast<uint64_t>(hi) << 32) | lo;
}
// (lo, hi) fp32 pair -> bf16x2, round to nearest even.
__device__ __forceinline__ uint32_t f2_to_bf2_packed(uint64_t v) {
    uint32_t d;
    asm("{\n\t.reg .f32 lo, hi;\n\tmov.b64 {lo, hi}, %1;\n\tcvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
        : "=r"(d) : "l"(v));
    return d;
}

template <>
struct Dequant<8> {  // word: 4 codes -> 2 pairs, through exact fp32 codes in packed pairs
    static constexpr int PAIRS = 2;
    __device__ static __forceinline__ void run_fast(uint32_t w, uint32_t s2, uint32_t b2, uint32_t* out) {
        const uint32_t m = s2 + 0x42804280u;  // (s * 2^133, s * 2^133)
#pragma unroll
        for (int i = 0; i < 2; ++i)  // bytes 2i, 2i + 1 into bytes 0 and 2, zeros elsewhere
            out[i] = bf2_fma(m, prmt(w, 0u, (2 * i) | (4 << 4) | ((2 * i + 1) << 8) | (4 << 12)), b2);
    }
    __device__ static __forceinline__ void run(uint32_t w, uint32_t, uint32_t, float s, float b,
                                               uint32_t, uint32_t, uint32_t, uint32_t* out) {
        const uint64_t one_m = f2_pack(0x3F800000u, 0x3F800000u);   // (1, 1)
        const uint64_t off = f2_pack(0xCB000000u, 0xCB000000u);     // (-2^23, -2^23)
        const uint64_t s2 = f2_pack(__float_as_uint(s), __float_as_uint(s));
        const uint64_t b2 = f2_pack(__float_as_uint(b), __float_as_uint(b));
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            // bytes 2i, 2i + 1 under the mantissa of 2^23: 2^23 + c, exact
            const uint64_t r = f2_pack(prmt(w, 0x4B000000u, (2 * i) | 0x7440),
                                       prmt(w, 0x4B000000u, (2 * i + 1) | 0x7440));
            const uint64_t c = f2_fma(r, one_m, off);                  // c, exact
            out[i] = f2_to_bf2_packed(f2_fma(s2, c, b2));              // s * c + b
        }
    }
};

}  // namespace tc
}  // namespace nvq
