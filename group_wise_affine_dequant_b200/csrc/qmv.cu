// Quantized matrix-vector products for 1 to 8 rows of bf16 activations,
// weights stored [N, K] ("Docs / Quantization", sections "Affine" and "Products
// on the GPU": small row counts go to matrix-vector kernels, and every weight
// group is read once however many rows there are).
//
// Design (sm_100a):
//  * The weights stream from HBM exactly once per call, by TMA: each warp
//    copies its slice of 16 rows per tile (one 2-D tensor copy, 128-byte
//    swizzle so the fragment reads below hit distinct banks) plus the slice's
//    scales and biases into its own ring of shared-memory stages, completing
//    on a per-warp mbarrier, several tiles ahead of the math.
//  * Every weight is dequantized in registers to bf16 w = scale * code + bias,
//    the exact value rounded once (one bf16 fused multiply-add on the code
//    held as an exact bf16 number; 8-bit codes through one fp32 fma and a
//    conversion), exactly as the tiled kernels do. Codes become exact bf16
//    with one mask each: OR-ing a field worth c * 2^p <= 127 into the mantissa
//    of 128.0 gives 128 + c * 2^p, then 128 is subtracted; a 2-bit field held
//    as c * 4^j meets the scale divided by 4^j (exact).
//  * The multiply-adds run on the tensor cores (mma.sync m16n8k16, bf16 in,
//    fp32 accumulate): A = 16 weight rows x 16 k of weights, B = the
//    activations (one column per activation row, up to 8). Which physical k
//    feeds which MMA k-slot is chosen so that each thread's loaded words feed
//    its own A fragments; the activations are permuted the same way once, in
//    registers.
//  * Activations enter the MMA as bf16, the type they arrive in: bf16 has the
//    exponent range of fp32, so no value is rounded or flushed on the way in.
//    Only a slice whose largest magnitude reaches 2^100 is first multiplied by
//    2^-(e - 100) (e its exponent), which keeps the fp32 sums finite, and its
//    partial sums are multiplied back by 2^(e - 100); both steps are exact.
//    Every product of an activation and a dequantized weight is exact in
//    fp32: the only roundings are the weights' (relative 2^-9) and the fp32
//    sums', so the error is bounded by a small multiple of sum_k |x_k w_k|
//    for every finite input.
//  * A warp owns a k-slice of 16 MMA k-steps (256 k at 2/4 bits, 128 at 8) and
//    keeps its activations in registers while it walks the rows of its CTA.
//    Each CTA owns a contiguous range of rows (N split evenly over the SMs) and
//    reduces the slices in a fixed order through shared memory.
//  * Every output (row n, activation row m) is computed by the same sequence
//    of operations whatever M is, so each row of an M-row call is bitwise equal
//    to a call with that row alone (row exactness, nuvec crate docs,
//    "Determinism").
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace nvq {
namespace {

// MMA k-steps per warp slice (16: a warp's activation fragments take 32
// registers) and warps per CTA (16 x 128 registers fill the register file).
// Measured on B200: 8-step slices with 32 warps of 64 registers ran slower.
constexpr int kSteps = 16;
constexpr int kMaxWarps = 16;

template <int BITS, int GS, int STEPS = (BITS == 8 ? kSteps / 2 : kSteps)>
struct Shape {
    static constexpr int PER = 32 / BITS;                // codes per word
    static constexpr int GW = GS * BITS / 32;            // words per group
    static constexpr int LW = GW / 4 < 4 ? GW / 4 : 4;   // words per thread per row per chunk
    static constexpr int MPW = BITS == 2 ? 4 : BITS == 4 ? 2 : 1;  // MMAs per word
    static constexpr int NP = 2 * MPW;                   // fp16x2 registers per unpacked word
    static constexpr int CW = 4 * LW;                    // words per chunk (one lane quad)
    static constexpr int CK = CW * PER;                  // k per chunk
    static constexpr int MMAS = LW * MPW;                // MMAs per chunk
    static constexpr int KS = STEPS / MMAS > 0 ? STEPS / MMAS : 1;  // chunks per warp slice
    static constexpr int KSLICE = KS * CK;               // k per warp slice
    static constexpr int GPS = KSLICE / GS > 0 ? KSLICE / GS : 1;  // groups per slice
    static constexpr int CPG = GS / CK;                  // chunks per group
    static_assert(LW >= 1, "group too small for this kernel");
    static_assert(CK <= GS && GS % CK == 0, "a chunk lies inside one group");
};

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

// A group's scale and bias for one weight row, ready for the dequantizers:
// (s, s) and (b, b) as bf16 pairs, taken from a word holding two groups'
// values (half i & 1), and whether the fast dequantizer applies.
struct GroupSB {
    uint32_t s2, b2;
    bool fast;
};
__device__ __forceinline__ GroupSB group_sb(uint32_t sv, uint32_t bv, int i) {
    GroupSB g;
    const uint32_t sel = (i & 1) ? 0x3232u : 0x1010u;
    g.s2 = __byte_perm(sv, 0u, sel);
    g.b2 = __byte_perm(bv, 0u, sel);
    // s normal and below 2^-5: biased exponent 1 .. 121
    g.fast = ((g.s2 >> 7) & 0xFFu) - 1u < 121u;
    return g;
}

// Word -> NP bf16x2 registers of dequantized weights; MMA u of the word uses
// p[2u] (k-slots 2t, 2t+1) and p[2u+1] (k-slots 2t+8, 2t+9). lo(i), hi(i):
// the codes of the word behind register i's low and high halves.
//
// Two exact forms of w = s * c + b, rounded once to bf16 (one bf16 fma):
//  * run: OR-ing a field worth c * 2^p <= 127 into the mantissa of 128.0
//    gives 128 + c * 2^p; 128 is subtracted (exact) and the fma takes s (or
//    s / 2^p, exact for these powers of two).
//  * run_fast (s a normal number below 2^-5): a 16-bit pattern below 0x100
//    read as a bf16 is exactly pattern * 2^-133 (subnormals and the lowest
//    binade are one linear scale), so a field masked in place is
//    c * 2^(p - 133) with no subtraction, and the fma takes s * 2^(133 - p),
//    formed by adding 133 - p to s's exponent (exact, and finite because s
//    is below 2^-5). The product is the same real number s * c, so both
//    forms round to the same bf16.
template <int BITS>
struct Dequant;

template <>
struct Dequant<4> {  // (c0,c4) (c1,c5) (c2,c6) (c3,c7)
    __host__ __device__ static constexpr int lo(int i) { return i; }
    __host__ __device__ static constexpr int hi(int i) { return i + 4; }
    __device__ static __forceinline__ void run(uint32_t w, const GroupSB& g, uint32_t* p) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            p[i] = bf2_fma(g.s2, bf2_sub(codes_to_bf16x2(w >> (4 * i), 0x000F000Fu), 0x43004300u), g.b2);
    }
    __device__ static __forceinline__ void run_fast(uint32_t w, const GroupSB& g, uint32_t* p) {
        const uint32_t s0 = g.s2 + 0x42804280u;  // s * 2^133: fields at bits 0-3
        const uint32_t s1 = g.s2 + 0x40804080u;  // s * 2^129: fields at bits 4-7
        const uint32_t v = w >> 8;
        p[0] = bf2_fma(s0, w & 0x000F000Fu, g.b2);
        p[1] = bf2_fma(s1, w & 0x00F000F0u, g.b2);
        p[2] = bf2_fma(s0, v & 0x000F000Fu, g.b2);
        p[3] = bf2_fma(s1, v & 0x00F000F0u, g.b2);
    }
};

template <>
struct Dequant<2> {  // (c_i, c_i+8), fields held as c * (1, 4, 16, 1, 4, 16, 1, 4)
    __host__ __device__ static constexpr int lo(int i) { return i; }
    __host__ __device__ static constexpr int hi(int i) { return i + 8; }
    __device__ static __forceinline__ void run(uint32_t w, const GroupSB& g, uint32_t* p) {
        // s / 4 and s / 16 for fields held as c * 4 and c * 16 (exact)
        const float sf = __uint_as_float(g.s2 << 16);
        const uint32_t s2q = (__float_as_uint(sf * 0.25f) >> 16) * 0x00010001u;
        const uint32_t s2h = (__float_as_uint(sf * 0.0625f) >> 16) * 0x00010001u;
        const uint32_t v = w >> 6, u = w >> 12;
        const uint32_t r[8] = {codes_to_bf16x2(w, 0x00030003u), codes_to_bf16x2(w, 0x000C000Cu),
                               codes_to_bf16x2(w, 0x00300030u), codes_to_bf16x2(v, 0x00030003u),
                               codes_to_bf16x2(v, 0x000C000Cu), codes_to_bf16x2(v, 0x00300030u),
                               codes_to_bf16x2(u, 0x00030003u), codes_to_bf16x2(u, 0x000C000Cu)};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t s2 = (i % 3) == 0 ? g.s2 : (i % 3) == 1 ? s2q : s2h;
            p[i] = bf2_fma(s2, bf2_sub(r[i], 0x43004300u), g.b2);
        }
    }
    __device__ static __forceinline__ void run_fast(uint32_t w, const GroupSB& g, uint32_t* p) {
        // fields at bits 0-1, 2-3, 4-5, 6-7 of each half: s * 2^133, 2^131, 2^129, 2^127
        const uint32_t m[4] = {g.s2 + 0x42804280u, g.s2 + 0x41804180u, g.s2 + 0x40804080u,
                               g.s2 + 0x3F803F80u};
        const uint32_t v = w >> 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            p[i] = bf2_fma(m[i], w & (0x00030003u << (2 * i)), g.b2);
            p[i + 4] = bf2_fma(m[i], v & (0x00030003u << (2 * i)), g.b2);
        }
    }
};

template <>
struct Dequant<8> {  // (c0,c2) (c1,c3)
    __host__ __device__ static constexpr int lo(int i) { return i; }
    __host__ __device__ static constexpr int hi(int i) { return i + 2; }
    __device__ static __forceinline__ void run(uint32_t w, const GroupSB& g, uint32_t* p) {
        // packed fp32 pairs: byte k under the mantissa of 2^23 is 2^23 + c_k;
        // one fma removes the 2^23 (exact), one applies scale and bias, and
        // the sum is converted once to bf16
        const uint64_t one = 0x3F8000003F800000ull, off = 0xCB000000CB000000ull;
        const uint32_t sf = g.s2 << 16, bf = g.b2 << 16;
        const uint64_t s2 = (static_cast<uint64_t>(sf) << 32) | sf;
        const uint64_t b2 = (static_cast<uint64_t>(bf) << 32) | bf;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint64_t r = (static_cast<uint64_t>(__byte_perm(w, 0x4B000000u, 0x7640 | hi(i))) << 32) |
                               __byte_perm(w, 0x4B000000u, 0x7640 | lo(i));
            uint64_t c, f;
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(c) : "l"(r), "l"(one), "l"(off));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(f) : "l"(s2), "l"(c), "l"(b2));
            asm("{\n\t.reg .f32 lo, hi;\n\tmov.b64 {lo, hi}, %1;\n\tcvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
                : "=r"(p[i]) : "l"(f));
        }
    }
    __device__ static __forceinline__ void run_fast(uint32_t w, const GroupSB& g, uint32_t* p) {
        const uint32_t s0 = g.s2 + 0x42804280u;  // s * 2^133: bytes at bits 0-7
        p[0] = bf2_fma(s0, w & 0x00FF00FFu, g.b2);
        p[1] = bf2_fma(s0, (w >> 8) & 0x00FF00FFu, g.b2);
    }
};

__device__ __forceinline__ float bf16_elem(const uint32_t* xv, int i) {
    return __uint_as_float((i & 1) ? (xv[i >> 1] & 0xFFFF0000u) : (xv[i >> 1] << 16));
}
__device__ __forceinline__ uint32_t f2_to_bf2x(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// The activations matching Dequant: b[u][0..1] for MMA u of a word whose first
// k is k0, from xv = x[k0 .. k0 + PER) as bf16 pairs, times f (a power of
// two: exact).
template <int BITS>
__device__ __forceinline__ void x_fragments(const uint32_t* xv, float f, uint32_t (*b)[2]) {
    using D = Dequant<BITS>;
#pragma unroll
    for (int i = 0; i < 2 * (BITS == 2 ? 4 : BITS == 4 ? 2 : 1); ++i)
        b[i >> 1][i & 1] = f2_to_bf2x(bf16_elem(xv, D::lo(i)) * f, bf16_elem(xv, D::hi(i)) * f);
}


struct QmvParams {
    const uint16_t* x;       // bf16 [x_rows, K]
    const uint32_t* codes;   // [E][N, K*bits/32]
    const uint16_t* scales;  // [E][N, K/gs]
    const uint16_t* biases;
    uint16_t* y;             // bf16 [*, N]
    int64_t N, K;
    int M;                   // rows (plain product)
    int ctas_per_problem;    // G: CTAs along N; CTA c takes tiles_q + (c < tiles_r) 16-row tiles
    int tiles_q, tiles_r;    // T / G and T % G, T = ceil(N / 16)
    int rows_cap;            // max rows of one CTA, multiple of 16
    int rows_max;            // max rows of one CTA (height of the scale/bias block)
    // Scales and biases: 2 = the CTA's whole block by TMA once (nbox boxes of
    // 2^sbw_log-byte rows along the groups, each in a `region`-byte area,
    // swizzled like the code tiles); 1 = per tile with the codes; 0 = loads.
    int sb_mode;
    int sbw_log, nbox;
    uint32_t region;
    uint32_t off_sb, off_bar, off_red;  // shared-memory layout (bytes)
    // gather only
    const uint32_t* lhs;     // nullable
    const uint32_t* perm;
    const uint32_t* problems;      // [P][4] = (expert, start, count, 0)
    const uint32_t* num_problems;
    int64_t E;
    uint32_t problem0;       // problem of blockIdx.y = 0 (launches of <= 65535 problems)
};


// Ring geometry of one warp: per stage, the code box (16 rows x CBYTES, TMA
// 128-byte swizzle when CBYTES is 128) and the scale and bias boxes (16 rows x
// SBOX bf16, unswizzled). Code stages are 1024-byte aligned.
template <int BITS, int GS>
struct Ring {
    using S = Shape<BITS, GS>;
    static constexpr int CBYTES = S::KSLICE * BITS / 8;          // code bytes per row and slice
    static constexpr bool SWZ = CBYTES >= 32;   // TMA swizzle span = row bytes (32/64/128)
    static constexpr int CODE_STAGE = 16 * CBYTES;               // 2048 or 1024
    static constexpr int SBOX = S::GPS > 8 ? S::GPS : 8;         // groups per scale box row
    static constexpr int SB_STAGE = 16 * SBOX * 2;               // one of scales / biases
    // byte offset of code word `word` of row `r` inside a code stage
    __device__ static __forceinline__ uint32_t code_off(int r, int word) {
        const uint32_t o = static_cast<uint32_t>(word) * 4;
        if constexpr (CBYTES == 128) return r * 128 + ((((o >> 4) ^ (r & 7)) << 4) | (o & 15));
        else if constexpr (CBYTES == 64) return r * 64 + ((((o >> 4) ^ ((r >> 1) & 3)) << 4) | (o & 15));
        else if constexpr (CBYTES == 32) return r * 32 + ((((o >> 4) ^ ((r >> 2) & 1)) << 4) | (o & 15));
        else return r * CBYTES + o;
    }
};

// Byte offset of group column `gc` of row `r` inside one scale/bias box region
// with rows of 2^sbw_log bytes, under the TMA swizzle of that row width.
__device__ __forceinline__ uint32_t sb_block_off(int r, int gc, int sbw_log) {
    const uint32_t o = static_cast<uint32_t>(gc) * 2;
    uint32_t c = o >> 4;
    if (sbw_log == 7) c ^= r & 7;
    else if (sbw_log == 6) c ^= (r >> 1) & 3;
    else if (sbw_log == 5) c ^= (r >> 2) & 1;
    return (static_cast<uint32_t>(r) << sbw_log) + (c << 4) + (o & 15);
}

template <int LW>
__device__ __forceinline__ void lds_words(const uint8_t* p, uint32_t* w) {
    if constexpr (LW == 1) {
        w[0] = *reinterpret_cast<const uint32_t*>(p);
    } else if constexpr (LW == 2) {
        uint2 v = *reinterpret_cast<const uint2*>(p);
        w[0] = v.x; w[1] = v.y;
    } else {
        uint4 v = *reinterpret_cast<const uint4*>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    }
}

// One lane of the warp, chosen by the hardware (all lanes must take part).
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n}"
        : "=r"(pred));
    return pred != 0;
}

// M1: the call has one activation row (only column 0 of the MMA is live). The
// arithmetic of every stored output is the same as in the general form.
template <int BITS, int GS, bool GATHER, int NS, bool M1>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
qmv_kernel(const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_s,
           const __grid_constant__ CUtensorMap map_b, const QmvParams prm) {
    using S = Shape<BITS, GS>;
    using RG = Ring<BITS, GS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ int64_t s_xrow[8];
    __shared__ int64_t s_yrow[8];

    const int lane = threadIdx.x & 31;
    // warp index as a warp-uniform value, so that the TMA operands derived from
    // it stay in uniform registers
    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
    const int nwarps = blockDim.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t N = prm.N, K = prm.K;
    const int64_t gpr = K / GS;  // groups per row

    // shared memory: [warps][NS] code stages | scale+bias block (mode 2) or
    // [warps][NS] scale+bias stages (mode 1) | [warps][NS] + 1 mbarriers |
    // slice partials
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prm.off_bar);
    uint64_t* full = bars + warp * NS;
    uint64_t* sb_full = bars + nwarps * NS;
    // The barriers live in this CTA's shared memory only, so they are set up
    // before the wait for the previous kernel (made visible by the barrier
    // below, before any use).
    if (lane == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
        if (warp == 0) mbar_init(sb_full, 1);
        mbar_init_fence();
    }

    int M;
    const uint16_t* scales = prm.scales;
    const uint16_t* biases = prm.biases;
    bool zero_problem = false;
    int expert = 0;
    pdl_launch_dependents();
    if constexpr (GATHER) {
        pdl_wait();  // the routing tables come from the previous kernel
        const uint32_t p = prm.problem0 + blockIdx.y;
        if (p >= __ldg(prm.num_problems)) return;
        const uint32_t e = __ldg(prm.problems + 4 * p);
        const uint32_t start = __ldg(prm.problems + 4 * p + 1);
        M = static_cast<int>(__ldg(prm.problems + 4 * p + 2));
        zero_problem = e >= prm.E;  // pairs with an invalid id get zeros
        if (!zero_problem) {
            expert = static_cast<int>(e);
            scales += static_cast<int64_t>(e) * N * gpr;
            biases += static_cast<int64_t>(e) * N * gpr;
        }
        if (threadIdx.x < M) {
            const uint32_t pair = __ldg(prm.perm + start + threadIdx.x);
            s_yrow[threadIdx.x] = pair;
            s_xrow[threadIdx.x] = prm.lhs ? __ldg(prm.lhs + pair) : pair;
        }
    } else {
        // The weights are not written by kernels of this library's stream
        // order that could still run, but the previous kernel may be anything:
        // only L2 prefetches (coherent) touch memory before the wait.
        {
            const int cta = static_cast<int>(blockIdx.x);
            const int r0 = 16 * (cta * prm.tiles_q + min(cta, prm.tiles_r));
            const int nrows = min(16 * (prm.tiles_q + (cta < prm.tiles_r ? 1 : 0)), static_cast<int>(N) - r0);
            const int nsl = static_cast<int>((K + S::KSLICE - 1) / S::KSLICE);
            // the first ring's worth of tiles of the warp's first slice
            // (prefetching everything floods HBM while the previous kernel
            // still streams its own tiles)
            // (every warp's first tile and the scale block first, then the rest)
            const int w = static_cast<int>(threadIdx.x >> 5);
            const bool lead = (threadIdx.x & 31) == 0 && w < nsl;
            const int cw = w * S::KSLICE * BITS / 32;
            const int gb = w * S::KSLICE / GS / RG::SBOX * RG::SBOX;
            for (int phase = 0; phase < 2; ++phase) {
                if (lead) {
                    for (int i = phase; i < (phase ? NS : 1) && i * 16 < nrows; ++i) {
                        tma_prefetch_3d(&map_c, cw, r0 + i * 16, 0);
                        if (prm.sb_mode == 1) {
                            tma_prefetch_3d(&map_s, gb, r0 + i * 16, 0);
                            tma_prefetch_3d(&map_b, gb, r0 + i * 16, 0);
                        }
                    }
                    if (phase == 0 && prm.sb_mode == 2 && w < prm.nbox) {
                        const int gcol = w << (prm.sbw_log - 1);
                        tma_prefetch_3d(&map_s, gcol, r0, 0);
                        tma_prefetch_3d(&map_b, gcol, r0, 0);
                    }
                }
                if (phase == 0) __syncthreads();
            }
        }
        pdl_wait();  // x may come from the previous kernel; y may still be read by it
        M = M1 ? 1 : prm.M;
        if (threadIdx.x < M) {
            s_xrow[threadIdx.x] = threadIdx.x;
            s_yrow[threadIdx.x] = threadIdx.x;
        }
    }
    __syncthreads();

    const int cta = static_cast<int>(blockIdx.x);
    // whole 16-row tiles per CTA (the last CTA's last tile may be partial)
    const int64_t n0 = 16 * (static_cast<int64_t>(cta) * prm.tiles_q + min(cta, prm.tiles_r));
    const int rows = static_cast<int>(
        min(static_cast<int64_t>(16 * (prm.tiles_q + (cta < prm.tiles_r ? 1 : 0))), N - n0));
    const int64_t n1 = n0 + rows;
    if (rows <= 0) return;

    if (zero_problem) {
        for (int i = threadIdx.x; i < rows * M; i += blockDim.x) {
            const int m = i / rows, r = i % rows;
            prm.y[s_yrow[m] * N + n0 + r] = 0;
        }
        return;
    }

    const int sb_mode = prm.sb_mode;
    uint8_t* code_ring = smem + static_cast<size_t>(warp) * NS * RG::CODE_STAGE;
    uint8_t* sb_base = smem + prm.off_sb;
    uint8_t* sb_ring = sb_base + static_cast<size_t>(warp) * NS * 2 * RG::SB_STAGE;
    float* red = reinterpret_cast<float*>(smem + prm.off_red);

    if (sb_mode == 2 && warp == 0 && elect_one()) {
        // the CTA's scales and biases: rows [n0, n0 + rows_max), all groups
        const uint32_t box = static_cast<uint32_t>(prm.rows_max) << prm.sbw_log;
        mbar_expect_tx(sb_full, 2u * prm.nbox * box);
        for (int bi = 0; bi < prm.nbox; ++bi) {
            const int gcol = bi << (prm.sbw_log - 1);
            tma_load_3d(sb_base + bi * prm.region, &map_s, sb_full, gcol, static_cast<int>(n0), expert);
            tma_load_3d(sb_base + (prm.nbox + bi) * prm.region, &map_b, sb_full, gcol,
                        static_cast<int>(n0), expert);
        }
    }

    const int tiles = (rows + 15) / 16;
    const int rows_cap = prm.rows_cap;
    const int nslices = static_cast<int>((K + S::KSLICE - 1) / S::KSLICE);
    const uint32_t stage_bytes = RG::CODE_STAGE + (sb_mode == 1 ? 2 * RG::SB_STAGE : 0);
    const int row0 = static_cast<int>(n0);
    const int MC = M1 ? 1 : M;  // columns kept per row in the slice partials

    // byte offsets of this lane's code words inside a stage (rows g and g + 8)
    uint32_t offa[S::KS], offb[S::KS];
#pragma unroll
    for (int q = 0; q < S::KS; ++q) {
        offa[q] = RG::code_off(g, q * S::CW + t * S::LW);
        offb[q] = RG::code_off(g + 8, q * S::CW + t * S::LW);
    }

    bool ok = true;
    int st = 0;       // ring stage of this warp's next tile
    uint32_t ph = 0;  // and the parity of its current use

    for (int sl = warp; sl < nslices && ok; sl += nwarps) {
        const int kslice0 = sl * S::KSLICE;
        const int g0 = kslice0 / GS;
        const int gbox = g0 / RG::SBOX * RG::SBOX;  // scale box start (16-B aligned)
        const int goff = g0 - gbox;                 // slice's first group in the box
        const int cword = kslice0 * BITS / 32;

        // ---- activations of this slice, loaded before the weight copies are
        // issued (so that these few loads do not queue behind the stream) ----
        uint32_t xall[S::KS][S::LW][S::PER / 2];
#pragma unroll
        for (int q = 0; q < S::KS; ++q) {
            const int64_t kq = static_cast<int64_t>(kslice0) + q * S::CK;
            const bool valid = kq < K && g < M;
#pragma unroll
            for (int j = 0; j < S::LW; ++j) {
                const int64_t k0 = kq + (t * S::LW + j) * S::PER;
                uint32_t* xv = xall[q][j];
                if (valid) {
                    const uint16_t* xp = prm.x + s_xrow[g] * K + k0;
                    if constexpr (S::PER == 4) {
                        uint2 v = __ldg(reinterpret_cast<const uint2*>(xp));
                        xv[0] = v.x; xv[1] = v.y;
                    } else {
#pragma unroll
                        for (int h = 0; h < S::PER / 8; ++h) {
                            uint4 v = __ldg(reinterpret_cast<const uint4*>(xp) + h);
                            xv[4 * h] = v.x; xv[4 * h + 1] = v.y;
                            xv[4 * h + 2] = v.z; xv[4 * h + 3] = v.w;
                        }
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < S::PER / 2; ++h) xv[h] = 0u;
                }
            }
        }

        // one lane: copy tile `tile` of this slice into ring stage `s`
        auto issue = [&](int tile, int s) {
            uint64_t* bar = &full[s];
            mbar_expect_tx(bar, stage_bytes);
            const int row = row0 + tile * 16;
            tma_load_3d(code_ring + s * RG::CODE_STAGE, &map_c, bar, cword, row, expert);
            if (sb_mode == 1) {
                uint8_t* sbs = sb_ring + s * 2 * RG::SB_STAGE;
                tma_load_3d(sbs, &map_s, bar, gbox, row, expert);
                tma_load_3d(sbs + RG::SB_STAGE, &map_b, bar, gbox, row, expert);
            }
        };
        // Fill the ring. On the first slice every warp queues its first tile,
        // then (after a CTA barrier) the rest, so that the SM's copy queue
        // holds every warp's first tile ahead of any second tile.
        const bool first_slice = sl == warp;
        if (elect_one()) issue(0, st);
        if (first_slice) __syncthreads();
        if (elect_one()) {
            int s = st;
            for (int i = 1; i < NS && i < tiles; ++i) {
                if (++s == NS) s = 0;
                issue(i, s);
            }
        }

        float xmax = 0.f;  // largest |x| of this lane's part of the slice
#pragma unroll
        for (int q = 0; q < S::KS; ++q)
#pragma unroll
            for (int j = 0; j < S::LW; ++j)
#pragma unroll
                for (int h = 0; h < S::PER / 2; ++h) {
                    xmax = fmaxf(xmax, fabsf(__uint_as_float(xall[q][j][h] << 16)));
                    xmax = fmaxf(xmax, fabsf(__uint_as_float(xall[q][j][h] & 0xFFFF0000u)));
                }
        // per activation row (lane quad g): a slice whose largest |x| reaches
        // 2^100 is brought below 2^101 by 2^-es (exact); the rest keep es = 0
        xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, 1));
        xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, 2));
        const int ex = static_cast<int>((__float_as_uint(xmax) >> 23) & 0xFF) - 127;
        const int es = ex > 100 ? ex - 100 : 0;  // 0 .. 28
        const float f = __uint_as_float(static_cast<uint32_t>(127 - es) << 23);  // 2^-es
        // 2^es of the activation rows of this lane's D columns 2t and 2t + 1
        const int e0 = __shfl_sync(0xffffffffu, es, 8 * t), e1 = __shfl_sync(0xffffffffu, es, 8 * t + 4);
        const float ef0 = __uint_as_float(static_cast<uint32_t>(127 + e0) << 23);
        const float ef1 = __uint_as_float(static_cast<uint32_t>(127 + e1) << 23);

        uint32_t bfr[S::KS][S::MMAS][2];
#pragma unroll
        for (int q = 0; q < S::KS; ++q)
#pragma unroll
            for (int j = 0; j < S::LW; ++j) x_fragments<BITS>(xall[q][j], f, &bfr[q][j * S::MPW]);

        const int oa = (g * RG::SBOX + goff) * 2, ob = ((g + 8) * RG::SBOX + goff) * 2;
        const int sbgmask = (1 << (prm.sbw_log - 1)) - 1;  // group columns per box - 1
        float* red_sl = red + sl * rows_cap * MC;

        // ---- walk the CTA's rows, 16 per tile, NS tiles in flight ----
        for (int tile = 0; tile < tiles; ++tile) {
            if (!(ok = mbar_wait(&full[st], ph, 10))) break;
            const uint8_t* cst = code_ring + st * RG::CODE_STAGE;

            constexpr int SBR = S::GPS >= 2 ? S::GPS / 2 : 1;
            uint32_t sa[SBR], sb[SBR], ba[SBR], bb[SBR];
#pragma unroll
            for (int i = 0; i < SBR; ++i) { sa[i] = sb[i] = ba[i] = bb[i] = 0u; }
            if (sb_mode == 2) {
                if (tile == 0 && sl == warp && !(ok = mbar_wait(sb_full, 0, 11))) break;
                const int r_a = tile * 16 + g;
                const uint32_t oa2 = sb_block_off(r_a, g0 & sbgmask, prm.sbw_log);
                const uint32_t ob2 = sb_block_off(r_a + 8, g0 & sbgmask, prm.sbw_log);
                const uint8_t* ss = sb_base + (g0 >> (prm.sbw_log - 1)) * prm.region;
                const uint8_t* bs = ss + prm.nbox * prm.region;
                if constexpr (S::GPS == 1) {
                    sa[0] = *reinterpret_cast<const uint16_t*>(ss + oa2);
                    sb[0] = *reinterpret_cast<const uint16_t*>(ss + ob2);
                    ba[0] = *reinterpret_cast<const uint16_t*>(bs + oa2);
                    bb[0] = *reinterpret_cast<const uint16_t*>(bs + ob2);
                } else {
                    lds_words<SBR>(ss + oa2, sa);
                    lds_words<SBR>(ss + ob2, sb);
                    lds_words<SBR>(bs + oa2, ba);
                    lds_words<SBR>(bs + ob2, bb);
                }
            } else if (sb_mode == 1) {
                const uint8_t* ss = sb_ring + st * 2 * RG::SB_STAGE;
                const uint8_t* bs = ss + RG::SB_STAGE;
                if constexpr (S::GPS == 1) {
                    sa[0] = *reinterpret_cast<const uint16_t*>(ss + oa);
                    sb[0] = *reinterpret_cast<const uint16_t*>(ss + ob);
                    ba[0] = *reinterpret_cast<const uint16_t*>(bs + oa);
                    bb[0] = *reinterpret_cast<const uint16_t*>(bs + ob);
                } else {
                    lds_words<SBR>(ss + oa, sa);
                    lds_words<SBR>(ss + ob, sb);
                    lds_words<SBR>(bs + oa, ba);
                    lds_words<SBR>(bs + ob, bb);
                }
            } else {
                const int64_t ra = n0 + tile * 16 + g, rb = ra + 8;
                const bool va = ra < n1, vb = rb < n1;
#pragma unroll
                for (int i = 0; i < S::GPS; ++i) {
                    if ((g0 + i) * static_cast<int64_t>(GS) < K) {
                        const int sh = (i & 1) * 16;
                        if (va) { sa[i >> 1] |= uint32_t(__ldg(scales + ra * gpr + g0 + i)) << sh;
                                  ba[i >> 1] |= uint32_t(__ldg(biases + ra * gpr + g0 + i)) << sh; }
                        if (vb) { sb[i >> 1] |= uint32_t(__ldg(scales + rb * gpr + g0 + i)) << sh;
                                  bb[i >> 1] |= uint32_t(__ldg(biases + rb * gpr + g0 + i)) << sh; }
                    }
                }
            }

            // acc: rows g, g + 8 x activation rows 2t, 2t + 1 (the MMA's D fragment)
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            // One dequantizer for the whole tile and warp: the fast form when
            // every group this warp meets in the tile allows it (the usual
            // case), else the general form (same results either way).
            bool lane_fast = true;
#pragma unroll
            for (int q = 0; q < S::KS; q += S::CPG) {
                const int gi = q / S::CPG;
                lane_fast = lane_fast && group_sb(sa[gi >> 1], ba[gi >> 1], gi).fast &&
                            group_sb(sb[gi >> 1], bb[gi >> 1], gi).fast;
            }
            auto tile_products = [&](auto fast_tag) {
#pragma unroll
                for (int q = 0; q < S::KS; ++q) {
                    uint32_t wa[S::LW], wb[S::LW];
                    lds_words<S::LW>(cst + offa[q], wa);
                    lds_words<S::LW>(cst + offb[q], wb);
                    const int gi = q / S::CPG;
                    const GroupSB gA = group_sb(sa[gi >> 1], ba[gi >> 1], gi);
                    const GroupSB gB = group_sb(sb[gi >> 1], bb[gi >> 1], gi);
#pragma unroll
                    for (int j = 0; j < S::LW; ++j) {
                        uint32_t pa[S::NP], pb[S::NP];
                        if constexpr (decltype(fast_tag)::value) {
                            Dequant<BITS>::run_fast(wa[j], gA, pa);
                            Dequant<BITS>::run_fast(wb[j], gB, pb);
                        } else {
                            Dequant<BITS>::run(wa[j], gA, pa);
                            Dequant<BITS>::run(wb[j], gB, pb);
                        }
#pragma unroll
                        for (int u = 0; u < S::MPW; ++u)
                            mma_bf16_16816(acc, pa[2 * u], pb[2 * u], pa[2 * u + 1], pb[2 * u + 1],
                                           bfr[q][j * S::MPW + u][0], bfr[q][j * S::MPW + u][1]);
                    }
                }
            };
            if (__all_sync(__activemask(), lane_fast)) tile_products(std::true_type{});
            else tile_products(std::false_type{});
            // every lane has read the stage: refill it with tile + NS
            __syncwarp();
            if (tile + NS < tiles && elect_one()) issue(tile + NS, st);
            if (++st == NS) { st = 0; ph ^= 1u; }

            const int r0 = tile * 16 + g;
            // undo the activations' 2^-es (exact)
            if (M1) {
                if (t == 0) { red_sl[r0] = acc[0] * ef0; red_sl[r0 + 8] = acc[2] * ef0; }
            } else {
                const int m0 = 2 * t, m1 = 2 * t + 1;
                if (m0 < M) { red_sl[r0 * M + m0] = acc[0] * ef0; red_sl[(r0 + 8) * M + m0] = acc[2] * ef0; }
                if (m1 < M) { red_sl[r0 * M + m1] = acc[1] * ef1; red_sl[(r0 + 8) * M + m1] = acc[3] * ef1; }
            }
        }
    }
    __syncthreads();

    // ---- fixed-order reduction over the slices: four interleaved chains
    // (slices j, j + 4, j + 8, ...), then (c0 + c1) + (c2 + c3) ----
    const int slice_stride = rows_cap * MC;
    for (int m = 0; m < MC; ++m) {
        for (int r = threadIdx.x; r < rows; r += blockDim.x) {
            const float* p = red + r * MC + m;
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (j < nslices) c[j] = p[j * slice_stride];
            for (int sl = 4; sl < nslices; sl += 4) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (sl + j < nslices) c[j] += p[(sl + j) * slice_stride];
            }
            prm.y[s_yrow[m] * N + n0 + r] = f32_to_bf16_bits((c[0] + c[1]) + (c[2] + c[3]));
        }
    }
}

template <bool GATHER>
using KernelPtr = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const QmvParams);

template <bool GATHER>
struct Variant {
    KernelPtr<GATHER> k[2][3];     // [one activation row][ring depth 4, 3, 2]
    int code_stage;                // code bytes per warp and stage
    int sb_stage;                  // bytes of one per-tile scale (or bias) box
    int code_row_bytes;            // code bytes per row and slice (TMA box row)
    int swizzle_bytes;             // 0, 32, 64 or 128
    int sbox;                      // groups per scale box row
    int kslice;
};

template <int BITS, int GS, bool GATHER>
Variant<GATHER> variant() {
    using RG = Ring<BITS, GS>;
    Variant<GATHER> v{};
    v.k[0][0] = qmv_kernel<BITS, GS, GATHER, 4, false>;
    v.k[0][1] = qmv_kernel<BITS, GS, GATHER, 3, false>;
    v.k[0][2] = qmv_kernel<BITS, GS, GATHER, 2, false>;
    // a gather problem's row count is only known on the device
    v.k[1][0] = GATHER ? v.k[0][0] : qmv_kernel<BITS, GS, GATHER, 4, !GATHER>;
    v.k[1][1] = GATHER ? v.k[0][1] : qmv_kernel<BITS, GS, GATHER, 3, !GATHER>;
    v.k[1][2] = GATHER ? v.k[0][2] : qmv_kernel<BITS, GS, GATHER, 2, !GATHER>;
    v.code_stage = RG::CODE_STAGE;
    v.sb_stage = RG::SB_STAGE;
    v.code_row_bytes = RG::CBYTES;
    v.swizzle_bytes = RG::SWZ ? RG::CBYTES : 0;
    v.sbox = RG::SBOX;
    v.kslice = Shape<BITS, GS>::KSLICE;
    return v;
}

template <bool GATHER>
bool pick(int bits, int gs, Variant<GATHER>& v) {
    if (bits == 4 && gs == 32) { v = variant<4, 32, GATHER>(); return true; }
    if (bits == 4 && gs == 64) { v = variant<4, 64, GATHER>(); return true; }
    if (bits == 4 && gs == 128) { v = variant<4, 128, GATHER>(); return true; }
    if (bits == 8 && gs == 32) { v = variant<8, 32, GATHER>(); return true; }
    if (bits == 8 && gs == 64) { v = variant<8, 64, GATHER>(); return true; }
    if (bits == 8 && gs == 128) { v = variant<8, 128, GATHER>(); return true; }
    if (bits == 2 && gs == 64) { v = variant<2, 64, GATHER>(); return true; }
    if (bits == 2 && gs == 128) { v = variant<2, 128, GATHER>(); return true; }
    return false;
}

// Dynamic shared memory budget: the per-block limit (227 KB) less the kernel's
// static shared memory (the row maps and the 1024-byte alignment of the ring).
constexpr size_t kSmemMax = 227 * 1024 - 2048;


// Split N over CTAs (every SM busy, at most 128 rows a CTA); choose how the
// scales and biases reach shared memory and the deepest ring that fits next to
// the slice partials (nslices x rows x M fp32).
struct Plan {
    int ctas, rows_cap, rows_max, warps, depth;
    int sb_mode, sbw_log, nbox;
    uint32_t region, off_sb, off_bar, off_red;
    size_t smem;
};

static size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

Plan plan(int64_t N, int64_t K, int M, int gs, int kslice, int code_stage, int sb_stage,
          int num_sms, bool gather) {
    const int64_t nslices = (K + kslice - 1) / kslice;
    const int warps = static_cast<int>(std::min<int64_t>(kMaxWarps, nslices));
    const int64_t gpr = K / gs;
    const bool sb_aligned = (gpr * 2) % 16 == 0;  // rows of scales are 16-byte multiples
    // A gather launches one set of CTAs per (expert, <= 8 pairs) problem, so
    // its CTAs take up to 128 rows each instead of spreading one matrix over
    // every SM.
    int64_t ctas = gather ? (N + 127) / 128
                          : std::max<int64_t>(std::min<int64_t>(num_sms, (N + 15) / 16),
                                              (N + 127) / 128);
    const int64_t tiles = (N + 15) / 16;
    for (;;) {
        // whole 16-row tiles per CTA: a CTA's last tile is never nearly empty
        const int64_t cap = (tiles + ctas - 1) / ctas * 16;
        const int64_t rows = std::min<int64_t>(cap, N);
        const size_t red = static_cast<size_t>(nslices * cap * M) * sizeof(float);
        Plan p{};
        p.ctas = static_cast<int>(ctas);
        p.rows_cap = static_cast<int>(cap);
        p.rows_max = static_cast<int>(rows);
        p.warps = warps;
        // layout for ring depth d with `sb_stage_bytes` of scales per stage and
        // `block` bytes of scale block; true if it fits
        auto fit = [&](int d, size_t sb_stage_bytes, size_t block) {
            const size_t codes = static_cast<size_t>(warps) * d * code_stage;
            const size_t sb = block + static_cast<size_t>(warps) * d * sb_stage_bytes;
            const size_t bars = round_up(static_cast<size_t>(warps * d + 1) * 8, 16);
            p.depth = d;
            p.off_sb = static_cast<uint32_t>(codes);
            p.off_bar = static_cast<uint32_t>(codes + sb);
            p.off_red = static_cast<uint32_t>(codes + sb + bars);
            p.smem = 1024 + codes + sb + bars + red;
            return p.smem <= kSmemMax;
        };
        // mode 2: the CTA's block of scales and biases, loaded once
        if (sb_aligned && rows <= 256 && (gpr >= 64 || gpr == 8 || gpr == 16 || gpr == 32)) {
            p.sb_mode = 2;
            const int sbw = gpr >= 64 ? 128 : static_cast<int>(gpr) * 2;
            p.sbw_log = sbw == 128 ? 7 : sbw == 64 ? 6 : sbw == 32 ? 5 : 4;
            p.nbox = gpr >= 64 ? static_cast<int>((gpr + 63) / 64) : 1;
            // the box holds rows_max rows; the region spans every row a tile can
            // address (rows_cap), so reads past the CTA's rows stay inside it
            p.region = static_cast<uint32_t>(round_up(static_cast<size_t>(cap) * sbw, 1024));
            for (int d = 4; d >= 2; --d)
                if (fit(d, 0, 2u * p.nbox * p.region)) return p;
        }
        // mode 1: scales and biases per tile with the codes; mode 0: plain loads
        p.sb_mode = sb_aligned ? 1 : 0;
        p.sbw_log = 4;
        p.nbox = 0;
        p.region = 0;
        for (int d = 4; d >= 2; --d)
            if (fit(d, sb_aligned ? 2 * sb_stage : 0, 0)) return p;
        if (cap <= 16) return p;  // nothing smaller to try: launch fails loudly
        ctas = ctas * 2;
    }
}

// 3-D tensor maps [E][rows][inner] over the codes, scales and biases.
template <bool GATHER>
bool encode_maps(const Variant<GATHER>& v, const Plan& p, const uint32_t* codes,
                 const void* scales, const void* biases, int64_t E, int64_t N, int64_t K, int gs,
                 int bits, CUtensorMap* mc, CUtensorMap* ms, CUtensorMap* mb) {
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return false;
    const int64_t wpr = K * bits / 32, gpr = K / gs;
    {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(wpr) * 4, static_cast<cuuint64_t>(wpr * N) * 4};
        cuuint32_t box[3] = {static_cast<cuuint32_t>(v.code_row_bytes / 4), 16, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(codes), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                v.swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                : v.swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                : v.swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                        : CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    if (p.sb_mode == 0) {
        *ms = *mc;  // unused
        *mb = *mc;
        return true;
    }
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(gpr), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(E)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(gpr) * 2, static_cast<cuuint64_t>(gpr * N) * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(v.sbox), 16, 1};
    CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE;
    if (p.sb_mode == 2) {  // whole rows of the CTA, 2^sbw_log bytes of groups per box
        box[0] = 1u << (p.sbw_log - 1);
        box[1] = static_cast<cuuint32_t>(p.rows_max);
        swz = p.sbw_log == 7   ? CU_TENSOR_MAP_SWIZZLE_128B
              : p.sbw_log == 6 ? CU_TENSOR_MAP_SWIZZLE_64B
              : p.sbw_log == 5 ? CU_TENSOR_MAP_SWIZZLE_32B
                               : CU_TENSOR_MAP_SWIZZLE_NONE;
    }
    cuuint32_t es[3] = {1, 1, 1};
    for (int i = 0; i < 2; ++i) {
        if (enc(i ? mb : ms, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                const_cast<void*>(i ? biases : scales), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

static void set_plan(QmvParams& prm, const Plan& p, int64_t N) {
    prm.ctas_per_problem = p.ctas;
    prm.tiles_q = static_cast<int>((N + 15) / 16 / p.ctas);
    prm.tiles_r = static_cast<int>((N + 15) / 16 % p.ctas);
    prm.rows_cap = p.rows_cap;
    prm.rows_max = p.rows_max;
    prm.sb_mode = p.sb_mode;
    prm.sbw_log = p.sbw_log;
    prm.nbox = p.nbox;
    prm.region = p.region;
    prm.off_sb = p.off_sb;
    prm.off_bar = p.off_bar;
    prm.off_red = p.off_red;
}

template <bool GATHER>
cudaError_t launch(const Variant<GATHER>& v, const Plan& p, dim3 grid, const CUtensorMap& mc,
                   const CUtensorMap& ms, const CUtensorMap& mb, const QmvParams& prm,
                   cudaStream_t stream) {
    const int one = prm.M == 1 ? 1 : 0;
    KernelPtr<GATHER> k = v.k[one][p.depth == 4 ? 0 : p.depth == 3 ? 1 : 2];
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(p.smem));
    if (e != cudaSuccess) return e;
    // Programmatic dependent launch: the kernel may start while the previous
    // kernel on the stream drains; it waits (griddepcontrol.wait) before it
    // reads anything but weights (prefetched into L2) or writes anything.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(static_cast<unsigned>(p.warps * 32), 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, mc, ms, mb, prm);
}

}  // namespace

bool qmv_supported(int bits, int gs) {
    Variant<false> v;
    return pick<false>(bits, gs, v);
}

unsigned int qmv_error_take() { return pipeline_error_take(); }

cudaError_t launch_qmv(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                       const void* scales, const void* biases, int gs, int bits, void* y,
                       cudaStream_t stream, int num_sms) {
    Variant<false> v;
    if (!pick<false>(bits, gs, v)) return cudaErrorInvalidValue;
    const Plan p = plan(N, K, static_cast<int>(M), gs, v.kslice, v.code_stage, v.sb_stage, num_sms,
                        false);
    CUtensorMap mc, ms, mb;
    if (!encode_maps(v, p, codes, scales, biases, 1, N, K, gs, bits, &mc, &ms, &mb))
        return cudaErrorInvalidValue;
    QmvParams prm{};
    prm.x = static_cast<const uint16_t*>(x);
    prm.codes = codes;
    prm.scales = static_cast<const uint16_t*>(scales);
    prm.biases = static_cast<const uint16_t*>(biases);
    prm.y = static_cast<uint16_t*>(y);
    prm.N = N;
    prm.K = K;
    prm.M = static_cast<int>(M);
    set_plan(prm, p, N);
    return launch<false>(v, p, dim3(p.ctas, 1, 1), mc, ms, mb, prm, stream);
}

cudaError_t launch_qmv_gather(const void* x, int64_t K, int64_t N, const uint32_t* codes,
                              const void* scales, const void* biases, int gs, int bits,
                              const uint32_t* lhs, const uint32_t* perm,
                              const uint32_t* problems, const uint32_t* num_problems,
                              int64_t max_problems, int64_t E, void* y, cudaStream_t stream,
                              int num_sms) {
    Variant<true> v;
    if (!pick<true>(bits, gs, v)) return cudaErrorInvalidValue;
    if (max_problems <= 0) return cudaSuccess;
    // Every problem covers all N rows of one expert for <= 8 pairs.
    const Plan p = plan(N, K, 8, gs, v.kslice, v.code_stage, v.sb_stage, num_sms, true);
    CUtensorMap mc, ms, mb;
    if (!encode_maps(v, p, codes, scales, biases, E, N, K, gs, bits, &mc, &ms, &mb))
        return cudaErrorInvalidValue;
    QmvParams prm{};
    prm.x = static_cast<const uint16_t*>(x);
    prm.codes = codes;
    prm.scales = static_cast<const uint16_t*>(scales);
    prm.biases = static_cast<const uint16_t*>(biases);
    prm.y = static_cast<uint16_t*>(y);
    prm.N = N;
    prm.K = K;
    prm.M = 8;
    set_plan(prm, p, N);
    prm.lhs = lhs;
    prm.perm = perm;
    prm.problems = problems;
    prm.num_problems = num_problems;
    prm.E = E;
    // The problem count is known only on the device; max_problems bounds it.
    // gridDim.y is limited to 65535, so larger bounds take several launches,
    // each covering the next 65535 problems (blocks past the count return).
    constexpr int64_t kMaxGridY = 65535;
    for (int64_t p0 = 0; p0 < max_problems; p0 += kMaxGridY) {
        const int64_t np = std::min(kMaxGridY, max_problems - p0);
        prm.problem0 = static_cast<uint32_t>(p0);
        cudaError_t e = launch<true>(v, p, dim3(p.ctas, static_cast<unsigned>(np), 1), mc, ms, mb,
                                     prm, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace nvq
