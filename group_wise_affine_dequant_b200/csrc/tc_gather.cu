// Tensor-core mixture-of-experts product ("Docs / Quantization", section
// "Mixture of experts": with rows sorted by expert, a grouped kernel reads each
// expert's weights once). Each expert sees a handful of rows (tens), so the
// product is computed transposed: D^T = W_e . X_e^T with the expert's weights as
// the 128-row MMA operand A (dequantized into shared memory) and the expert's
// gathered activation rows as the N side (16 .. 256 columns). Every weight tile
// is read from HBM once and used for all of the expert's rows.
//
// Work unit: (expert e, 128 weight rows). Roles, per CTA (persistent):
//   warp 0      producer: per unit, loads the pair -> activation-row map of the
//               unit's pairs into shared memory; per k-step, TMA the code tile
//               (128 rows x 64 k) and gather the activation rows with TMA
//               tile::gather4 (4 rows per copy, 128-byte swizzle) straight into
//               the B operand; scales/biases by TMA in blocks of 8 groups.
//   warp 1      TMEM allocation; one thread issues tcgen05.mma (M = 128,
//               N = pairs rounded up to 16, K = 16) into a double-buffered
//               TMEM accumulator.
//   warps 2-5   epilogue: TMEM lane = weight row, column = pair; each column is
//               stored to its pair's output row (32 lanes -> 64 contiguous bytes).
//   warps 6-13  dequantize, two threads per weight row (half a k-step each),
//               into the canonical K-major 128-byte-swizzled A tile.
// Waits are bounded by a timer like the other pipelines.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tma.cuh"

namespace nvq {
namespace {

using namespace tc;

constexpr int WM = 128;          // weight rows per unit (TMEM lanes)
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int kMaxPairs = 256;   // pairs per pass (TMEM columns of one accumulator)
constexpr int kThreads = 448;
constexpr int kDequantWarp0 = 6;
constexpr int kDequantThreads = 256;

__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int col, int r0, int r1, int r2, int r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(col), "r"(r0), "r"(r1),
        "r"(r2), "r"(r3)
        : "memory");
}

struct GParams {
    uint16_t* y;                // [R, N]
    const uint32_t* lhs;        // nullable
    const uint32_t* perm;       // [R] pairs in expert order
    const uint32_t* offsets;    // [E + 2]
    const uint16_t* scales;
    const uint16_t* biases;
    int64_t N, K, E;
    int gs, lg_gs;
    int wtiles;                 // ceil(N / 128)
    int stages;
    uint32_t a_off, x_off, c_off, sb_off, idx_off, bar_off;
    uint32_t c_stage_bytes;
    int sb_tma;
    uint32_t m2, m4, m6;        // shift counts 2, 4, 6
};

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
tc_gather_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_c,
                 const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_b,
                 const GParams prm) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = prm.stages;
    constexpr uint32_t A_STAGE = WM * BK * 2;            // 16 KB
    constexpr uint32_t X_STAGE = kMaxPairs * BK * 2;     // 32 KB
    uint8_t* a_ring = smem + prm.a_off;
    uint8_t* x_ring = smem + prm.x_off;
    uint8_t* c_ring = smem + prm.c_off;
    uint8_t* sb_ring = smem + prm.sb_off;
    int* s_rows = reinterpret_cast<int*>(smem + prm.idx_off);  // activation row per pair
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prm.bar_off);
    uint64_t* full_x = bars;            // gathered activations (TMA)
    uint64_t* full_c = bars + NS;       // codes (TMA)
    uint64_t* full_a = bars + 2 * NS;   // dequantized weights (dequant warps)
    uint64_t* empty = bars + 3 * NS;    // stage consumed (tcgen05.commit)
    uint64_t* acc_full = bars + 4 * NS;
    uint64_t* acc_empty = bars + 4 * NS + 2;
    uint64_t* sb_full = bars + 4 * NS + 4;
    uint64_t* sb_empty = bars + 4 * NS + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * NS + 8);
    constexpr uint32_t SB_SLOT = 2u * WM * 16u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full_x[s], 1);
            mbar_init(&full_c[s], 1);
            mbar_init(&full_a[s], kDequantThreads / 32);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
            mbar_init(&sb_full[a], 1);
            mbar_init(&sb_empty[a], kDequantThreads / 32);
        }
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int ksteps = static_cast<int>(prm.K / BK);
    const int sgk = 8 * prm.gs / BK;  // k-steps per block of 8 groups
    const int units = static_cast<int>(prm.E) * prm.wtiles;

    // Every role walks the same sequence of (unit, pass) items: a unit's pairs
    // are cut into passes of at most kMaxPairs.
    auto unit_pairs = [&](int u, int& e, int& wt, int& first, int& count) {
        e = u / prm.wtiles;
        wt = u - e * prm.wtiles;
        first = static_cast<int>(__ldg(prm.offsets + e));
        count = static_cast<int>(__ldg(prm.offsets + e + 1)) - first;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int s = 0;
        uint32_t use = 0, blk = 0;
        int issued = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
                const int cn = min(kMaxPairs, count - p0);
                const int groups4 = (cn + 3) / 4;
                // activation rows of this pass (padding repeats the last row)
                __syncwarp();
                for (int j = lane; j < groups4 * 4; j += 32) {
                    const int jj = j < cn ? j : cn - 1;
                    const uint32_t pair = __ldg(prm.perm + first + p0 + jj);
                    s_rows[j] = prm.lhs ? static_cast<int>(__ldg(prm.lhs + pair)) : static_cast<int>(pair);
                }
                __syncwarp();
                if (lane == 0) {
                    int kb = 0;
                    for (int ks = 0; ks < ksteps && ok; ++ks) {
                        if (prm.sb_tma && kb == 0) {
                            const int slot = blk & 1;
                            const uint32_t bu = blk >> 1;
                            if (bu > 0 && !(ok = mbar_wait(&sb_empty[slot], (bu - 1) & 1, 27))) break;
                            mbar_expect_tx(&sb_full[slot], SB_SLOT);
                            uint8_t* dst = sb_ring + slot * SB_SLOT;
                            const int gcol = blk_in_tile(ks, sgk) * 8;
                            tma_load_3d(dst, &map_s, &sb_full[slot], gcol, wt * WM, e);
                            tma_load_3d(dst + WM * 16, &map_b, &sb_full[slot], gcol, wt * WM, e);
                            ++blk;
                        }
                        if (++kb == sgk) kb = 0;
                        if (use > 0 && !(ok = mbar_wait(&empty[s], (use - 1) & 1, 21))) break;
                        mbar_expect_tx(&full_c[s], WM * BK * BITS / 8);
                        tma_load_3d(c_ring + s * prm.c_stage_bytes, &map_c, &full_c[s],
                                    ks * BK * BITS / 32, wt * WM, e);
                        mbar_expect_tx(&full_x[s], static_cast<uint32_t>(groups4) * 4 * BK * 2);
                        uint8_t* xd = x_ring + s * X_STAGE;
                        for (int g4 = 0; g4 < groups4; ++g4)
                            tma_gather4(xd + g4 * 4 * BK * 2, &map_x, &full_x[s], ks * BK,
                                        s_rows[4 * g4], s_rows[4 * g4 + 1], s_rows[4 * g4 + 2],
                                        s_rows[4 * g4 + 3]);
                        ++issued;
                        if (++s == NS) { s = 0; ++use; }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            }
        }
        if (lane == 0) {
            for (int j = 0; j < NS && j < issued; ++j) {  // drain the last copies
                if (--s < 0) { s = NS - 1; --use; }
                mbar_wait(&full_c[s], use & 1, 29);
                mbar_wait(&full_x[s], use & 1, 29);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0;
            uint32_t use = 0;
            int local = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int e, wt, first, count;
                unit_pairs(u, e, wt, first, count);
                for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs, ++local) {
                    const int cn = min(kMaxPairs, count - p0);
                    const int npad = (cn + 15) / 16 * 16;
                    const uint32_t idesc = idesc_bf16(WM, npad);
                    const int a = local & 1;
                    const uint32_t ause = static_cast<uint32_t>(local >> 1);
                    if (ause > 0 && !(ok = mbar_wait(&acc_empty[a], (ause - 1) & 1, 22))) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * kMaxPairs);
                    for (int ks = 0; ks < ksteps; ++ks) {
                        if (!(ok = mbar_wait(&full_a[s], use & 1, 23))) break;
                        if (!(ok = mbar_wait(&full_x[s], use & 1, 24))) break;
                        tc_fence_after();
                        const uint64_t ad = sw128_desc(a_ring + s * A_STAGE);
                        const uint64_t bd = sw128_desc(x_ring + s * X_STAGE);
#pragma unroll
                        for (int kk = 0; kk < BK / UMMA_K; ++kk)
                            tc_mma(d_tmem, ad + (kk * UMMA_K * 2 >> 4), bd + (kk * UMMA_K * 2 >> 4), idesc,
                                   (ks > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&empty[s]);
                        if (++s == NS) { s = 0; ++use; }
                    }
                    if (ok) tc_commit(&acc_full[a]);
                }
            }
        }
    } else if (warp < kDequantWarp0) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int wrow = q * 32 + lane;  // weight row within the unit = TMEM lane
        int local = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            const int64_t n = static_cast<int64_t>(wt) * WM + wrow;
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs, ++local) {
                const int cn = min(kMaxPairs, count - p0);
                const int a = local & 1;
                const uint32_t ause = static_cast<uint32_t>(local >> 1);
                if (!(ok = mbar_wait(&acc_full[a], ause & 1, 25))) break;
                tc_fence_after();
                for (int c0 = 0; c0 < cn; c0 += 16) {
                    uint32_t v[16];
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                           static_cast<uint32_t>(a * kMaxPairs + c0);
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                          "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                          "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                        : "r"(taddr));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (c0 + j < cn && n < prm.N) {
                            const uint32_t pair = __ldg(prm.perm + first + p0 + c0 + j);
                            prm.y[static_cast<int64_t>(pair) * prm.N + n] =
                                f32_to_bf16_bits(__uint_as_float(v[j]));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[a]);
            }
        }
    } else {
        // ------------------------------------------------------------ dequantize
        const int dt = threadIdx.x - kDequantWarp0 * 32;  // 0 .. 255
        const int r = dt >> 1;                            // weight row within the unit
        const int half = dt & 1;                          // chunks 4*half .. 4*half+3
        constexpr int WPS = BK * BITS / 32;               // code words per row per k-step
        constexpr int WPH = WPS / 2;                      // ... per half
        using DQ = Dequant<BITS>;
        const int64_t gpr = prm.K / prm.gs;
        int s = 0;
        uint32_t use = 0, blk = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            const int64_t n = static_cast<int64_t>(wt) * WM + r;
            const bool live = n < prm.N;
            const uint16_t* srow = prm.scales + (static_cast<int64_t>(e) * prm.N + (live ? n : 0)) * gpr;
            const uint16_t* brow = prm.biases + (static_cast<int64_t>(e) * prm.N + (live ? n : 0)) * gpr;
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
                int kb = 0;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int gfirst = (ks * BK) >> prm.lg_gs;
                    const int slot = blk & 1;
                    // this thread's chunks lie in one group unless groups are 32 wide
                    const int gsel = (prm.gs < BK) ? half : 0;
                    float sc = 0.f, bc = 0.f;
                    if (prm.sb_tma) {
                        if (kb == 0 && !(ok = mbar_wait(&sb_full[slot], (blk >> 1) & 1, 28))) break;
                        const uint16_t* ss = reinterpret_cast<const uint16_t*>(sb_ring + slot * SB_SLOT);
                        const int gi = (gfirst & 7) + gsel;
                        sc = bf16_bits_to_f32(ss[r * 8 + gi]);
                        bc = bf16_bits_to_f32(ss[WM * 8 + r * 8 + gi]);
                    } else if (live) {
                        sc = bf16_bits_to_f32(__ldg(srow + gfirst + gsel));
                        bc = bf16_bits_to_f32(__ldg(brow + gfirst + gsel));
                    }
                    if (!(ok = mbar_wait(&full_c[s], use & 1, 26))) break;
                    // codes of row r, this half: 16 bytes (4-bit), 32 (8-bit) or 8 (2-bit)
                    const uint8_t* cst = c_ring + s * prm.c_stage_bytes;
                    uint32_t w[WPH];
                    if constexpr (BITS == 4) {
                        const uint32_t off = r * 32 + ((half ^ ((r >> 2) & 1)) << 4);
                        const uint4 v4 = *reinterpret_cast<const uint4*>(cst + off);
                        w[0] = v4.x; w[1] = v4.y; w[2] = v4.z; w[3] = v4.w;
                    } else if constexpr (BITS == 8) {
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int j = 2 * half + jj;
                            const uint32_t off = r * 64 + ((j ^ ((r >> 1) & 3)) << 4);
                            const uint4 v4 = *reinterpret_cast<const uint4*>(cst + off);
                            w[4 * jj] = v4.x; w[4 * jj + 1] = v4.y; w[4 * jj + 2] = v4.z; w[4 * jj + 3] = v4.w;
                        }
                    } else {
                        const uint2 v2 = *reinterpret_cast<const uint2*>(cst + r * 16 + half * 8);
                        w[0] = v2.x; w[1] = v2.y;
                    }
                    uint8_t* arow = a_ring + s * A_STAGE + (r >> 3) * 1024 + (r & 7) * 128;
                    const uint32_t s2 = (__float_as_uint(sc) >> 16) * 0x00010001u;
                    const uint32_t b2 = (__float_as_uint(bc) >> 16) * 0x00010001u;
                    constexpr int WPC = BITS == 2 ? 1 : 8 * BITS / 32;  // words per 16-byte chunk (2-bit: 2 chunks per word)
#pragma unroll
                    for (int cw = 0; cw < (BITS == 2 ? 2 : 4); ++cw) {
                        uint32_t out[8];
                        if constexpr (BITS == 2) {
                            DQ::run(w[cw], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6, out);
                        } else {
#pragma unroll
                            for (int uu = 0; uu < WPC; ++uu)
                                DQ::run(w[cw * WPC + uu], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6,
                                        out + uu * DQ::PAIRS);
                        }
#pragma unroll
                        for (int h = 0; h < (BITS == 2 ? 2 : 1); ++h) {
                            const int c = 4 * half + (BITS == 2 ? 2 * cw + h : cw);
                            uint4 o;
                            o.x = out[4 * h]; o.y = out[4 * h + 1]; o.z = out[4 * h + 2]; o.w = out[4 * h + 3];
                            *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) = o;
                        }
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_a[s]);
                    if (prm.sb_tma && (kb == sgk - 1 || ks == ksteps - 1)) {
                        if (lane == 0) mbar_arrive(&sb_empty[slot]);
                        ++blk;
                    }
                    if (++kb == sgk) kb = 0;
                    if (++s == NS) { s = 0; ++use; }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512));
    }
}

// Pairs whose expert or token id is out of range (bucket E of the router) get
// zero rows.
__global__ void zero_invalid_pairs(uint16_t* y, const uint32_t* perm, const uint32_t* offsets,
                                   int64_t E, int64_t N) {
    const int64_t first = offsets[E], last = offsets[E + 1];
    for (int64_t i = first + blockIdx.x; i < last; i += gridDim.x)
        for (int64_t n = threadIdx.x; n < N; n += blockDim.x) y[static_cast<int64_t>(perm[i]) * N + n] = 0;
}

}  // namespace

bool tc_gather_supported(int64_t K, int64_t N, int bits, int gs) {
    return K % BK == 0 && K >= BK && N > 0 && (bits == 2 || bits == 4 || bits == 8) &&
           (gs == 32 || gs == 64 || gs == 128);
}

unsigned int tc_gather_error_take() { return pipeline_error_take(); }

cudaError_t launch_tc_gather(const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs,
                             const uint32_t* perm, const uint32_t* offsets, int64_t E, int64_t N,
                             const uint32_t* codes, const void* scales, const void* biases, int gs,
                             int bits, void* y, cudaStream_t stream, int num_sms) {
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map_x, map_c, map_s, map_b;
    {   // activation rows, gathered 4 at a time: box one row high
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(x_rows)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
        cuuint32_t box[2] = {BK, 1};
        cuuint32_t es[2] = {1, 1};
        if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int64_t wpr = K * bits / 32, gpr = K / gs;
    {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(wpr) * 4, static_cast<cuuint64_t>(wpr * N) * 4};
        cuuint32_t box[3] = {static_cast<cuuint32_t>(BK * bits / 32), WM, 1};
        cuuint32_t es[3] = {1, 1, 1};
        const CUtensorMapSwizzle swz = bits == 4   ? CU_TENSOR_MAP_SWIZZLE_32B
                                       : bits == 8 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_NONE;
        if (enc(&map_c, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(codes), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const bool sb_tma = (gpr * 2) % 16 == 0;
    if (sb_tma) {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(gpr), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(gpr) * 2, static_cast<cuuint64_t>(gpr * N) * 2};
        cuuint32_t box[3] = {8, WM, 1};
        cuuint32_t es[3] = {1, 1, 1};
        for (int i = 0; i < 2; ++i)
            if (enc(i ? &map_b : &map_s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                    const_cast<void*>(i ? biases : scales), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
    } else {
        map_s = map_c;
        map_b = map_c;
    }
    GParams prm{};
    prm.y = static_cast<uint16_t*>(y);
    prm.lhs = lhs;
    prm.perm = perm;
    prm.offsets = offsets;
    prm.scales = static_cast<const uint16_t*>(scales);
    prm.biases = static_cast<const uint16_t*>(biases);
    prm.N = N;
    prm.K = K;
    prm.E = E;
    prm.gs = gs;
    prm.lg_gs = gs == 32 ? 5 : gs == 64 ? 6 : 7;
    prm.wtiles = static_cast<int>((N + WM - 1) / WM);
    prm.sb_tma = sb_tma ? 1 : 0;
    prm.m2 = 2;
    prm.m4 = 4;
    prm.m6 = 6;
    const uint32_t a_stage = WM * BK * 2;
    const uint32_t x_stage = kMaxPairs * BK * 2;
    const uint32_t c_stage = (static_cast<uint32_t>(WM) * BK * bits / 8 + 1023) / 1024 * 1024;
    const uint32_t sb_ring = 2u * 2u * WM * 16u;
    const uint32_t idx = kMaxPairs * 4;
    const uint32_t per_stage = a_stage + x_stage + c_stage;
    const uint32_t budget = 227 * 1024 - 1024 - 512 - sb_ring - idx;
    int stages = static_cast<int>(budget / per_stage);
    if (stages > 4) stages = 4;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    prm.stages = stages;
    prm.a_off = 0;
    prm.x_off = a_stage * stages;
    prm.c_off = prm.x_off + x_stage * stages;
    prm.sb_off = prm.c_off + c_stage * stages;
    prm.idx_off = prm.sb_off + sb_ring;
    prm.bar_off = prm.idx_off + idx;
    prm.c_stage_bytes = c_stage;
    const size_t smem = prm.bar_off + (4 * stages + 8) * 8 + 16 + 1024;
    const int units = static_cast<int>(E) * prm.wtiles;
    const int grid = units < num_sms ? units : num_sms;
    void (*k)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const GParams) =
        bits == 4 ? tc_gather_kernel<4> : bits == 8 ? tc_gather_kernel<8> : tc_gather_kernel<2>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, stream>>>(map_x, map_c, map_s, map_b, prm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    zero_invalid_pairs<<<64, 256, 0, stream>>>(static_cast<uint16_t*>(y), perm, offsets, E, N);
    return cudaGetLastError();
}

}  // namespace nvq
