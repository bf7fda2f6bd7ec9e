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
constexpr int kMaxPairs = 128;   // pairs per pass (TMEM columns of one accumulator)
constexpr int kEpilogueWarp0 = 2;
constexpr int kXWarp = 6;        // activation-row producer
constexpr int kDequantWarp0 = 7; // warps 7-22: dequantize, four threads per weight row
constexpr int kDequantThreads = 512;
constexpr int kThreads = kDequantWarp0 * 32 + kDequantThreads;

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
    int dx, dc, da;             // depths: gathered activations, codes, dequantized weights
    uint32_t x_off, c_off, a_off, sb_off, idx_off, bar_off;
    uint32_t c_stage_bytes;
    int sb_tma;
    uint32_t m2, m4, m6;        // shift counts 2, 4, 6
};

struct RingPos {
    int s = 0;
    uint32_t use = 0;
    __device__ __forceinline__ void next(int depth) {
        if (++s == depth) { s = 0; ++use; }
    }
};

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
tc_gather_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_c,
                 const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_b,
                 const GParams prm) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int DX = prm.dx, DC = prm.dc, DA = prm.da;
    constexpr uint32_t A_STAGE = WM * BK * 2;            // 16 KB
    constexpr uint32_t X_STAGE = kMaxPairs * BK * 2;     // 16 KB
    uint8_t* a_ring = smem + prm.a_off;
    uint8_t* x_ring = smem + prm.x_off;
    uint8_t* c_ring = smem + prm.c_off;
    uint8_t* sb_ring = smem + prm.sb_off;
    int* s_rows = reinterpret_cast<int*>(smem + prm.idx_off);  // activation row per pair
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prm.bar_off);
    uint64_t* full_x = bars;
    uint64_t* empty_x = full_x + DX;
    uint64_t* full_c = empty_x + DX;
    uint64_t* empty_c = full_c + DC;
    uint64_t* full_a = empty_c + DC;
    uint64_t* empty_a = full_a + DA;
    uint64_t* acc_full = empty_a + DA;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* sb_full = acc_empty + 2;
    uint64_t* sb_empty = sb_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sb_empty + 2);
    constexpr uint32_t SB_SLOT = 2u * WM * 16u;
    constexpr int kDequantWarps = kDequantThreads / 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < DX; ++i) { mbar_init(&full_x[i], 1); mbar_init(&empty_x[i], 1); }
        for (int i = 0; i < DC; ++i) { mbar_init(&full_c[i], 1); mbar_init(&empty_c[i], kDequantWarps); }
        for (int i = 0; i < DA; ++i) { mbar_init(&full_a[i], kDequantWarps); mbar_init(&empty_a[i], 1); }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
            mbar_init(&sb_full[a], 1);
            mbar_init(&sb_empty[a], kDequantWarps);
        }
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(2 * kMaxPairs));
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
        // -------------------------------------------- producer: codes, scales
        if (lane == 0) {
            RingPos c;
            uint32_t blk = 0;
            int issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int e, wt, first, count;
                unit_pairs(u, e, wt, first, count);
                for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
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
                        if (c.use > 0 && !(ok = mbar_wait(&empty_c[c.s], (c.use - 1) & 1, 21))) break;
                        mbar_expect_tx(&full_c[c.s], WM * BK * BITS / 8);
                        tma_load_3d(c_ring + c.s * prm.c_stage_bytes, &map_c, &full_c[c.s],
                                    ks * BK * BITS / 32, wt * WM, e);
                        ++issued;
                        c.next(DC);
                    }
                }
            }
            for (int j = 0; j < DC && j < issued; ++j) {  // drain the last copies
                if (--c.s < 0) { c.s = DC - 1; --c.use; }
                mbar_wait(&full_c[c.s], c.use & 1, 29);
            }
        }
    } else if (warp == kXWarp) {
        // -------------------------------------------- producer: activation rows
        RingPos x;
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
                    for (int ks = 0; ks < ksteps && ok; ++ks) {
                        if (x.use > 0 && !(ok = mbar_wait(&empty_x[x.s], (x.use - 1) & 1, 31))) break;
                        mbar_expect_tx(&full_x[x.s], static_cast<uint32_t>(groups4) * 4 * BK * 2);
                        uint8_t* xd = x_ring + x.s * X_STAGE;
                        for (int g4 = 0; g4 < groups4; ++g4)
                            tma_gather4(xd + g4 * 4 * BK * 2, &map_x, &full_x[x.s], ks * BK,
                                        s_rows[4 * g4], s_rows[4 * g4 + 1], s_rows[4 * g4 + 2],
                                        s_rows[4 * g4 + 3]);
                        ++issued;
                        x.next(DX);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            }
        }
        if (lane == 0) {
            for (int j = 0; j < DX && j < issued; ++j) {
                if (--x.s < 0) { x.s = DX - 1; --x.use; }
                mbar_wait(&full_x[x.s], x.use & 1, 30);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            RingPos x, a;
            int local = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int e, wt, first, count;
                unit_pairs(u, e, wt, first, count);
                for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs, ++local) {
                    const int cn = min(kMaxPairs, count - p0);
                    const int npad = (cn + 15) / 16 * 16;
                    const uint32_t idesc = idesc_bf16(WM, npad);
                    const int acc = local & 1;
                    const uint32_t ause = static_cast<uint32_t>(local >> 1);
                    if (ause > 0 && !(ok = mbar_wait(&acc_empty[acc], (ause - 1) & 1, 22))) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kMaxPairs);
                    for (int ks = 0; ks < ksteps; ++ks) {
                        if (!(ok = mbar_wait(&full_a[a.s], a.use & 1, 23))) break;
                        if (!(ok = mbar_wait(&full_x[x.s], x.use & 1, 24))) break;
                        tc_fence_after();
                        const uint64_t ad = sw128_desc(a_ring + a.s * A_STAGE);
                        const uint64_t bd = sw128_desc(x_ring + x.s * X_STAGE);
#pragma unroll
                        for (int kk = 0; kk < BK / UMMA_K; ++kk)
                            tc_mma(d_tmem, ad + (kk * UMMA_K * 2 >> 4), bd + (kk * UMMA_K * 2 >> 4), idesc,
                                   (ks > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&empty_a[a.s]);
                        tc_commit(&empty_x[x.s]);
                        a.next(DA);
                        x.next(DX);
                    }
                    if (ok) tc_commit(&acc_full[acc]);
                }
            }
        }
    } else if (warp < kEpilogueWarp0 + 4) {
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
                const int acc = local & 1;
                const uint32_t ause = static_cast<uint32_t>(local >> 1);
                if (!(ok = mbar_wait(&acc_full[acc], ause & 1, 25))) break;
                tc_fence_after();
                for (int c0 = 0; c0 < cn; c0 += 16) {
                    uint32_t v[16];
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                           static_cast<uint32_t>(acc * kMaxPairs + c0);
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
                if (lane == 0) mbar_arrive(&acc_empty[acc]);
            }
        }
    } else if (warp >= kDequantWarp0) {
        // ------------------------------------------------------------ dequantize
        const int dt = threadIdx.x - kDequantWarp0 * 32;  // 0 .. 511
        const int r = dt >> 2;                            // weight row within the unit
        const int qt = dt & 3;                            // k chunks 2*qt, 2*qt + 1 (16 k)
        constexpr int WPQ = BK * BITS / 32 / 4;           // code words per quarter row
        using DQ = Dequant<BITS>;
        const int64_t gpr = prm.K / prm.gs;
        RingPos c, a;
        uint32_t blk = 0;
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
                    const int gsel = (prm.gs < BK) ? (qt >> 1) : 0;  // 32-wide groups: two per k-step
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
                    // this thread's quarter row of codes, then release the code stage
                    if (!(ok = mbar_wait(&full_c[c.s], c.use & 1, 26))) break;
                    const uint8_t* cst = c_ring + c.s * prm.c_stage_bytes;
                    uint32_t w[WPQ];
                    if constexpr (BITS == 4) {
                        const uint32_t off = r * 32 + ((((qt >> 1) ^ ((r >> 2) & 1))) << 4) + (qt & 1) * 8;
                        const uint2 v2 = *reinterpret_cast<const uint2*>(cst + off);
                        w[0] = v2.x; w[1] = v2.y;
                    } else if constexpr (BITS == 8) {
                        const uint32_t off = r * 64 + ((qt ^ ((r >> 1) & 3)) << 4);
                        const uint4 v4 = *reinterpret_cast<const uint4*>(cst + off);
                        w[0] = v4.x; w[1] = v4.y; w[2] = v4.z; w[3] = v4.w;
                    } else {
                        w[0] = *reinterpret_cast<const uint32_t*>(cst + r * 16 + qt * 4);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty_c[c.s]);
                    c.next(DC);
                    if (a.use > 0 && !(ok = mbar_wait(&empty_a[a.s], (a.use - 1) & 1, 32))) break;
                    uint8_t* arow = a_ring + a.s * A_STAGE + (r >> 3) * 1024 + (r & 7) * 128;
                    const uint32_t s2 = (__float_as_uint(sc) >> 16) * 0x00010001u;
                    const uint32_t b2 = (__float_as_uint(bc) >> 16) * 0x00010001u;
                    uint32_t out[8];
                    if constexpr (BITS == 2) {
                        DQ::run(w[0], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6, out);  // 16 k
                    } else if constexpr (BITS == 4) {
                        DQ::run(w[0], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6, out);
                        DQ::run(w[1], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6, out + 4);
                    } else {
#pragma unroll
                        for (int uu = 0; uu < 4; ++uu)
                            DQ::run(w[uu], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6, out + 2 * uu);
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int ch = 2 * qt + h;
                        uint4 o;
                        o.x = out[4 * h]; o.y = out[4 * h + 1]; o.z = out[4 * h + 2]; o.w = out[4 * h + 3];
                        *reinterpret_cast<uint4*>(arow + ((ch ^ (r & 7)) << 4)) = o;
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_a[a.s]);
                    a.next(DA);
                    if (prm.sb_tma && (kb == sgk - 1 || ks == ksteps - 1)) {
                        if (lane == 0) mbar_arrive(&sb_empty[slot]);
                        ++blk;
                    }
                    if (++kb == sgk) kb = 0;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(2 * kMaxPairs));
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
    int dx = 6, dc = 8, da = 2;
    auto bytes = [&]() {
        return static_cast<size_t>(x_stage) * dx + static_cast<size_t>(c_stage) * dc +
               static_cast<size_t>(a_stage) * da + sb_ring + idx +
               static_cast<size_t>(2 * (dx + dc + da) + 8) * 8 + 16;
    };
    const size_t budget = 227 * 1024 - 2048 - 1024;
    while (bytes() > budget && (dx > 2 || dc > 2)) {
        if (dc >= dx && dc > 2) --dc; else --dx;
    }
    if (bytes() > budget) return cudaErrorInvalidConfiguration;
    prm.dx = dx;
    prm.dc = dc;
    prm.da = da;
    prm.a_off = 0;
    prm.x_off = a_stage * da;
    prm.c_off = prm.x_off + x_stage * dx;
    prm.sb_off = prm.c_off + c_stage * dc;
    prm.idx_off = prm.sb_off + sb_ring;
    prm.bar_off = prm.idx_off + idx;
    prm.c_stage_bytes = c_stage;
    const size_t smem = bytes() + 1024;
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
