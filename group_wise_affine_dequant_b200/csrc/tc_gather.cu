// Tensor-core mixture-of-experts product ("Docs / Quantization", section
// "Mixture of experts": with rows sorted by expert, a grouped kernel reads each
// expert's weights once). Each expert sees a handful of rows (tens), so the
// product is computed transposed: D^T = W_e . X_e^T with the expert's weights as
// the 128-row MMA operand A (dequantized into tensor memory) and the expert's
// gathered activation rows as the N side (16 .. 64 columns per pass). Every
// weight tile is read from HBM once and used for all of the expert's rows.
//
// Work unit: (expert e, 256 weight rows = two 128-row tiles that share every
// activation stage); a unit's pairs are taken in passes of at most 64, and K
// in steps of 128 (every pipeline handshake moves a 128-k slab: 16 MMAs, 16 KB
// of codes at 4 bits, 16 KB of activations per k-step). The
// kernel is the programmatic dependent of the routing kernel: it sets up and
// prefetches its first weights into L2 before waiting for the routing tables,
// then lets the next kernel launch (the next product of a SwiGLU block, or the
// next call's router, each of which waits for this grid before any access).
// Roles, per CTA (persistent):
//   warp 0      one lane streams the code tiles by TMA, 256 rows x 128 bytes
//               (several k-steps) per copy, into a ring released by the
//               dequantizing warps once they have read them; scales and biases
//               arrive per unit in blocks of up to 16 groups (swizzled boxes).
//   warp 1      TMEM allocation; one thread issues tcgen05.mma (M = 128,
//               N = pairs rounded up to 16, K = 16), one per tile, into a
//               double-buffered TMEM accumulator (64 columns per tile).
//   warps 2-5   epilogue: TMEM lane = weight row, column = pair; each column is
//               stored to its pair's output row (32 lanes -> 64 contiguous bytes).
//               With a gate buffer (the SwiGLU block) each warp first copies the
//               pass's gate values into its shared-memory staging area by
//               cp.async while the MMAs run, then stores silu(g) * product.
//   warps 6-9   copy the pairs' activation rows with cp.async (16 bytes per
//               thread per row and k-step) into the 128-byte-swizzled B layout;
//               each thread fences its completed copies into the async proxy
//               before it arrives on the stage's barrier.
//   warps 10-25 dequantize, one thread per (weight row, 64 k) of each tile
//               (two runs of 32 k, each inside one group), straight into
//               tensor memory (tcgen05.st): the MMA reads A from TMEM, so the
//               dequantized tiles cost no shared-memory bandwidth, and two
//               128-k A stages fit beside the two accumulators.
// At the end every CTA writes zero rows for its share of the pairs whose
// expert or token id is out of range. Waits are bounded by a timer like the
// other pipelines.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tma.cuh"

namespace nvq {
namespace {

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

using namespace tc;

constexpr int WM = 128;          // weight rows per tile (TMEM lanes)
constexpr int kTiles = 2;        // weight tiles per unit: every activation stage serves both
constexpr int UW = WM * kTiles;  // weight rows per unit
constexpr int BK = 128;
constexpr int UMMA_K = 16;
constexpr int kMaxPairs = 64;    // pairs per pass (TMEM columns of one tile's accumulator)
static_assert(kMaxPairs == 64, "the epilogue keeps two pair ids per lane");
constexpr int kEpilogueWarp0 = 2;
constexpr int kXWarp0 = 6;       // activation-row loaders: warps 6-9
constexpr int kXThreads = 128;
constexpr int kDequantWarp0 = 10; // warps 10-25: dequantize, one tile and 64 k per thread
constexpr int kDequantThreads = 512;
constexpr int kThreads = kDequantWarp0 * 32 + kDequantThreads;
constexpr uint32_t kXStage = kMaxPairs * BK * 2;  // activation stage: kMaxPairs rows x BK k (two swizzle atoms)
constexpr int kXChunks = BK * 2 / 16;         // 16-byte pieces of a row per k-step
constexpr int kXRS = kXThreads / kXChunks;    // rows a pass of the loader threads covers
constexpr uint32_t kXoffBytes = kMaxPairs / kXRS * kXThreads * 4;
constexpr uint32_t kCStage = UW * 128;         // code stage: the unit's rows x 128 code bytes
constexpr int kAccCols = kTiles * kMaxPairs;   // accumulator columns of one pass
constexpr int kACols = kTiles * (BK / 2);      // TMEM columns of one A stage (BK k per tile)
constexpr int kDA = 2;                         // A stages, in TMEM after the accumulators
constexpr uint32_t kTmemCols = 512;
static_assert(2 * kAccCols + kDA * kACols <= static_cast<int>(kTmemCols), "TMEM budget");

struct GParams {
    uint16_t* y;                // [R, N]
    // nullable: gate values g [R, N] (bf16); the stored result is then
    // silu(g) * (the product), the SwiGLU activation of a mixture-of-experts
    // block, written over g in place
    const uint16_t* act;
    const uint16_t* x;          // [x_rows, K]
    const uint32_t* lhs;        // nullable
    const uint32_t* perm;       // [R] pairs in expert order
    const uint32_t* offsets;    // [E + 2]
    int64_t N, K, E;
    int lg_gs;
    int wunits;                 // ceil(N / UW)
    int spk;                    // k-steps per code stage (128-byte code rows)
    int sbg, lg_sbw;            // groups per scale/bias box; log2 of its row bytes
    int sb_slot;                // bytes of one slot (scales + biases)
    int dx, dc, da;             // depths: activations, codes, dequantized weights
    uint32_t x_off, c_off, a_off, sb_off, bar_off, row_off;
    uint32_t g_off;             // act: gate staging, [4 warps][2 tiles][64 pairs][32 columns] bf16
};

struct RingPos {
    int s = 0;
    uint32_t use = 0;
    __device__ __forceinline__ void next(int depth) {
        if (++s == depth) { s = 0; ++use; }
    }
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
tc_gather_kernel(const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_s,
                 const __grid_constant__ CUtensorMap map_b, const GParams prm) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int DX = prm.dx, DC = prm.dc, DA = kDA;
    uint8_t* x_ring = smem + prm.x_off;
    uint8_t* c_ring = smem + prm.c_off;
    uint8_t* sb_ring = smem + prm.sb_off;
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
    // [kMaxPairs / (kXThreads / 8)][kXThreads]: x element offsets of each loader thread's rows
    uint32_t* s_xoff = reinterpret_cast<uint32_t*>(smem + prm.row_off);
    constexpr int kDequantWarps = kDequantThreads / 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < DX; ++i) { mbar_init(&full_x[i], kXThreads); mbar_init(&empty_x[i], 1); }
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
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    const int ksteps = static_cast<int>(prm.K / BK);
    const int spk = prm.spk;
    const int sgk = (prm.sbg << prm.lg_gs) / BK;  // k-steps per scale/bias block
    const int units = static_cast<int>(prm.E) * prm.wunits;

    // The launch may overlap the routing kernel (programmatic dependent
    // launch): until the wait below, touch nothing it writes. The weights of
    // the CTA's first unit do not depend on the routing, so their first code
    // stages and scale/bias block are prefetched into L2 meanwhile.
    if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < units) {
        const int e = static_cast<int>(blockIdx.x) / prm.wunits;
        const int row = (static_cast<int>(blockIdx.x) - e * prm.wunits) * UW;
        const int words = static_cast<int>(prm.K * BITS / 32);
        for (int i = 0; i < DC && i * 32 < words; ++i) tma_prefetch_3d(&map_c, i * 32, row, e);
        tma_prefetch_3d(&map_s, 0, row, e);
        tma_prefetch_3d(&map_b, 0, row, e);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // the routing tables (offsets, perm) come from the previous kernel
    // A following grouped product (the next one of a SwiGLU block) may launch
    // now: it sets up and prefetches its own weights as SMs free up, and waits
    // for this grid before it reads anything this one writes.
    pdl_launch_dependents();

    auto unit_pairs = [&](int u, int& e, int& wt, int& first, int& count) {
        e = u / prm.wunits;
        wt = u - e * prm.wunits;
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
                    int kb = 0, kc = 0;
                    for (int ks = 0; ks < ksteps && ok; ++ks) {
                        if (kb == 0) {
                            const int slot = blk & 1;
                            const uint32_t bu = blk >> 1;
                            if (bu > 0 && !(ok = mbar_wait_backoff(&sb_empty[slot], (bu - 1) & 1, 27, 512))) break;
                            const uint32_t half = static_cast<uint32_t>(prm.sb_slot) / 2;
                            mbar_expect_tx(&sb_full[slot], static_cast<uint32_t>(prm.sb_slot));
                            uint8_t* dst = sb_ring + slot * prm.sb_slot;
                            const int gcol = (ks * BK) >> prm.lg_gs;
                            tma_load_3d(dst, &map_s, &sb_full[slot], gcol, wt * UW, e);
                            tma_load_3d(dst + half, &map_b, &sb_full[slot], gcol, wt * UW, e);
                            ++blk;
                        }
                        if (++kb == sgk) kb = 0;
                        if (kc == 0) {
                            if (c.use > 0 && !(ok = mbar_wait_backoff(&empty_c[c.s], (c.use - 1) & 1, 21, 512))) break;
                            mbar_expect_tx(&full_c[c.s], kCStage);
                            tma_load_3d(c_ring + c.s * kCStage, &map_c, &full_c[c.s], ks * BK * BITS / 32,
                                        wt * UW, e);
                            ++issued;
                            c.next(DC);
                        }
                        if (++kc == spk) kc = 0;
                    }
                }
            }
            for (int j = 0; j < DC && j < issued; ++j) {  // drain the last copies
                if (--c.s < 0) { c.s = DC - 1; --c.use; }
                mbar_wait(&full_c[c.s], c.use & 1, 29);
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
                    if (ause > 0 && !(ok = mbar_wait_backoff(&acc_empty[acc], (ause - 1) & 1, 22, 256))) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
                    for (int ks = 0; ks < ksteps; ++ks) {
                        if (!(ok = mbar_wait(&full_a[a.s], a.use & 1, 23))) break;
                        if (!(ok = mbar_wait(&full_x[x.s], x.use & 1, 24))) break;
                        tc_fence_after();
                        const uint32_t at = tmem_base + 2 * kAccCols + kACols * a.s;  // A stage columns
                        const uint64_t bd = sw128_desc(x_ring + x.s * kXStage);
#pragma unroll
                        for (int tt = 0; tt < kTiles; ++tt)  // both tiles against the same activations
#pragma unroll
                            for (int kk = 0; kk < BK / UMMA_K; ++kk)  // 16 k = 8 TMEM columns of A; B: 4 per 128-byte atom
                                tc_mma_ts(d_tmem + tt * kMaxPairs, at + tt * (BK / 2) + kk * (UMMA_K / 2),
                                          bd + static_cast<uint64_t>((kk >> 2) * (kMaxPairs * 128 >> 4)) +
                                              (((kk & 3) * UMMA_K * 2) >> 4),
                                          idesc, (ks > 0 || kk > 0) ? 1u : 0u);
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
        int local = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs, ++local) {
                const int cn = min(kMaxPairs, count - p0);
                const int acc = local & 1;
                const uint32_t ause = static_cast<uint32_t>(local >> 1);
                // output rows of the pass's pairs, loaded while the products
                // run: lane l holds those of columns l and l + 32
                uint32_t prow[kMaxPairs / 32];
#pragma unroll
                for (int h = 0; h < kMaxPairs / 32; ++h) {
                    const int c = h * 32 + lane;
                    prow[h] = c < cn ? __ldg(prm.perm + first + p0 + c) : 0u;
                }
                if (prm.act) {
                    // SwiGLU: bring the pass's gate values into L2 while the
                    // products run (each is read once, below, then overwritten)
                    for (int tt = 0; tt < kTiles; ++tt) {
                        const int64_t n = static_cast<int64_t>(wt) * UW + tt * WM + q * 32 + lane;
                        for (int c = 0; c < cn; ++c) {
                            const uint32_t pair = __shfl_sync(0xffffffffu, (c >> 5) ? prow[1] : prow[0], c & 31);
                            if (n < prm.N) prefetch_l2(prm.act + static_cast<int64_t>(pair) * prm.N + n);
                        }
                    }
                }
                // SwiGLU: the pass's gate values (this warp's 32 columns of both
                // tiles, every pair) are copied into the warp's staging area while
                // the products run, 4 bytes a lane (lanes 0-15 one pair, 16-31 the
                // next), before any output of the pass is written over them
                const uint32_t gst = smem_u32(smem + prm.g_off) + static_cast<uint32_t>(q) * (kTiles * kMaxPairs * 64);
                if (prm.act) {
#pragma unroll
                    for (int tt = 0; tt < kTiles; ++tt) {
                        const int64_t n0 = static_cast<int64_t>(wt) * UW + tt * WM + q * 32;
                        if (n0 < prm.N) {
                            for (int c = 0; c < cn; c += 2) {
                                const int ci = c + (lane >> 4);
                                const uint32_t pair = __shfl_sync(0xffffffffu, (ci >> 5) ? prow[1] : prow[0], ci & 31);
                                const int64_t col = n0 + (lane & 15) * 2;  // columns col, col + 1
                                const uint16_t* src = prm.act + static_cast<int64_t>(pair) * prm.N + col;
                                const uint32_t dst = gst + (tt * kMaxPairs + ci) * 64 + (lane & 15) * 4;
                                if (ci < cn) {
                                    if ((prm.N & 1) == 0 && col + 1 < prm.N) {
                                        cp_async4(dst, src);  // 4-byte aligned: N and col even
                                    } else {                  // odd N or the last column
                                        for (int h = 0; h < 2; ++h)
                                            if (col + h < prm.N)
                                                asm volatile("st.shared.u16 [%0], %1;" ::"r"(dst + 2 * h),
                                                             "h"(src[h]) : "memory");
                                    }
                                }
                            }
                        }
                    }
                    cp_async_commit();
                }
                if (!(ok = mbar_wait_backoff(&acc_full[acc], ause & 1, 25, 2048))) break;
                tc_fence_after();
                if (prm.act) {
                    cp_async_wait<0>();
                    __syncwarp();
                }
                float gv[16];
                for (int tt = 0; tt < kTiles; ++tt)
                for (int c0 = 0; c0 < cn; c0 += 16) {
                    // weight row of the unit = tile * 128 + TMEM lane
                    const int64_t n = static_cast<int64_t>(wt) * UW + tt * WM + q * 32 + lane;
                    const uint32_t rows = (c0 >> 5) ? prow[1] : prow[0];
                    if (prm.act) {  // the chunk's 16 gate values from the staging area
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            uint16_t gb;
                            asm volatile("ld.shared.u16 %0, [%1];"
                                         : "=h"(gb)
                                         : "r"(gst + (tt * kMaxPairs + c0 + j) * 64 + lane * 2));
                            gv[j] = bf16_bits_to_f32(gb);
                        }
                    }
                    uint32_t v[16];
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                           static_cast<uint32_t>(acc * kAccCols + tt * kMaxPairs + c0);
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                          "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                          "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                        : "r"(taddr));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    if (prm.act) {
                        // silu(g) * u = g / (1 + e^-g) * u, for all 16 columns at once
                        // (no branch between them); fast exponential and division,
                        // within a few ulp in fp32
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            v[j] = __float_as_uint(__fdividef(gv[j], 1.0f + __expf(-gv[j])) * __uint_as_float(v[j]));
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint32_t pair = __shfl_sync(0xffffffffu, rows, (c0 + j) & 31);
                        if (c0 + j < cn && n < prm.N)
                            prm.y[static_cast<int64_t>(pair) * prm.N + n] = f32_to_bf16_bits(__uint_as_float(v[j]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[acc]);
            }
        }
    } else if (warp < kDequantWarp0) {
        // ------------------------------------------- activation rows (cp.async)
        // Thread i copies 16-byte chunk (i & 7) of rows (i >> 3) + 16 j of every
        // k-step. Stages are completed in order, LAG k-steps behind the copies.
        const int xt = threadIdx.x - kXWarp0 * 32;  // 0 .. kXThreads - 1
        constexpr int RS = kXRS;                     // row stride between a thread's rows
        const int ch = xt % kXChunks, r0 = xt / kXChunks;
        const int lag = DX - 1 < 3 ? DX - 1 : 3;
        RingPos x, done;  // next stage to fill, next stage to complete
        int pending = 0;
        bool ok = true;
        auto complete_one = [&]() {
            fence_proxy_async();
            mbar_arrive(&full_x[done.s]);
            done.next(DX);
            --pending;
        };
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
                const int cn = min(kMaxPairs, count - p0);
                const int nr = cn > r0 ? (cn - r0 + RS - 1) / RS : 0;  // rows of this thread
                // offsets of this thread's rows, once per pass, into its own slots
                // of shared memory (no other thread reads them: no barrier)
                for (int j = 0; j < nr; ++j) {
                    const uint32_t pair = __ldg(prm.perm + first + p0 + r0 + RS * j);
                    const uint32_t row = prm.lhs ? __ldg(prm.lhs + pair) : pair;
                    // in 16-byte units (K is a multiple of 64): x up to 2^35 elements
                    s_xoff[j * kXThreads + xt] = row * static_cast<uint32_t>(prm.K / 8) + ch;
                }
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (x.use > 0 && !(ok = mbar_wait_backoff(&empty_x[x.s], (x.use - 1) & 1, 31, 256))) break;
                    uint8_t* dst = x_ring + x.s * kXStage;
                    for (int j = 0; j < nr; ++j) {
                        const int r = r0 + RS * j;
                        cp_async16(dst + (ch >> 3) * (kMaxPairs * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                                       (((ch & 7) ^ (r & 7)) << 4),
                                   reinterpret_cast<const uint4*>(prm.x) + s_xoff[j * kXThreads + xt] +
                                       ks * (BK / 8));
                    }
                    cp_async_commit();
                    x.next(DX);
                    if (++pending > lag) {
                        // the oldest of the lag + 1 outstanding groups has landed
                        if (lag == 4) cp_async_wait<4>();
                        else if (lag == 3) cp_async_wait<3>();
                        else if (lag == 2) cp_async_wait<2>();
                        else cp_async_wait<0>();
                        complete_one();
                    }
                }
            }
        }
        cp_async_wait<0>();
        while (pending > 0) complete_one();
    } else {
        // ------------------------------------------------------------ dequantize
        // warp w writes TMEM lanes 32 (w % 4) ..: row = its lane there; the
        // four warps of each lane quarter take (tile, 32-k half) of a k-step
        const int r = 32 * (warp & 3) + lane;                 // weight row within a tile
        const int dw = warp - kDequantWarp0;                  // 0 .. 15
        const int tt = (dw >> 2) & 1;                         // tile of the unit
        const int hf = dw >> 3;                               // k 32 hf .. 32 hf + 31
        const int rr = tt * WM + r;                           // row within the unit
        const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        using DQ = Dequant<BITS>;
        RingPos c, a;
        uint32_t blk = 0;
        bool ok = true;
        const uint32_t half = static_cast<uint32_t>(prm.sb_slot) / 2;
        // this thread's fixed parts of the scale/bias box offsets (row rr, the
        // box's swizzle by row width) and of its code row (128-byte swizzle)
        const int lg = prm.lg_sbw;
        const uint32_t sb_row = static_cast<uint32_t>(rr) << lg;
        const uint32_t sb_x = lg == 7 ? (rr & 7) : lg == 6 ? ((rr >> 1) & 3) : lg == 5 ? ((rr >> 2) & 1) : 0;
        const uint32_t c_row = static_cast<uint32_t>(rr) * 128;
        const uint32_t r7 = static_cast<uint32_t>(r & 7);
        const bool two_groups = prm.lg_gs == 5;  // the two 32-k runs lie in different groups
        auto sb_off = [&](int gc) {
            const uint32_t o = static_cast<uint32_t>(gc) * 2;
            return sb_row + (((o >> 4) ^ sb_x) << 4) + (o & 15);
        };
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
                int kb = 0, kc = 0, gb = 0;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int slot = blk & 1;
                    if (kb == 0) {
                        if (!(ok = mbar_wait_backoff(&sb_full[slot], (blk >> 1) & 1, 28, 256))) break;
                        gb = (ks * BK) >> prm.lg_gs;  // first group of the block
                    }
                    const uint8_t* ss = sb_ring + slot * prm.sb_slot;
                    if (kc == 0 && !(ok = mbar_wait(&full_c[c.s], c.use & 1, 26))) break;
                    // this thread's 64 k of its row (part kc of the code rows), as two
                    // runs of 32 k, each inside one group (groups are multiples of 32)
                    constexpr int NW = BITS;  // code words per 32 k
                    uint32_t w[2][NW];
                    uint32_t sv[2], bv[2];  // bf16 bits of the runs' scales and biases
                    {
                        const uint32_t so = sb_off(((ks * BK + 64 * hf) >> prm.lg_gs) - gb);
                        sv[0] = sv[1] = *reinterpret_cast<const uint16_t*>(ss + so);
                        bv[0] = bv[1] = *reinterpret_cast<const uint16_t*>(ss + half + so);
                        if (two_groups) {
                            const uint32_t so1 = sb_off(((ks * BK + 64 * hf) >> prm.lg_gs) + 1 - gb);
                            sv[1] = *reinterpret_cast<const uint16_t*>(ss + so1);
                            bv[1] = *reinterpret_cast<const uint16_t*>(ss + half + so1);
                        }
                    }
                    const uint8_t* crow = c_ring + c.s * kCStage + c_row;
                    // 16-byte chunk of run 0 in the row: o = kc * (BK BITS / 8) + 64 hf BITS / 8
                    const uint32_t o0 = static_cast<uint32_t>(kc * (BK * BITS / 8) + 64 * hf * BITS / 8);
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const uint32_t o = o0 + 32 * h2 * BITS / 8;
                        if constexpr (BITS == 4) {
                            const uint4 v4 = *reinterpret_cast<const uint4*>(crow + (((o >> 4) ^ r7) << 4));
                            w[h2][0] = v4.x; w[h2][1] = v4.y; w[h2][2] = v4.z; w[h2][3] = v4.w;
                        } else if constexpr (BITS == 8) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint4 v4 = *reinterpret_cast<const uint4*>(
                                    crow + ((((o >> 4) + h) ^ r7) << 4));
                                w[h2][4 * h] = v4.x; w[h2][4 * h + 1] = v4.y;
                                w[h2][4 * h + 2] = v4.z; w[h2][4 * h + 3] = v4.w;
                            }
                        } else {
                            const uint2 v2 = *reinterpret_cast<const uint2*>(
                                crow + (((o >> 4) ^ r7) << 4) + (o & 15));
                            w[h2][0] = v2.x; w[h2][1] = v2.y;
                        }
                    }
                    const bool last_part = (kc == spk - 1) || (ks == ksteps - 1);
                    if (last_part) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&empty_c[c.s]);
                        c.next(DC);
                    }
                    if (++kc == spk) kc = 0;
                    if (a.use > 0 && !(ok = mbar_wait_backoff(&empty_a[a.s], (a.use - 1) & 1, 32, 128))) break;
                    tc_fence_after();
                    const uint32_t s2[2] = {sv[0] * 0x00010001u, sv[1] * 0x00010001u};
                    const uint32_t b2[2] = {bv[0] * 0x00010001u, bv[1] * 0x00010001u};
                    // one dequantizer for the warp's step: the fast form when every
                    // lane's groups allow it (same results either way)
                    const bool fast = __all_sync(__activemask(), dq_fast_ok(s2[0]) && dq_fast_ok(s2[1]));
                    const uint32_t ta = tmem_base + lane_addr + 2 * kAccCols + kACols * a.s + (BK / 2) * tt + 32 * hf;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t out[16];
                        if (fast) {
#pragma unroll
                            for (int i = 0; i < NW; ++i) DQ::run_fast(w[h2][i], s2[h2], b2[h2], out + i * DQ::PAIRS);
                        } else {
                            const float sc = __uint_as_float(sv[h2] << 16), bc = __uint_as_float(bv[h2] << 16);
#pragma unroll
                            for (int i = 0; i < NW; ++i)
                                DQ::run(w[h2][i], s2[h2], b2[h2], sc, bc, 2u, 4u, 6u, out + i * DQ::PAIRS);
                        }
                        tmem_st_x16_async(ta + 16 * h2, out);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_a[a.s]);
                    a.next(DA);
                    if (kb == sgk - 1 || ks == ksteps - 1) {
                        if (lane == 0) mbar_arrive(&sb_empty[slot]);
                        ++blk;
                    }
                    if (++kb == sgk) kb = 0;
                }
            }
        }
    }

    // pairs whose expert or token id is out of range (the router's last
    // bucket) get zero rows
    {
        const int64_t first = __ldg(prm.offsets + prm.E), last = __ldg(prm.offsets + prm.E + 1);
        for (int64_t i = first + blockIdx.x; i < last; i += gridDim.x) {
            uint16_t* row = prm.y + static_cast<int64_t>(__ldg(prm.perm + i)) * prm.N;
            for (int64_t n = threadIdx.x; n < prm.N; n += blockDim.x) row[n] = 0;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols));
    }
}

}  // namespace

bool tc_gather_supported(int64_t K, int64_t N, int bits, int gs) {
    // scale rows must be 16-byte multiples for their TMA boxes
    return K % BK == 0 && K >= BK && N > 0 && (bits == 2 || bits == 4 || bits == 8) &&
           (gs == 32 || gs == 64 || gs == 128) && (K / gs) % 8 == 0;
}

unsigned int tc_gather_error_take() { return pipeline_error_take(); }

cudaError_t launch_tc_gather(const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs,
                             const uint32_t* perm, const uint32_t* offsets, int64_t E, int64_t N,
                             const uint32_t* codes, const void* scales, const void* biases, int gs,
                             int bits, void* y, cudaStream_t stream, int num_sms,
                             const void* act_gate) {
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    if (x_rows * K >= (int64_t(1) << 35)) return cudaErrorInvalidValue;  // 32-bit 16-byte offsets
    CUtensorMap map_c, map_s, map_b;
    const int64_t wpr = K * bits / 32, gpr = K / gs;
    {   // code rows of 128 bytes (several k-steps), 128-byte swizzle
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(wpr) * 4, static_cast<cuuint64_t>(wpr * N) * 4};
        cuuint32_t box[3] = {32, UW, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&map_c, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(codes), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    // scale/bias boxes: up to 32 groups (64 bytes) per row, swizzled by row width
    const int sbg = gpr >= 16 ? 16 : static_cast<int>(gpr);
    const int sbw = sbg * 2;
    const int lg_sbw = sbw == 128 ? 7 : sbw == 64 ? 6 : sbw == 32 ? 5 : 4;
    {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(gpr), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(gpr) * 2, static_cast<cuuint64_t>(gpr * N) * 2};
        cuuint32_t box[3] = {static_cast<cuuint32_t>(sbg), UW, 1};
        cuuint32_t es[3] = {1, 1, 1};
        const CUtensorMapSwizzle swz = lg_sbw == 7   ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : lg_sbw == 6 ? CU_TENSOR_MAP_SWIZZLE_64B
                                       : lg_sbw == 5 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                     : CU_TENSOR_MAP_SWIZZLE_NONE;
        for (int i = 0; i < 2; ++i)
            if (enc(i ? &map_b : &map_s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                    const_cast<void*>(i ? biases : scales), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
    }
    GParams prm{};
    prm.y = static_cast<uint16_t*>(y);
    prm.act = static_cast<const uint16_t*>(act_gate);
    prm.x = static_cast<const uint16_t*>(x);
    prm.lhs = lhs;
    prm.perm = perm;
    prm.offsets = offsets;
    prm.N = N;
    prm.K = K;
    prm.E = E;
    prm.lg_gs = gs == 32 ? 5 : gs == 64 ? 6 : 7;
    prm.wunits = static_cast<int>((N + UW - 1) / UW);
    prm.spk = 128 / (BK * bits / 8);  // k-steps per 128-byte code row: 8, 4, 2
    prm.sbg = sbg;
    prm.lg_sbw = lg_sbw;
    prm.sb_slot = 2 * UW * sbw;
    const size_t sb_ring = 2u * static_cast<size_t>(prm.sb_slot);
    int dx = 7, dc = 2;
    // SwiGLU: the epilogue warps' gate staging, 4 x 2 x 64 pairs x 64 bytes
    const size_t g_bytes = act_gate ? static_cast<size_t>(4 * kTiles * kMaxPairs * 64) : 0;
    auto bytes = [&]() {
        return static_cast<size_t>(kXStage) * dx + static_cast<size_t>(kCStage) * dc + sb_ring +
               kXoffBytes + g_bytes +
               static_cast<size_t>(2 * (dx + dc + kDA) + 8) * 8 + 16;
    };
    const size_t budget = 227 * 1024 - 2048 - 1024;
    while (bytes() > budget && dx > 3) --dx;
    if (bytes() > budget) return cudaErrorInvalidConfiguration;
    prm.dx = dx;
    prm.dc = dc;
    prm.da = kDA;
    prm.x_off = 0;
    prm.c_off = kXStage * dx;
    prm.a_off = 0;  // A stages live in TMEM
    prm.sb_off = prm.c_off + kCStage * dc;
    prm.row_off = prm.sb_off + static_cast<uint32_t>(sb_ring);
    prm.g_off = prm.row_off + kXoffBytes;
    prm.bar_off = prm.g_off + static_cast<uint32_t>(g_bytes);
    const size_t smem = bytes() + 1024;
    const int units = static_cast<int>(E) * prm.wunits;
    const int grid = units < num_sms ? units : num_sms;
    void (*k)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const GParams) =
        bits == 4 ? tc_gather_kernel<4> : bits == 8 ? tc_gather_kernel<8> : tc_gather_kernel<2>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // Programmatic dependent launch on the routing kernel: the CTAs set up
    // (barriers, tensor memory, L2 prefetch of their first weights) while the
    // routing runs and wait for its tables with griddepcontrol.wait.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, map_c, map_s, map_b, prm);
}

}  // namespace nvq
