// Tensor-core mixture-of-experts product with quantized experts stored [K, N]
// (gather_qmm with transpose = 0: "Docs / Quantization", section "Mixture of
// experts", each row meets its own expert's weights; the product's transpose
// flag, section "Affine", and the crate docs' GatherQmm take either layout).
// The experts are [E][K, N], grouped along N, so the scale varies along the
// contraction. The same grouped, transposed form as the other grouped kernels:
// D^T = W_e . X_e^T with 256 weight columns n (two 128-row tiles) as the MMA's
// M side and the expert's gathered activation rows (<= 64 per pass) as N, so
// each expert's weights cross HBM once for all its rows. Roles, per CTA
// (persistent):
//   warp 0      one lane streams code boxes of 64 k-rows x 256 columns by TMA
//               (with the boxes of scales and biases that cover the unit,
//               when N / gs is a multiple of 8) into a ring released by the
//               dequantizing warps; the warp prefetches later stages into L2.
//   warp 1      TMEM allocation; one thread issues tcgen05.mma (M = 128,
//               N = pairs rounded up to 16, K = 16) with both operands in
//               shared memory, two tiles per k-step, into a double-buffered
//               accumulator (64 columns per tile).
//   warps 2-5   epilogue: TMEM lane = A-tile row (a permutation of the unit's
//               columns), column = pair; each pair's value is stored to its
//               output row.
//   warps 6-9   copy the pairs' activation rows with cp.async into the
//               128-byte-swizzled B layout.
//   warps 10-25 dequantize and transpose, as two groups of eight warps on
//               alternate stages: each column's 4 consecutive k-values
//               w = s[k, g(n)] * code + b[k, g(n)] (one bf16 fma on the exact
//               code, rounded once) go to the column's row of the K-major A
//               tile as one 8-byte piece.
// The kernel is the programmatic dependent of the routing kernel. Pairs with
// an out-of-range id get zero rows. Waits are bounded by a timer.
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

constexpr int WM = 128;          // weight rows per tile (TMEM lanes)
constexpr int kTiles = 2;        // tiles per unit, sharing every activation stage
constexpr int UW = WM * kTiles;  // weight rows per unit
constexpr int BK = 64;           // k per stage: one 128-byte swizzle atom of bf16
constexpr int UMMA_K = 16;
constexpr int kMaxPairs = 64;    // pairs per pass (accumulator columns per tile)
static_assert(kMaxPairs == 64, "the epilogue keeps two pair ids per lane");
constexpr int kXWarp0 = 6;       // activation-row loaders: warps 6-9
constexpr int kXThreads = 128;
constexpr int kDequantWarp0 = 10; // warps 10-25: dequantize into the A tiles
constexpr int kDequantThreads = 512;
constexpr int kDequantGroups = 2; // groups of dequantizing warps on alternate stages
constexpr int kL2Ahead = 8;       // stages prefetched into L2 ahead of the code copies
constexpr int kThreads = kDequantWarp0 * 32 + kDequantThreads;  // 832
constexpr int kWStage = UW * BK * 2;                  // 32 KB of dequantized weights per stage
constexpr int kXStage = kMaxPairs * BK * 2;           // 8 KB of activations per stage
constexpr int kAccCols = kTiles * kMaxPairs;          // 128 columns per accumulator
constexpr uint32_t kTmemCols = 2 * kAccCols;          // double-buffered: 256

struct TParams {
    uint16_t* y;                // [R, N]
    const uint16_t* scales;     // [E][K, N / gs]
    const uint16_t* biases;
    int gs, lg_gs;
    int dc;                     // code ring depth
    uint32_t c_off;
    uint32_t c_stage;           // bytes of one code stage (64 k-rows x 256 columns)
    uint32_t sb_off;            // staged scales and biases (STAGED): 2 KB per code stage
    const uint16_t* x;          // [x_rows, K]
    const uint32_t* lhs;        // nullable
    const uint32_t* perm;       // [R] pairs in expert order
    const uint32_t* offsets;    // [E + 2]
    int64_t N, K, E;
    int wunits;                 // ceil(N / UW)
    int dw, dx;                 // ring depths: weights, activations
    uint32_t x_off, w_off, row_off, bar_off;
};

struct RingPos {
    int s = 0;
    uint32_t use = 0;
    __device__ __forceinline__ void next(int depth) {
        if (++s == depth) { s = 0; ++use; }
    }
};

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint32_t vmin_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Row of the A tiles that holds column n of a unit, and (being an involution)
// the column that TMEM lane (tile * 128 + lane) holds: the low three bits are
// XORed with three bits above them, those of the code word index for 2- and
// 4-bit codes.
template <int BITS>
__device__ __forceinline__ int a_row(int n) {
    constexpr int S = BITS == 2 ? 4 : 3;
    return n ^ ((n >> S) & 7);
}

// STAGED (N / gs a multiple of 8): each stage's scales and biases arrive by
// TMA with its codes, as [64 k-rows][8 groups] boxes that cover the unit's
// groups; otherwise the dequantizers read them from global memory.
template <int BITS, bool STAGED>
__global__ void __launch_bounds__(kThreads, 1)
tc_gather_t0_kernel(const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_s,
                    const __grid_constant__ CUtensorMap map_b, const TParams prm) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int DW = prm.dw, DX = prm.dx, DC = prm.dc;
    uint8_t* x_ring = smem + prm.x_off;
    uint8_t* w_ring = smem + prm.w_off;
    uint8_t* c_ring = smem + prm.c_off;
    uint8_t* sb_ring = smem + prm.sb_off;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prm.bar_off);
    uint64_t* full_w = bars;
    uint64_t* empty_w = full_w + DW;
    uint64_t* full_x = empty_w + DW;
    uint64_t* empty_x = full_x + DX;
    uint64_t* full_c = empty_x + DX;
    uint64_t* empty_c = full_c + DC;
    uint64_t* acc_full = empty_c + DC;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    // [kMaxPairs / (kXThreads / 8)][kXThreads]: x element offsets of each loader thread's rows
    uint32_t* s_xoff = reinterpret_cast<uint32_t*>(smem + prm.row_off);

    if (threadIdx.x == 0) {
        // a stage is dequantized by one group of warps
        for (int i = 0; i < DW; ++i) { mbar_init(&full_w[i], kDequantThreads / 32 / kDequantGroups); mbar_init(&empty_w[i], 1); }
        for (int i = 0; i < DC; ++i) { mbar_init(&full_c[i], 1); mbar_init(&empty_c[i], kDequantThreads / 32 / kDequantGroups); }
        for (int i = 0; i < DX; ++i) { mbar_init(&full_x[i], kXThreads); mbar_init(&empty_x[i], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], 4); }
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    const int ksteps = static_cast<int>(prm.K / BK);
    const int units = static_cast<int>(prm.E) * prm.wunits;

    // Before the routing tables exist: L2 prefetch of the first unit's first
    // code stages (the weights do not depend on the routing).
    if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < units) {
        const int e = static_cast<int>(blockIdx.x) / prm.wunits;
        const int col = (static_cast<int>(blockIdx.x) - e * prm.wunits) * UW;
        for (int i = 0; i < kL2Ahead && i < ksteps; ++i) tma_prefetch_3d(&map_c, col * BITS / 32, i * BK, e);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // the routing tables (offsets, perm) come from the previous kernel

    auto unit_pairs = [&](int u, int& e, int& wt, int& first, int& count) {
        e = u / prm.wunits;
        wt = u - e * prm.wunits;
        first = static_cast<int>(__ldg(prm.offsets + e));
        count = static_cast<int>(__ldg(prm.offsets + e + 1)) - first;
    };

    if (warp == 0) {
        // --------------------------------------------------- producer: codes
        // Lane 0 copies the code box of each stage. The warp also prefetches
        // into L2, kL2Ahead stages ahead of the copies (into the next unit at
        // the end of one), the code box and the 64 rows of the unit's scales
        // and biases (first and last element of each row), so the copies and
        // the dequantizers' loads meet L2 rather than HBM: the ring alone
        // holds too few bytes in flight to cover HBM's latency.
        const int64_t gpr = prm.N >> prm.lg_gs;
        const int gu = UW >> prm.lg_gs;  // groups of a unit
        auto prefetch_stage = [&](int u2, int ks2) {
            const int e2 = u2 / prm.wunits, wt2 = u2 - e2 * prm.wunits;
            if (lane == 0) tma_prefetch_3d(&map_c, wt2 * UW * BITS / 32, ks2 * BK, e2);
            if constexpr (STAGED) {
                if (lane == 0) {
                    tma_prefetch_3d(&map_s, (wt2 * gu) & ~7, ks2 * BK, e2);
                    tma_prefetch_3d(&map_b, (wt2 * gu) & ~7, ks2 * BK, e2);
                }
                return;
            }
            const int64_t g0 = static_cast<int64_t>(wt2) * gu;
            const int64_t g1 = min(g0 + gu, gpr) - 1;
#pragma unroll
            for (int h = 0; h < BK / 32; ++h) {
                const int64_t row = (static_cast<int64_t>(e2) * prm.K + ks2 * BK + h * 32 + lane) * gpr;
                prefetch_l2(prm.scales + row + g0);
                prefetch_l2(prm.scales + row + g1);
                prefetch_l2(prm.biases + row + g0);
                prefetch_l2(prm.biases + row + g1);
            }
        };
        if (static_cast<int>(blockIdx.x) < units)
            for (int i = 0; i < kL2Ahead && i < ksteps; ++i) prefetch_stage(blockIdx.x, i);
        RingPos c;
        int issued = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (lane == 0) {
                        if (c.use > 0) ok = mbar_wait_backoff(&empty_c[c.s], (c.use - 1) & 1, 61, 512);
                        if (ok) {
                            mbar_expect_tx(&full_c[c.s], prm.c_stage + (STAGED ? 2048u : 0u));
                            tma_load_3d(c_ring + c.s * prm.c_stage, &map_c, &full_c[c.s],
                                        wt * UW * BITS / 32, ks * BK, e);
                            if constexpr (STAGED) {
                                uint8_t* sbs = sb_ring + c.s * 2048;
                                tma_load_3d(sbs, &map_s, &full_c[c.s], (wt * gu) & ~7, ks * BK, e);
                                tma_load_3d(sbs + 1024, &map_b, &full_c[c.s], (wt * gu) & ~7, ks * BK, e);
                            }
                            ++issued;
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    if (ks + kL2Ahead < ksteps) prefetch_stage(u, ks + kL2Ahead);
                    else if (p0 + kMaxPairs >= count && u + static_cast<int>(gridDim.x) < units &&
                             ks + kL2Ahead - ksteps < ksteps)
                        prefetch_stage(u + gridDim.x, ks + kL2Ahead - ksteps);
                    c.next(DC);
                }
            }
        }
        if (lane == 0) {
            for (int j = 0; j < DC && j < issued; ++j) {  // drain the last copies
                if (--c.s < 0) { c.s = DC - 1; --c.use; }
                mbar_wait(&full_c[c.s], c.use & 1, 69);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            RingPos w, x;
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
                    if (ause > 0 && !(ok = mbar_wait_backoff(&acc_empty[acc], (ause - 1) & 1, 42, 256))) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
                    for (int ks = 0; ks < ksteps; ++ks) {
                        if (!(ok = mbar_wait(&full_w[w.s], w.use & 1, 43))) break;
                        if (!(ok = mbar_wait(&full_x[x.s], x.use & 1, 44))) break;
                        tc_fence_after();
                        const uint64_t bd = sw128_desc(x_ring + x.s * kXStage);
#pragma unroll
                        for (int tt = 0; tt < kTiles; ++tt) {  // both tiles against the same activations
                            const uint64_t ad = sw128_desc(w_ring + w.s * kWStage + tt * (WM * BK * 2));
#pragma unroll
                            for (int kk = 0; kk < BK / UMMA_K; ++kk)  // 16 k = 32 bytes of each row
                                tc_mma(d_tmem + tt * kMaxPairs, ad + (kk * UMMA_K * 2 >> 4),
                                       bd + (kk * UMMA_K * 2 >> 4), idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                        }
                        tc_commit(&empty_w[w.s]);
                        tc_commit(&empty_x[x.s]);
                        w.next(DW);
                        x.next(DX);
                    }
                    if (ok) tc_commit(&acc_full[acc]);
                }
            }
        }
    } else if (warp < 6) {
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
                // output rows of the pass's pairs: lane l holds columns l and l + 32
                uint32_t prow[kMaxPairs / 32];
#pragma unroll
                for (int h = 0; h < kMaxPairs / 32; ++h) {
                    const int c = h * 32 + lane;
                    prow[h] = c < cn ? __ldg(prm.perm + first + p0 + c) : 0u;
                }
                if (!(ok = mbar_wait_backoff(&acc_full[acc], ause & 1, 45, 2048))) break;
                tc_fence_after();
                for (int tt = 0; tt < kTiles; ++tt)
                for (int c0 = 0; c0 < cn; c0 += 16) {
                    // column of W held by TMEM lane (tile * 128 + lane)
                    const int64_t n = static_cast<int64_t>(wt) * UW + a_row<BITS>(tt * WM + q * 32 + lane);
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
                    const uint32_t rows = (c0 >> 5) ? prow[1] : prow[0];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint32_t pair = __shfl_sync(0xffffffffu, rows, (c0 + j) & 31);
                        if (c0 + j < cn && n < prm.N)
                            prm.y[static_cast<int64_t>(pair) * prm.N + n] =
                                f32_to_bf16_bits(__uint_as_float(v[j]));
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
        constexpr int RS = kXThreads / 8;            // row stride between a thread's rows
        const int ch = xt & 7, r0 = xt >> 3;
        const int lag = DX - 1 < 4 ? DX - 1 : 4;
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
                for (int j = 0; j < nr; ++j) {
                    const uint32_t pair = __ldg(prm.perm + first + p0 + r0 + RS * j);
                    const uint32_t row = prm.lhs ? __ldg(prm.lhs + pair) : pair;
                    // in 16-byte units (K is a multiple of 64): x up to 2^35 elements
                    s_xoff[j * kXThreads + xt] = row * static_cast<uint32_t>(prm.K / 8) + ch;
                }
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (x.use > 0 && !(ok = mbar_wait_backoff(&empty_x[x.s], (x.use - 1) & 1, 46, 256))) break;
                    uint8_t* dst = x_ring + x.s * kXStage;
                    for (int j = 0; j < nr; ++j) {
                        const int r = r0 + RS * j;
                        cp_async16(dst + (r >> 3) * 1024 + (r & 7) * 128 + ((ch ^ (r & 7)) << 4),
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
        // ------------------------------------------ dequantize and transpose
        // Two groups of 8 warps take alternate stages, so one group's loads of
        // scales and biases overlap the other's arithmetic. A warp task is 16
        // code words x 8 k-rows: lane l takes word j = 16 jh + (l >> 1) and
        // k-rows 4 kq .. 4 kq + 3 with kq = 2 kh + (l & 1). Column n of the unit
        // goes to A-row a_row(n) (an involution on the low three bits), so each
        // half-warp's 8-byte stores cover the 32 banks once; the code reads are
        // two-way.
        constexpr int PER = 32 / BITS;
        constexpr int WPR = UW * BITS / 32;          // code words per k-row of a stage
        constexpr int WTASKS = (WPR / 16) * (BK / 8);
        constexpr int GW = kDequantThreads / 32 / kDequantGroups;  // warps per group
        const int dw = warp - kDequantWarp0;          // 0 .. 15
        const int grp = dw / GW, wig = dw % GW;
        const int jl = lane >> 1, kl = lane & 1;
        const int64_t gpr = prm.N >> prm.lg_gs;       // groups per k-row of W
        RingPos c, w;
        bool ok = true;
        int st = 0;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int e, wt, first, count;
            unit_pairs(u, e, wt, first, count);
            const uint16_t* se = prm.scales + static_cast<int64_t>(e) * prm.K * gpr;
            const uint16_t* be = prm.biases + static_cast<int64_t>(e) * prm.K * gpr;
            for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
                for (int ks = 0; ks < ksteps; ++ks, c.next(DC), w.next(DW)) {
                    if (st++ % kDequantGroups != grp) continue;
                    if (!(ok = mbar_wait(&full_c[c.s], c.use & 1, 62))) break;
                    if (w.use > 0 && !(ok = mbar_wait_backoff(&empty_w[w.s], (w.use - 1) & 1, 63, 128))) break;
                    const uint8_t* cst = c_ring + c.s * prm.c_stage;
                    const uint32_t wst = smem_u32(w_ring + w.s * kWStage);
#pragma unroll
                    for (int mt = 0; mt < WTASKS / GW; ++mt) {
                        const int wtask = wig + mt * GW;
                        const int j = (wtask / (BK / 8)) * 16 + jl;
                        const int kq = (wtask % (BK / 8)) * 2 + kl;
                        const int64_t ng = static_cast<int64_t>(wt) * UW + j * PER;  // first column in W
                        // scales and biases of k-rows kg .. kg + 3 in the words' group
                        // (a word past N reads column N - 1's: its outputs are dropped)
                        const uint32_t kg = static_cast<uint32_t>(ks * BK + 4 * kq);
                        const uint32_t gc = static_cast<uint32_t>((ng < prm.N ? ng : prm.N - 1) >> prm.lg_gs);
                        const uint32_t o = kg * static_cast<uint32_t>(gpr) + gc;
                        uint32_t cw[4], sraw[4], braw[4];
                        // staged: [64 k-rows][8 groups] from group (wt * gu) & ~7 on, scales
                        // then biases
                        const uint16_t* sbs = reinterpret_cast<const uint16_t*>(sb_ring + c.s * 2048) + 4 * kq * 8 +
                                              (gc & 7);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            cw[i] = *reinterpret_cast<const uint32_t*>(cst + (4 * kq + i) * (WPR * 4) + 4 * j);
                            if constexpr (STAGED) {
                                sraw[i] = sbs[i * 8];
                                braw[i] = sbs[512 + i * 8];
                            } else {
                                sraw[i] = __ldg(se + o + i * static_cast<uint32_t>(gpr));
                                braw[i] = __ldg(be + o + i * static_cast<uint32_t>(gpr));
                            }
                        }
                        // (k, k + 1) pairs of scales and biases as bf16x2
                        const uint32_t s01 = prmt(sraw[0], sraw[1], 0x5410), s23 = prmt(sraw[2], sraw[3], 0x5410);
                        const uint32_t b01 = prmt(braw[0], braw[1], 0x5410), b23 = prmt(braw[2], braw[3], 0x5410);
                        // Shared address of column (j * PER + f), k-rows 4 kq .. 4 kq + 3: its A-row
                        // ar = a_row(n) has ar & 7 = (f & 7) ^ t and ar >> 3 = r8 + (f >> 3), so
                        // the address is A ^ ((f & 7) * 0x90) + (f >> 3) * 1024 (the XOR only
                        // touches bits 4 - 9, which A holds as (t << 7) | ((q ^ t) << 4)).
                        const int r8 = PER >= 8 ? j * (PER / 8) : j >> 1;
                        const int t = PER >= 8 ? (j & 7) : ((4 * (j & 1)) ^ ((j >> 1) & 7));
                        const int q = kq >> 1;
                        const uint32_t A = wst + static_cast<uint32_t>(r8 * 1024 + (kq & 1) * 8 +
                                                                      ((t << 7) | ((q ^ t) << 4)));
                        auto put = [&](int f, uint32_t v0, uint32_t v1) {
                            const uint32_t a = (A ^ static_cast<uint32_t>((f & 7) * 0x90)) + (f >> 3) * 1024;
                            // no memory clobber: the stage is published by the fence and
                            // arrive below, and no load here reads the A tiles
                            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a), "r"(v0), "r"(v1));
                        };
                        // fast form (every scale of the warp task normal and below 2^-5): a
                        // code field masked in place at bit p of a half is c * 2^(p - 133)
                        // as a bf16, and the fma takes s * 2^(133 - p): the same exact
                        // product s * c, rounded once with the bias.
                        // (magnitudes of the four scales in [2^-126, 2^-5): bf16 patterns
                        // 0x0080 .. 0x3CFF without the sign)
                        const uint32_t mn = vmin_u16x2(s01 & 0x7FFF7FFFu, s23 & 0x7FFF7FFFu);
                        const uint32_t mx = vmax_u16x2(s01 & 0x7FFF7FFFu, s23 & 0x7FFF7FFFu);
                        const bool fast = vmin_u16x2(mn, mn >> 16) >= 0x0080u &&
                                          (vmax_u16x2(mx, mx >> 16) & 0xFFFFu) < 0x3D00u;
                        if (__all_sync(0xffffffffu, fast)) {
                            constexpr int FPB = 8 / BITS;  // fields per byte
                            constexpr uint32_t FM = ((1u << BITS) - 1u) * 0x00010001u;
                            uint32_t m01[FPB], m23[FPB];
#pragma unroll
                            for (int p = 0; p < FPB; ++p) {
                                const uint32_t ex = static_cast<uint32_t>(133 - p * BITS) * 0x00800080u;
                                m01[p] = s01 + ex;
                                m23[p] = s23 + ex;
                            }
#pragma unroll
                            for (int by = 0; by < 4; ++by) {
                                // byte by of k-rows (k, k + 1) into the low bytes of the halves
                                const uint32_t sel = static_cast<uint32_t>(by | ((4 + by) << 8));
                                const uint32_t x01 = prmt(cw[0], cw[1], sel), x23 = prmt(cw[2], cw[3], sel);
#pragma unroll
                                for (int p = 0; p < FPB; ++p)
                                    put(by * FPB + p, bf2_fma(m01[p], x01 & (FM << (p * BITS)), b01),
                                        bf2_fma(m23[p], x23 & (FM << (p * BITS)), b23));
                            }
                        } else {
#pragma unroll
                            for (int f = 0; f < PER; ++f) {
                                uint32_t v[2];
                                if constexpr (BITS == 8) {
                                    // packed fp32: 2^23 + c exactly, minus 2^23, then s c + b
                                    const uint64_t one_m = f2_pack(0x3F800000u, 0x3F800000u);
                                    const uint64_t off = f2_pack(0xCB000000u, 0xCB000000u);
#pragma unroll
                                    for (int pp = 0; pp < 2; ++pp) {
                                        const uint64_t r = f2_pack(prmt(cw[2 * pp], 0x4B000000u, f | 0x7440),
                                                                   prmt(cw[2 * pp + 1], 0x4B000000u, f | 0x7440));
                                        const uint64_t cc = f2_fma(r, one_m, off);
                                        const uint64_t sc = f2_pack(sraw[2 * pp] << 16, sraw[2 * pp + 1] << 16);
                                        const uint64_t bc = f2_pack(braw[2 * pp] << 16, braw[2 * pp + 1] << 16);
                                        v[pp] = f2_to_bf2_packed(f2_fma(sc, cc, bc));
                                    }
                                } else {
                                    // field f of k-rows (k, k + 1) into the two halves: 128 + c
                                    const int byte = (f * BITS) >> 3, sh = (f * BITS) & 7;
                                    const uint32_t sel = static_cast<uint32_t>(byte | ((4 + byte) << 8));
                                    constexpr uint32_t MSK = ((1u << BITS) - 1u) * 0x00010001u;
                                    const uint32_t r0 = codes_to_bf16x2(prmt(cw[0], cw[1], sel) >> sh, MSK);
                                    const uint32_t r1 = codes_to_bf16x2(prmt(cw[2], cw[3], sel) >> sh, MSK);
                                    v[0] = bf2_fma(s01, bf2_sub(r0, 0x43004300u), b01);
                                    v[1] = bf2_fma(s23, bf2_sub(r1, 0x43004300u), b23);
                                }
                                put(f, v[0], v[1]);
                            }
                        }
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) { mbar_arrive(&empty_c[c.s]); mbar_arrive(&full_w[w.s]); }
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

bool tc_gather_t0_supported(int64_t K, int64_t N, int bits, int gs) {
    // code rows of 16-byte multiples (TMA), 64-k steps, 32-bit offsets into
    // one expert's scales
    return K % BK == 0 && K >= BK && N > 0 && (bits == 2 || bits == 4 || bits == 8) &&
           (gs == 32 || gs == 64 || gs == 128) && N % gs == 0 && (N * bits) % 128 == 0 &&
           K * (N / gs) < (int64_t(1) << 32);
}

unsigned int tc_gather_t0_error_take() { return pipeline_error_take(); }

cudaError_t launch_tc_gather_t0(const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs,
                                const uint32_t* perm, const uint32_t* offsets, int64_t E, int64_t N,
                                const uint32_t* codes, const void* scales, const void* biases, int gs,
                                int bits, void* y, cudaStream_t stream, int num_sms) {
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    if (x_rows * K >= (int64_t(1) << 35)) return cudaErrorInvalidValue;  // 32-bit 16-byte offsets
    CUtensorMap map_c;
    const int64_t wpr = N * bits / 32;
    {   // codes [E][K][N * bits / 32]: boxes of 256 columns x 64 k-rows, unswizzled
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(K),
                              static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(wpr) * 4, static_cast<cuuint64_t>(wpr * K) * 4};
        cuuint32_t box[3] = {static_cast<cuuint32_t>(UW * bits / 32), BK, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&map_c, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(codes), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    // scales and biases [E][K][N / gs] as boxes of 8 groups x 64 k-rows, when
    // their rows are whole multiples of 16 bytes
    const int64_t gpr = N / gs;
    const bool staged = gpr % 8 == 0;
    CUtensorMap map_s = map_c, map_b = map_c;
    if (staged) {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(gpr), static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(gpr) * 2, static_cast<cuuint64_t>(gpr * K) * 2};
        cuuint32_t box[3] = {8, BK, 1};
        cuuint32_t es[3] = {1, 1, 1};
        for (int i = 0; i < 2; ++i)
            if (enc(i ? &map_b : &map_s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(i ? biases : scales),
                    dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
    }
    TParams prm{};
    prm.y = static_cast<uint16_t*>(y);
    prm.x = static_cast<const uint16_t*>(x);
    prm.scales = static_cast<const uint16_t*>(scales);
    prm.biases = static_cast<const uint16_t*>(biases);
    prm.gs = gs;
    prm.lg_gs = gs == 32 ? 5 : gs == 64 ? 6 : 7;
    prm.lhs = lhs;
    prm.perm = perm;
    prm.offsets = offsets;
    prm.N = N;
    prm.K = K;
    prm.E = E;
    prm.wunits = static_cast<int>((N + UW - 1) / UW);
    prm.c_stage = static_cast<uint32_t>(BK * UW * bits / 8);
    int dw = 4, dx = 8, dc = 4;
    auto bytes = [&]() {
        return static_cast<size_t>(kXStage) * dx + static_cast<size_t>(kWStage) * dw +
               static_cast<size_t>(prm.c_stage + (staged ? 2048 : 0)) * dc + kMaxPairs * 8 * 4 +
               static_cast<size_t>(2 * (dw + dx + dc) + 4) * 8 + 16;
    };
    const size_t budget = 227 * 1024 - 2048 - 1024;
    while (bytes() > budget && dx > 4) --dx;
    while (bytes() > budget && dc > 3) --dc;
    while (bytes() > budget && dw > 3) --dw;
    if (bytes() > budget) return cudaErrorInvalidConfiguration;
    prm.dw = dw;
    prm.dx = dx;
    prm.dc = dc;
    prm.x_off = 0;
    prm.w_off = kXStage * dx;
    prm.c_off = prm.w_off + kWStage * dw;
    prm.sb_off = prm.c_off + prm.c_stage * dc;
    prm.row_off = prm.sb_off + (staged ? 2048 : 0) * dc;
    prm.bar_off = prm.row_off + kMaxPairs * 8 * 4;
    const size_t smem = bytes() + 1024;
    const int units = static_cast<int>(E) * prm.wunits;
    const int grid = units < num_sms ? units : num_sms;
    void (*k)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const TParams) =
        staged ? (bits == 4 ? tc_gather_t0_kernel<4, true> : bits == 8 ? tc_gather_t0_kernel<8, true>
                                                                      : tc_gather_t0_kernel<2, true>)
               : (bits == 4 ? tc_gather_t0_kernel<4, false> : bits == 8 ? tc_gather_t0_kernel<8, false>
                                                                       : tc_gather_t0_kernel<2, false>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // programmatic dependent launch on the routing kernel (see the kernel)
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
