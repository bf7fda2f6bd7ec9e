// Tensor-core mixture-of-experts product with full-precision (bf16) experts:
// gather_mm, the unquantized companion of gather_qmm ("Docs / Quantization",
// section "Mixture of experts": with rows sorted by expert, a grouped kernel
// reads each expert's weights once; the nuvec crate docs list gather_mm beside
// gather_qmm).
//
// The same transposed form as the quantized grouped kernel: D^T = W_e . X_e^T
// with 256 expert rows (two 128-row tiles) as the MMA's M side and the
// expert's gathered activation rows (<= 64 per pass) as N, so each expert's
// weights cross HBM once for all its rows. With nothing to dequantize, the
// weight tiles go from HBM to shared memory by TMA (128-byte swizzle) and the
// MMA reads both operands from shared memory. Roles, per CTA (persistent):
//   warp 0      one lane streams the weight tiles, 256 rows x 64 k (32 KB)
//               per copy, into a ring released by the MMA.
//   warp 1      TMEM allocation; one thread issues tcgen05.mma (M = 128,
//               N = pairs rounded up to 16, K = 16), two tiles per k-step, into
//               a double-buffered accumulator (64 columns per tile).
//   warps 2-5   epilogue: TMEM lane = weight row, column = pair; each column
//               is stored to its pair's output row.
//   warps 6-9   copy the pairs' activation rows with cp.async into the
//               128-byte-swizzled B layout, fencing each completed stage into
//               the async proxy before arriving on its barrier.
// The kernel is the programmatic dependent of the routing kernel: it sets up
// and prefetches its first weight stages into L2 before waiting for the
// routing tables. Pairs with an out-of-range id get zero rows. Waits are
// bounded by a timer like the other pipelines.
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
constexpr int kThreads = (kXWarp0 * 32) + kXThreads;  // 320
constexpr int kWStage = UW * BK * 2;                  // 32 KB of weights per stage
constexpr int kXStage = kMaxPairs * BK * 2;           // 8 KB of activations per stage
constexpr int kAccCols = kTiles * kMaxPairs;          // 128 columns per accumulator
constexpr uint32_t kTmemCols = 2 * kAccCols;          // double-buffered: 256

struct MParams {
    uint16_t* y;                // [R, N]
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
tc_gather_mm_kernel(const __grid_constant__ CUtensorMap map_w, const MParams prm) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int DW = prm.dw, DX = prm.dx;
    uint8_t* x_ring = smem + prm.x_off;
    uint8_t* w_ring = smem + prm.w_off;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prm.bar_off);
    uint64_t* full_w = bars;
    uint64_t* empty_w = full_w + DW;
    uint64_t* full_x = empty_w + DW;
    uint64_t* empty_x = full_x + DX;
    uint64_t* acc_full = empty_x + DX;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    // [kMaxPairs / (kXThreads / 8)][kXThreads]: x element offsets of each loader thread's rows
    uint32_t* s_xoff = reinterpret_cast<uint32_t*>(smem + prm.row_off);

    if (threadIdx.x == 0) {
        for (int i = 0; i < DW; ++i) { mbar_init(&full_w[i], 1); mbar_init(&empty_w[i], 1); }
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
    // weight stages (the weights do not depend on the routing).
    if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < units) {
        const int e = static_cast<int>(blockIdx.x) / prm.wunits;
        const int row = (static_cast<int>(blockIdx.x) - e * prm.wunits) * UW;
        for (int i = 0; i < DW && i < ksteps; ++i) tma_prefetch_3d(&map_w, i * BK, row, e);
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
        // ------------------------------------------------- producer: weights
        if (lane == 0) {
            RingPos w;
            int issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int e, wt, first, count;
                unit_pairs(u, e, wt, first, count);
                for (int p0 = 0; p0 < count && ok; p0 += kMaxPairs) {
                    for (int ks = 0; ks < ksteps; ++ks) {
                        if (w.use > 0 && !(ok = mbar_wait_backoff(&empty_w[w.s], (w.use - 1) & 1, 41, 512))) break;
                        mbar_expect_tx(&full_w[w.s], kWStage);
                        tma_load_3d(w_ring + w.s * kWStage, &map_w, &full_w[w.s], ks * BK, wt * UW, e);
                        ++issued;
                        w.next(DW);
                    }
                }
            }
            for (int j = 0; j < DW && j < issued; ++j) {  // drain the last copies
                if (--w.s < 0) { w.s = DW - 1; --w.use; }
                mbar_wait(&full_w[w.s], w.use & 1, 49);
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
                    // weight row of the unit = tile * 128 + TMEM lane
                    const int64_t n = static_cast<int64_t>(wt) * UW + tt * WM + q * 32 + lane;
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
    } else {
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

bool tc_gather_mm_supported(int64_t K, int64_t N) { return K % BK == 0 && K >= BK && N > 0; }

unsigned int tc_gather_mm_error_take() { return pipeline_error_take(); }

cudaError_t launch_tc_gather_mm(const void* x, int64_t x_rows, int64_t K, const uint32_t* lhs,
                                const uint32_t* perm, const uint32_t* offsets, int64_t E, int64_t N,
                                const void* w, void* y, cudaStream_t stream, int num_sms) {
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    if (x_rows * K >= (int64_t(1) << 35)) return cudaErrorInvalidValue;  // 32-bit 16-byte offsets
    CUtensorMap map_w;
    {   // experts [E][N][K] bf16: boxes of 64 k (128 bytes) x 256 rows, 128-byte swizzle
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(E)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(N * K) * 2};
        cuuint32_t box[3] = {BK, UW, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    MParams prm{};
    prm.y = static_cast<uint16_t*>(y);
    prm.x = static_cast<const uint16_t*>(x);
    prm.lhs = lhs;
    prm.perm = perm;
    prm.offsets = offsets;
    prm.N = N;
    prm.K = K;
    prm.E = E;
    prm.wunits = static_cast<int>((N + UW - 1) / UW);
    int dw = 4, dx = 8;
    auto bytes = [&]() {
        return static_cast<size_t>(kXStage) * dx + static_cast<size_t>(kWStage) * dw +
               kMaxPairs * 8 * 4 + static_cast<size_t>(2 * (dw + dx) + 4) * 8 + 16;
    };
    const size_t budget = 227 * 1024 - 2048 - 1024;
    while (bytes() > budget && dw > 2) --dw;
    if (bytes() > budget) return cudaErrorInvalidConfiguration;
    prm.dw = dw;
    prm.dx = dx;
    prm.x_off = 0;
    prm.w_off = kXStage * dx;
    prm.row_off = prm.w_off + kWStage * dw;
    prm.bar_off = prm.row_off + kMaxPairs * 8 * 4;
    const size_t smem = bytes() + 1024;
    const int units = static_cast<int>(E) * prm.wunits;
    const int grid = units < num_sms ? units : num_sms;
    cudaError_t e = cudaFuncSetAttribute(tc_gather_mm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
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
    return cudaLaunchKernelEx(&cfg, tc_gather_mm_kernel, map_w, prm);
}

}  // namespace nvq
