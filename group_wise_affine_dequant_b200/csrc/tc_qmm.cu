// Tensor-core quantized GEMM for many rows (the tiled kernel of "Docs /
// Quantization", section "Products on the GPU"): y[M, N] = x[M, K] . w^T, bf16
// activations, weights [N, K] as packed codes + per-group scale and bias.
//
// Blackwell design (sm_100a, one CTA per SM, persistent over 128 x BN tiles):
//   warp 0      TMA producer: the x tile (128 x 64 bf16, 128-byte swizzle) and
//               the packed code tile (BN rows x 64 k) per k-step, into a ring
//               of NS stages, completing on mbarriers.
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (kind::f16,
//               M = 128, N = BN, K = 16) from shared memory into a TMEM fp32
//               accumulator, double-buffered across tiles, and frees ring
//               stages with tcgen05.commit.
//   warps 2-5   epilogue: tcgen05.ld the accumulator (32 lanes each), round to
//               bf16, store y.
//   warps 6-21  dequantize: two threads per weight row of the tile (32 k
//               each); they turn codes into bf16 w = scale * code + bias (one rounding:
//               the code is made exact first, then one bf16 fma) and writes the
//               row into the B tile in the canonical K-major 128-byte-swizzled
//               layout the MMA reads. Codes arrive swizzled (32/64-byte TMA
//               swizzle) so the row reads hit distinct banks; scales and biases
//               arrive by TMA in blocks of 8 groups x BN rows through a 2-slot
//               ring that the dequant warps release.
// Split-K (the split-K kernel of "Docs / Quantization", section "Products on
// the GPU", for outputs too small to fill the GPU with tiles while K is long):
// the S CTAs of a thread-block cluster share one output tile, CTA r running
// the same pipeline over k-steps [r * ks / S, (r + 1) * ks / S). Each writes its
// fp32 partial tile from TMEM into its own shared memory; after a cluster
// barrier, CTA r sums rows [r * 128 / S, (r + 1) * 128 / S) of the S partials
// through distributed shared memory in rank order 0, 1, ..., S - 1 and stores
// bf16 y. The order is fixed, so results are deterministic; no global scratch
// is needed.
// The contraction runs on the tensor cores in bf16 with fp32 accumulation; the
// dequantized weight is rounded once to bf16 (relative error <= 2^-9), and the
// result once to bf16 on output: together within the product tolerance.
// Every wait on an mbarrier is bounded by a timer; on expiry the kernel records
// an error code, stops issuing work and exits after draining its copies.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tma.cuh"

namespace nvq {
namespace {

using namespace tc;

constexpr int BM = 128;          // rows of x per tile (TMEM lanes)
constexpr int BK = 64;           // k per stage: one 128-byte swizzle atom of bf16
constexpr int UMMA_K = 16;
constexpr int kDequantWarp0 = 6;
constexpr int kDequantThreads = 512;  // two threads per weight row (32 k each)
constexpr int kThreads = kDequantWarp0 * 32 + kDequantThreads;

struct TcParams {
    uint16_t* y;
    const uint16_t* scales;
    const uint16_t* biases;
    int64_t M, N, K;
    int gs;
    int bn;            // tile columns (weight rows), multiple of 32, <= 256
    int m_tiles, n_tiles;
    int stages;
    uint32_t a_off, b_off, c_off, bar_off;  // shared-memory layout (bytes)
    uint32_t b_stage_bytes, c_stage_bytes;
    uint32_t tmem_cols;
    uint32_t sb_off;          // scale/bias ring: 2 slots x (scales, biases) x bn x 16 bytes
    int sb_tma;               // scales/biases by TMA (rows of 16-byte multiples)
    uint32_t m2, m4, m6;      // shift counts 2, 4, 6
    int lg_gs;                // log2(group size)
    int splits;               // split-K: CTAs per cluster (1 = no split)
};

// Cluster helpers (split-K): this CTA's rank, the shared::cluster address of
// a local shared-memory location in CTA `rank`, a load from it, and a barrier
// of every thread of the cluster (release / acquire: shared-memory writes
// before it are visible to the other CTAs' reads after it).
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_map(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
// Byte offset of columns [4 c, 4 c + 4) of row r in a [128][bn] fp32 partial
// tile whose 16-byte chunks are XOR-swizzled by (row mod 8): the epilogue's
// stores (one row per lane) and the reduction's loads hit distinct banks.
__device__ __forceinline__ uint32_t part_off(int r, int c, int bn) {
    return static_cast<uint32_t>(r * bn * 4 + ((c ^ (r & 7)) << 4));
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Floating-point modes (FMT 1 = MXFP4, 2 = MXFP8, 3 = NVFP4): codes decode
// exactly to f16 pairs by the hardware conversion, widen to fp32, take the
// group's scale (E8M0 or E4M3 code, one uint8 per group) and round once to
// bf16 pairs: the products of small floats and their scales are bf16 numbers,
// so the B tile holds the exact dequantized weights.
__device__ __forceinline__ float fp_scale(int fmt, uint32_t code) {
    if (fmt == 3) {
        uint32_t h;
        asm("{\n\t.reg .b16 s;\n\tcvt.u16.u32 s, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, s;\n\t}" : "=r"(h) : "r"(code & 255u));
        return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
    }
    return code == 0 ? __uint_as_float(0x00400000u) : code == 255 ? __uint_as_float(0x7FC00000u)
                                                                  : __uint_as_float(code << 23);
}
template <int FMT>
__device__ __forceinline__ void fp_dequant_word(uint32_t w, float S, uint32_t* out) {
    constexpr int PAIRS = FMT == 2 ? 2 : 4;
#pragma unroll
    for (int i = 0; i < PAIRS; ++i) {
        uint32_t h;
        if constexpr (FMT == 2)
            asm("{\n\t.reg .b16 s;\n\tcvt.u16.u32 s, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, s;\n\t}" : "=r"(h) : "r"((w >> (16 * i)) & 0xFFFFu));
        else
            asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h) : "r"((w >> (8 * i)) & 255u));
        float lo, hi;
        asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
            : "=f"(lo), "=f"(hi) : "r"(h));
        out[i] = f2_to_bf2(lo * S, hi * S);
    }
}

template <int BITS, bool SPLIT, bool TR0, int MS = 1, int FMT = 0>
__global__ void __launch_bounds__(kThreads, 1)
tc_qmm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_c,
              const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_b,
              const TcParams prm) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base: the 128-byte swizzle pattern repeats every 8 rows
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = prm.stages;
    const int BN = prm.bn;
    uint8_t* a_ring = smem + prm.a_off;
    uint8_t* b_ring = smem + prm.b_off;
    uint8_t* c_ring = smem + prm.c_off;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prm.bar_off);
    uint64_t* full_a = bars;
    uint64_t* full_c = bars + NS;
    uint64_t* full_b = bars + 2 * NS;
    uint64_t* empty = bars + 3 * NS;
    uint64_t* acc_full = bars + 4 * NS;
    uint64_t* acc_empty = bars + 4 * NS + 2;
    uint64_t* sb_full = bars + 4 * NS + 4;
    uint64_t* sb_empty = bars + 4 * NS + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * NS + 8);
    uint8_t* sb_ring = smem + prm.sb_off;
    const uint32_t sb_slot_bytes = 2u * BN * 16u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&full_c[s], 1);
            mbar_init(&full_b[s], kDequantThreads / 32);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
            mbar_init(&sb_full[a], 1);
            mbar_init(&sb_empty[a], kDequantThreads / 32);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(prm.tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // launched as the programmatic dependent of the previous kernel: set up
    // above, then let the next product launch and wait for the previous grid
    // (x, the weights or y may be its) before the first global access
    pdl_launch_dependents();
    pdl_wait();

    const int ksteps = static_cast<int>(prm.K / BK);
    const int sgk = 8 * prm.gs / BK;  // k-steps per block of 8 groups
    const int tiles = prm.m_tiles * prm.n_tiles;
    // Tiles of this CTA: persistent over tiles, or (split-K) the one tile of
    // its cluster, k-steps [k0, k1) of it.
    const int S = SPLIT ? prm.splits : 1;
    const int rank = SPLIT ? static_cast<int>(cluster_rank()) : 0;
    const int tile0 = SPLIT ? static_cast<int>(blockIdx.x) / S : static_cast<int>(blockIdx.x);
    const int tstep = SPLIT ? tiles : static_cast<int>(gridDim.x);
    const int k0 = SPLIT ? rank * ksteps / S : 0;
    const int k1 = SPLIT ? (rank + 1) * ksteps / S : ksteps;
    const uint32_t a_bytes = MS * BM * BK * 2;  // MS row subtiles of 128 x 64
    const uint32_t c_bytes = static_cast<uint32_t>(BN) * BK * BITS / 8;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int s = 0;            // ring stage and its use count (no divisions in the loop)
            uint32_t use = 0;
            uint32_t blk = 0;     // scale/bias blocks issued
            int issued = 0;       // loads issued (bounded by the drain below)
            bool ok = true;
            for (int tile = tile0; tile < tiles && ok; tile += tstep) {
                const int mt = tile % prm.m_tiles, nt = tile / prm.m_tiles;
                int kb = k0 % sgk;  // k-step within the current scale block
                for (int ks = k0; ks < k1 && ok; ++ks) {
                    if (prm.sb_tma && (kb == 0 || ks == k0)) {
                        const int slot = blk & 1;
                        const uint32_t u = blk >> 1;
                        if (u > 0 && !(ok = mbar_wait(&sb_empty[slot], (u - 1) & 1, 7))) break;
                        mbar_expect_tx(&sb_full[slot], sb_slot_bytes);
                        uint8_t* dst = sb_ring + slot * sb_slot_bytes;
                        const int gcol = static_cast<int>((blk_in_tile(ks, sgk)) * 8);
                        tma_load_2d(dst, &map_s, &sb_full[slot], gcol, nt * BN);
                        tma_load_2d(dst + BN * 16, &map_b, &sb_full[slot], gcol, nt * BN);
                        ++blk;
                    }
                    if (++kb == sgk) kb = 0;
                    if (use > 0 && !(ok = mbar_wait(&empty[s], (use - 1) & 1, 1))) break;
                    mbar_expect_tx(&full_a[s], a_bytes);
                    tma_load_2d(a_ring + s * a_bytes, &map_x, &full_a[s], ks * BK, mt * BM * MS);
                    mbar_expect_tx(&full_c[s], c_bytes);
                    if constexpr (TR0)  // weights [K, N]: 64 k-rows x BN columns
                        tma_load_2d(c_ring + s * prm.c_stage_bytes, &map_c, &full_c[s],
                                    nt * BN * BITS / 32, ks * BK);
                    else
                        tma_load_2d(c_ring + s * prm.c_stage_bytes, &map_c, &full_c[s],
                                    ks * BK * BITS / 32, nt * BN);
                    ++issued;
                    if (++s == NS) { s = 0; ++use; }
                }
            }
            // drain: the last loads in flight land before the CTA may exit
            for (int j = 0; j < NS && j < issued; ++j) {
                if (--s < 0) { s = NS - 1; --use; }
                mbar_wait(&full_a[s], use & 1, 9);
                mbar_wait(&full_c[s], use & 1, 9);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, BN);
            int s = 0;
            uint32_t use = 0;
            int local = 0;
            bool ok = true;
            for (int tile = tile0; tile < tiles && ok; tile += tstep, ++local) {
                const int a = local & 1;
                const uint32_t ause = static_cast<uint32_t>(local >> 1);
                if (ause > 0 && !(ok = mbar_wait(&acc_empty[a], (ause - 1) & 1, 2))) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * MS * BN);
                for (int ks = k0; ks < k1; ++ks) {
                    if (!(ok = mbar_wait(&full_a[s], use & 1, 3))) break;
                    if (!(ok = mbar_wait(&full_b[s], use & 1, 4))) break;
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(a_ring + s * a_bytes);
                    const uint64_t bd = sw128_desc(b_ring + s * prm.b_stage_bytes);
#pragma unroll
                    for (int m = 0; m < MS; ++m)  // every row subtile against the same weights
#pragma unroll
                        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                            // advance 16 bf16 (32 bytes) along K inside the swizzle atom
                            tc_mma(d_tmem + m * BN, ad + (m * (BM * BK * 2) >> 4) + (kk * UMMA_K * 2 >> 4),
                                   bd + (kk * UMMA_K * 2 >> 4), idesc, (ks > k0 || kk > 0) ? 1u : 0u);
                        }
                    tc_commit(&empty[s]);
                    if (++s == NS) { s = 0; ++use; }
                }
                if (ok) tc_commit(&acc_full[a]);
            }
        }
    } else if (warp < kDequantWarp0) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int row_in_tile = q * 32 + lane;
        int local = 0;
        for (int tile = tile0; tile < tiles; tile += tstep, ++local) {
            const int a = local & 1;
            const uint32_t ause = static_cast<uint32_t>(local >> 1);
            if (!mbar_wait_backoff(&acc_full[a], ause & 1, 5, 2048)) break;
            tc_fence_after();
            if constexpr (SPLIT) {
                // the partial tile into this CTA's shared memory, [row][BN] fp32
                // with swizzled 16-byte chunks (the pipeline's stages are all
                // consumed by now)
                for (int j = 0; j < BN / 32; ++j) {
                    uint32_t v[32];
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                           static_cast<uint32_t>(a * BN + j * 32);
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                          "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                          "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
                          "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                          "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]),
                          "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                        : "r"(taddr));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4*>(smem + part_off(row_in_tile, j * 8 + c, BN)) =
                            make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                }
                tc_fence_before();
                continue;
            }
            const int mt = tile % prm.m_tiles, nt = tile / prm.m_tiles;
            const int64_t col0 = static_cast<int64_t>(nt) * BN;
            for (int m = 0; m < MS; ++m)
            for (int j = 0; j < BN / 32; ++j) {
                const int64_t row = (static_cast<int64_t>(mt) * MS + m) * BM + row_in_tile;
                uint32_t v[32];
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                       static_cast<uint32_t>((a * MS + m) * BN + j * 32);
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                    "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                    "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                      "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                      "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
                      "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                      "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]),
                      "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                const int64_t c = col0 + j * 32;
                if (row < prm.M) {
                    uint16_t* yp = prm.y + row * prm.N + c;
                    if (c + 32 <= prm.N && (prm.N % 8) == 0) {
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            uint4 o;
                            o.x = f2_to_bf2(__uint_as_float(v[8 * h + 0]), __uint_as_float(v[8 * h + 1]));
                            o.y = f2_to_bf2(__uint_as_float(v[8 * h + 2]), __uint_as_float(v[8 * h + 3]));
                            o.z = f2_to_bf2(__uint_as_float(v[8 * h + 4]), __uint_as_float(v[8 * h + 5]));
                            o.w = f2_to_bf2(__uint_as_float(v[8 * h + 6]), __uint_as_float(v[8 * h + 7]));
                            *reinterpret_cast<uint4*>(yp + 8 * h) = o;
                        }
                    } else {
                        for (int e = 0; e < 32; ++e)
                            if (c + e < prm.N) yp[e] = f32_to_bf16_bits(__uint_as_float(v[e]));
                    }
                }
            }
            if (BN & 16) {  // tiles 16 columns past a multiple of 32
                for (int m = 0; m < MS; ++m) {
                    const int64_t row = (static_cast<int64_t>(mt) * MS + m) * BM + row_in_tile;
                    uint32_t v[16];
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                           static_cast<uint32_t>((a * MS + m) * BN + (BN & ~31));
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                          "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                          "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                        : "r"(taddr));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    const int64_t c = col0 + (BN & ~31);
                    if (row < prm.M) {
                        uint16_t* yp = prm.y + row * prm.N + c;
                        if (c + 16 <= prm.N && (prm.N % 8) == 0) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                uint4 o;
                                o.x = f2_to_bf2(__uint_as_float(v[8 * h + 0]), __uint_as_float(v[8 * h + 1]));
                                o.y = f2_to_bf2(__uint_as_float(v[8 * h + 2]), __uint_as_float(v[8 * h + 3]));
                                o.z = f2_to_bf2(__uint_as_float(v[8 * h + 4]), __uint_as_float(v[8 * h + 5]));
                                o.w = f2_to_bf2(__uint_as_float(v[8 * h + 6]), __uint_as_float(v[8 * h + 7]));
                                *reinterpret_cast<uint4*>(yp + 8 * h) = o;
                            }
                        } else {
                            for (int e = 0; e < 16; ++e)
                                if (c + e < prm.N) yp[e] = f32_to_bf16_bits(__uint_as_float(v[e]));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
    } else {
        // ------------------------------------------------------------ dequantize
        if constexpr (TR0) {
            // Weights stored [K, N], grouped along N: the stage holds 64 k-rows of
            // BN * BITS / 32 code words. A task is (4 consecutive k-rows, one code
            // word): PER columns x 4 k, dequantized into (k, k + 1) pairs and
            // written transposed into the K-major B tile (row = column n).
            constexpr int PER = 32 / BITS;
            const int wpr = BN * BITS / 32;
            const int tasks = (BK / 4) * wpr;
            const int dt = threadIdx.x - kDequantWarp0 * 32;
            const int64_t gpr = prm.N / prm.gs;  // groups per k-row of W
            int s = 0;
            uint32_t use = 0;
            bool ok = true;
            for (int tile = tile0; tile < tiles && ok; tile += tstep) {
                const int nt = tile / prm.m_tiles;
                for (int ks = k0; ks < k1; ++ks) {
                    if (!(ok = mbar_wait(&full_c[s], use & 1, 6))) break;
                    const uint8_t* cst = c_ring + s * prm.c_stage_bytes;
                    uint8_t* bst = b_ring + s * prm.b_stage_bytes;
                    for (int task = dt; task < tasks; task += kDequantThreads) {
                        const int kq = task % (BK / 4), j = task / (BK / 4);
                        const int nl = j * PER;                                  // first column in the tile
                        const int64_t ng = static_cast<int64_t>(nt) * BN + nl;   // and in W
                        const int64_t kg = static_cast<int64_t>(ks) * BK + 4 * kq;
                        uint32_t w[4], sraw[4], braw[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            w[i] = *reinterpret_cast<const uint32_t*>(cst + (4 * kq + i) * (wpr * 4) + 4 * j);
                            const int64_t gi = (kg + i) * gpr + (ng < prm.N ? ng / prm.gs : 0);
                            sraw[i] = ng < prm.N ? __ldg(prm.scales + gi) : 0u;
                            braw[i] = ng < prm.N ? __ldg(prm.biases + gi) : 0u;
                        }
                        // (k, k + 1) pairs of scales and biases as bf16x2
                        const uint32_t s01 = sraw[0] | (sraw[1] << 16), s23 = sraw[2] | (sraw[3] << 16);
                        const uint32_t b01 = braw[0] | (braw[1] << 16), b23 = braw[2] | (braw[3] << 16);
#pragma unroll
                        for (int f = 0; f < PER; ++f) {
                            uint32_t v[2];
                            if constexpr (BITS == 8) {
                                // packed fp32: 2^23 + c exactly, minus 2^23, then s c + b
                                const uint64_t one_m = f2_pack(0x3F800000u, 0x3F800000u);
                                const uint64_t off = f2_pack(0xCB000000u, 0xCB000000u);
#pragma unroll
                                for (int p = 0; p < 2; ++p) {
                                    const uint64_t r = f2_pack(prmt(w[2 * p], 0x4B000000u, f | 0x7440),
                                                               prmt(w[2 * p + 1], 0x4B000000u, f | 0x7440));
                                    const uint64_t c = f2_fma(r, one_m, off);
                                    const uint64_t sc = f2_pack(sraw[2 * p] << 16, sraw[2 * p + 1] << 16);
                                    const uint64_t bc = f2_pack(braw[2 * p] << 16, braw[2 * p + 1] << 16);
                                    v[p] = f2_to_bf2_packed(f2_fma(sc, c, bc));
                                }
                            } else {
                                // field f of k-rows (k, k + 1) into the two halves: 128 + c
                                const int byte = (f * BITS) >> 3, sh = (f * BITS) & 7;
                                const uint32_t sel = static_cast<uint32_t>(byte | ((4 + byte) << 8));
                                constexpr uint32_t MSK = ((1u << BITS) - 1u) * 0x00010001u;
                                const uint32_t r0 = codes_to_bf16x2(prmt(w[0], w[1], sel) >> sh, MSK);
                                const uint32_t r1 = codes_to_bf16x2(prmt(w[2], w[3], sel) >> sh, MSK);
                                v[0] = bf2_fma(s01, bf2_sub(r0, 0x43004300u), b01);
                                v[1] = bf2_fma(s23, bf2_sub(r1, 0x43004300u), b23);
                            }
                            // row n = nl + f of the B tile: k-chunk kq / 2 (8 k), half (kq & 1)
                            const int n = nl + f;
                            *reinterpret_cast<uint2*>(bst + (n >> 3) * 1024 + (n & 7) * 128 +
                                                      ((((kq >> 1) ^ (n & 7))) << 4) + (kq & 1) * 8) =
                                make_uint2(v[0], v[1]);
                        }
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_b[s]);
                    if (++s == NS) { s = 0; ++use; }
                }
            }
        } else {
        const int dt = threadIdx.x - kDequantWarp0 * 32;  // 0 .. 511
        // tiles of up to 128 columns: four threads per weight row (16 k each);
        // wider tiles: two (32 k each)
        const bool quad = BN <= 128;
        const int r = quad ? dt >> 2 : dt >> 1;           // weight row within the tile
        const int h = quad ? dt & 3 : dt & 1;             // k part of the k-step
        const int kpart = quad ? 16 : 32;                 // k per thread and step
        const bool has_row = r < BN;
        const int64_t gpr = prm.K / prm.gs;
        using DQ = Dequant<BITS>;
        int s = 0;
        uint32_t use = 0;
        uint32_t blk = 0;
        bool ok = true;
        for (int tile = tile0; tile < tiles && ok; tile += tstep) {
            const int nt = tile / prm.m_tiles;
            int kb = k0 % sgk;
            const int64_t n = static_cast<int64_t>(nt) * BN + r;
            const bool live = has_row && n < prm.N;
            const uint16_t* srow = prm.scales + (live ? n : 0) * gpr;
            const uint16_t* brow = prm.biases + (live ? n : 0) * gpr;
            for (int ks = k0; ks < k1; ++ks) {
                // a thread's k part lies in one group (groups are 32-k aligned multiples of 32)
                const int g = ((ks * BK + kpart * h) >> prm.lg_gs);
                float sc = 0.f, bc = 0.f;
                const int slot = blk & 1;
                if (prm.sb_tma) {
                    if ((kb == 0 || ks == k0) && !(ok = mbar_wait(&sb_full[slot], (blk >> 1) & 1, 8))) break;
                    if (has_row) {
                        const uint16_t* ss = reinterpret_cast<const uint16_t*>(sb_ring + slot * sb_slot_bytes);
                        const int gi = g & 7;
                        sc = bf16_bits_to_f32(ss[r * 8 + gi]);
                        bc = bf16_bits_to_f32(ss[BN * 8 + r * 8 + gi]);
                    }
                } else if (live) {
                    if constexpr (FMT != 0) {  // uint8 scale codes; NVFP4: a second group for k 16..31
                        const uint8_t* s8 = reinterpret_cast<const uint8_t*>(prm.scales) + n * gpr;
                        sc = fp_scale(FMT, __ldg(s8 + g));
                        bc = (FMT == 3 && kpart == 32) ? fp_scale(FMT, __ldg(s8 + g + 1)) : sc;
                    } else {
                        sc = bf16_bits_to_f32(__ldg(srow + g));
                        bc = bf16_bits_to_f32(__ldg(brow + g));
                    }
                }
                if (!(ok = mbar_wait(&full_c[s], use & 1, 6))) break;
                // one dequantizer for the warp's step: the fast form when every
                // live row's group allows it (same results either way)
                const bool fast = __all_sync(__activemask(),
                                             !live || dq_fast_ok((__float_as_uint(sc) >> 16) * 0x00010001u));
                if (has_row && !quad) {
                    const uint8_t* cst = c_ring + s * prm.c_stage_bytes;
                    constexpr int NW = BITS;  // code words per 32 k
                    uint32_t w[NW];
                    if constexpr (BITS == 4) {
                        const uint4 v4 = *reinterpret_cast<const uint4*>(cst + r * 32 + ((h ^ ((r >> 2) & 1)) << 4));
                        w[0] = v4.x; w[1] = v4.y; w[2] = v4.z; w[3] = v4.w;
                    } else if constexpr (BITS == 8) {
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int j = 2 * h + jj;
                            const uint4 v4 = *reinterpret_cast<const uint4*>(cst + r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
                            w[4 * jj] = v4.x; w[4 * jj + 1] = v4.y; w[4 * jj + 2] = v4.z; w[4 * jj + 3] = v4.w;
                        }
                    } else {
                        const uint2 v2 = *reinterpret_cast<const uint2*>(cst + r * 16 + h * 8);
                        w[0] = v2.x; w[1] = v2.y;
                    }
                    uint8_t* brow_s = b_ring + s * prm.b_stage_bytes + (r >> 3) * 1024 + (r & 7) * 128;
                    const uint32_t s2 = (__float_as_uint(sc) >> 16) * 0x00010001u;
                    const uint32_t b2 = (__float_as_uint(bc) >> 16) * 0x00010001u;
                    uint32_t out[16];
                    if constexpr (FMT != 0) {
#pragma unroll
                        for (int i = 0; i < NW; ++i)  // NVFP4: words 2, 3 hold k 16..31 (second group)
                            fp_dequant_word<FMT>(w[i], (FMT == 3 && i >= 2) ? bc : sc, out + i * DQ::PAIRS);
                    } else if (fast) {
#pragma unroll
                        for (int i = 0; i < NW; ++i) DQ::run_fast(w[i], s2, b2, out + i * DQ::PAIRS);
                    } else {
#pragma unroll
                        for (int i = 0; i < NW; ++i)
                            DQ::run(w[i], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6, out + i * DQ::PAIRS);
                    }
                    // chunks 4 h .. 4 h + 3 (8 k each) of the row, under the 128-byte swizzle
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint4 o;
                        o.x = out[4 * c]; o.y = out[4 * c + 1]; o.z = out[4 * c + 2]; o.w = out[4 * c + 3];
                        *reinterpret_cast<uint4*>(brow_s + (((4 * h + c) ^ (r & 7)) << 4)) = o;
                    }
                    fence_proxy_async();
                } else if (has_row) {
                    // 16 k of the row: k 16 h .. 16 h + 15 of the k-step
                    const uint8_t* cst = c_ring + s * prm.c_stage_bytes;
                    constexpr int NW = BITS / 2;  // code words per 16 k
                    uint32_t w[NW];
                    if constexpr (BITS == 4) {  // 32-byte rows, 32-byte swizzle: 8 bytes
                        const uint2 v2 = *reinterpret_cast<const uint2*>(
                            cst + r * 32 + (((h >> 1) ^ ((r >> 2) & 1)) << 4) + (h & 1) * 8);
                        w[0] = v2.x; w[1] = v2.y;
                    } else if constexpr (BITS == 8) {  // 64-byte rows, 64-byte swizzle: 16 bytes
                        const uint4 v4 = *reinterpret_cast<const uint4*>(cst + r * 64 + ((h ^ ((r >> 1) & 3)) << 4));
                        w[0] = v4.x; w[1] = v4.y; w[2] = v4.z; w[3] = v4.w;
                    } else {  // 16-byte rows, unswizzled: one word
                        w[0] = *reinterpret_cast<const uint32_t*>(cst + r * 16 + h * 4);
                    }
                    uint8_t* brow_s = b_ring + s * prm.b_stage_bytes + (r >> 3) * 1024 + (r & 7) * 128;
                    const uint32_t s2 = (__float_as_uint(sc) >> 16) * 0x00010001u;
                    const uint32_t b2 = (__float_as_uint(bc) >> 16) * 0x00010001u;
                    uint32_t out[8];
                    if constexpr (FMT != 0) {
#pragma unroll
                        for (int i = 0; i < NW; ++i) fp_dequant_word<FMT>(w[i], sc, out + i * DQ::PAIRS);
                    } else if (fast) {
#pragma unroll
                        for (int i = 0; i < NW; ++i) DQ::run_fast(w[i], s2, b2, out + i * DQ::PAIRS);
                    } else {
#pragma unroll
                        for (int i = 0; i < NW; ++i)
                            DQ::run(w[i], s2, b2, sc, bc, prm.m2, prm.m4, prm.m6, out + i * DQ::PAIRS);
                    }
                    // chunks 2 h, 2 h + 1 (8 k each) of the row, under the 128-byte swizzle
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint4 o;
                        o.x = out[4 * c]; o.y = out[4 * c + 1]; o.z = out[4 * c + 2]; o.w = out[4 * c + 3];
                        *reinterpret_cast<uint4*>(brow_s + (((2 * h + c) ^ (r & 7)) << 4)) = o;
                    }
                    fence_proxy_async();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_b[s]);
                if (prm.sb_tma && (kb == sgk - 1 || ks == k1 - 1)) {
                    if (lane == 0) mbar_arrive(&sb_empty[slot]);  // this warp is done with the block
                    ++blk;
                }
                if (++kb == sgk) kb = 0;
                if (++s == NS) { s = 0; ++use; }
            }
        }
        }  // TR0
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (SPLIT) {
        // Sum the cluster's S partial tiles in rank order: CTA `rank` owns rows
        // [rank * 128 / S, (rank + 1) * 128 / S); a thread takes 4 columns of a
        // row, loads them from all S partials (16-byte loads, all in flight)
        // and adds them in order 0, 1, ..., S - 1.
        cluster_sync();
        const int mt = tile0 % prm.m_tiles, nt = tile0 / prm.m_tiles;
        const int r_lo = rank * BM / S, r_hi = (rank + 1) * BM / S;
        const uint32_t part0 = smem_u32(smem);
        const int chunks = BN / 4;
        for (int i = threadIdx.x; i < (r_hi - r_lo) * chunks; i += kThreads) {
            const int r = r_lo + i / chunks, c = i % chunks;
            const int64_t row = static_cast<int64_t>(mt) * BM + r;
            if (row >= prm.M) continue;
            const uint32_t off = part0 + part_off(r, c, BN);
            float4 v[8];
#pragma unroll
            for (int src = 0; src < 8; ++src)
                if (src < S) v[src] = ld_cluster_f32x4(cluster_map(off, src));
            float4 acc = v[0];
#pragma unroll
            for (int src = 1; src < 8; ++src)
                if (src < S) { acc.x += v[src].x; acc.y += v[src].y; acc.z += v[src].z; acc.w += v[src].w; }
            const int64_t col = static_cast<int64_t>(nt) * BN + 4 * c;
            uint16_t* yp = prm.y + row * prm.N + col;
            const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
            if (col + 4 <= prm.N && (prm.N % 4) == 0) {
                *reinterpret_cast<uint2*>(yp) = make_uint2(f2_to_bf2(a4[0], a4[1]), f2_to_bf2(a4[2], a4[3]));
            } else {
                for (int e = 0; e < 4; ++e)
                    if (col + e < prm.N) yp[e] = f32_to_bf16_bits(a4[e]);
            }
        }
        cluster_sync();  // no CTA leaves while the others still read its partial
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(prm.tmem_cols));
    }
}

// ---------------------------------------------------------------- host side
// Tile width of least padded work over whole waves, for tiles of bm rows and
// bn in [bn_lo, bn_hi] (steps of `step`).
int pick_bn(int64_t M, int64_t N, int num_sms, int step = 32, int bm = BM, int bn_hi = 256,
            int bn_lo = 128) {
    const int64_t mt = (M + bm - 1) / bm;
    int best = bn_hi;
    double best_eff = -1.0;
    for (int bn = bn_hi; bn >= bn_lo; bn -= step) {
        const int64_t tiles = mt * ((N + bn - 1) / bn);
        const int64_t waves = (tiles + num_sms - 1) / num_sms;
        // useful work over the work of the waves, counting padded rows and columns
        const double eff = static_cast<double>(M * N) /
                           (static_cast<double>(waves * num_sms) * bm * bn);
        if (eff > best_eff + 1e-9) { best_eff = eff; best = bn; }
    }
    return best;
}

// Split-K plan for an item of m_rows rows: when the unsplit tiles would fill
// less than half of the SMs and K holds at least 8 k-steps, split K over a
// cluster of S <= 8 CTAs (at least 4 k-steps each) and pick the tile width
// that keeps the most SMs busy with the least column padding. A pure function
// of (rows, N, K, SM count).
struct TcPlan {
    int bn, splits;
    int ms = 1;  // 128-row subtiles per tile: 2 pairs every dequantized weight tile with 256 rows
};

// Clusters of `size` CTAs (one CTA per SM) that the device runs at once: a
// property of the device's GPC layout (e.g. 74, 33 and 15 clusters of 2, 4
// and 8 on a 148-SM B200), queried once per device and size.
int max_clusters(int size) {
    static int cache[64][4] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    const int slot = size == 2 ? 0 : size == 4 ? 1 : size == 8 ? 2 : 3;
    if (cache[dev][slot] > 0) return cache[dev][slot];
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(size), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 160 * 1024;  // > half an SM: one CTA per SM, as every plan here
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(size);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void (*k)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
              const TcParams) = tc_qmm_kernel<4, true, false>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(cfg.dynamicSmemBytes)) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(k), &cfg) != cudaSuccess ||
        n <= 0) {
        cudaGetLastError();  // clear a failed query; assume one cluster per 8 SMs
        n = 148 / (size * 2);
    }
    cache[dev][slot] = n;
    return n;
}

// The tiling and split-K plan for an item of m_rows rows: with the unsplit
// tiles filling at least half the SMs (or fewer than 8 k-steps), no split;
// otherwise the (tile width bn, cluster size S in {2, 4, 8}) of least
// estimated time, counting waves of co-resident clusters, k-steps per CTA and
// a per-step time that grows with bn (measured on B200: about 0.5 us per
// 64-k step at bn 64, 0.8 at bn 256, plus about 8 us of fixed cost per CTA).
// A pure function of (rows, N, K) and the device.
double tc_cost(int64_t waves, int64_t steps, int bn) {
    return static_cast<double>(waves) * (static_cast<double>(steps) * (0.45 + 0.0013 * bn) + 8.0);
}

TcPlan plan_tc(int64_t m_rows, int64_t N, int64_t K, int num_sms, int step = 32, int step2 = 16) {
    const int bn0 = pick_bn(m_rows, N, num_sms, step);
    const int64_t mt = (m_rows + BM - 1) / BM;
    const int64_t ks = K / BK;
    const int64_t tiles0 = mt * ((N + bn0 - 1) / bn0);
    if (2 * tiles0 > num_sms || ks < 8) {
        // Enough tiles without a split. From 256 rows on, tiles of 256 rows x
        // bn <= 128 columns (four accumulators fill TMEM's 512 columns) use
        // every dequantized weight tile for twice the rows; widths step by 16.
        if (m_rows >= 2 * BM) {
            const int bn2 = pick_bn(m_rows, N, num_sms, step2, 2 * BM, 128, 64);
            const int64_t tiles2 = ((m_rows + 2 * BM - 1) / (2 * BM)) * ((N + bn2 - 1) / bn2);
            if (2 * tiles2 > num_sms) return {bn2, 1, 2};
        }
        return {bn0, 1};
    }
    TcPlan best{bn0, 1};
    double best_cost = tc_cost((tiles0 + num_sms - 1) / num_sms, ks, bn0);
    for (int sp = 2; sp <= 8; sp *= 2) {
        if (ks / sp < 4) break;
        const int64_t mc = max_clusters(sp);
        for (int bn = step < 64 ? 64 : step; bn <= 256; bn += step) {
            const int64_t tiles = mt * ((N + bn - 1) / bn);
            const double cost = tc_cost((tiles + mc - 1) / mc, (ks + sp - 1) / sp, bn);
            if (cost < best_cost - 1e-9) { best_cost = cost; best = {bn, sp}; }
        }
    }
    return best;
}

}  // namespace

unsigned int tc_error_take() { return pipeline_error_take(); }

// Tile widths the transposed layout can take: the code rows of a tile
// (bn * bits / 8 bytes) must be 16-byte multiples for its TMA box. bn_step:
// 128-row tiles (multiples of 32 for the split-K partial tiles); bn_step2:
// 256-row tiles (multiples of 16, the MMA's N granularity).
static int bn_step(int bits, int transpose) { return (!transpose && bits == 2) ? 64 : 32; }
static int bn_step2(int bits, int transpose) {
    return transpose ? 16 : bits == 2 ? 64 : bits == 4 ? 32 : 16;
}

int tc_splits(int64_t m_rows, int64_t K, int64_t N, int num_sms, int bits, int transpose) {
    return plan_tc(m_rows, N, K, num_sms, bn_step(bits, transpose), bn_step2(bits, transpose)).splits;
}

bool tc_supported_t0(int64_t M, int64_t K, int64_t N, int bits, int gs) {
    // weights [K, N] grouped along N: rows of codes are 16-byte multiples
    return tc_supported(M, K, N, bits, gs) && (N * bits / 8) % 16 == 0 && N % gs == 0;
}

bool tc_supported(int64_t M, int64_t K, int64_t N, int bits, int gs) {
    return M > 0 && N > 0 && K % BK == 0 && K >= BK && (bits == 2 || bits == 4 || bits == 8) &&
           (gs == 32 || gs == 64 || gs == 128) && M < (int64_t(1) << 31) && N < (int64_t(1) << 31);
}

cudaError_t launch_tc_qmm(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                          const void* scales, const void* biases, int gs, int bits, void* y,
                          cudaStream_t stream, int num_sms, int64_t item_rows, int transpose, int fmt) {
    if (fmt != 0) {  // floating-point modes: weights [N, K], uint8 scale codes, no biases
        transpose = 1;
        biases = scales;
    }
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    // the tiling and the split follow one item's rows (all of x for a plain
    // product): every row's arithmetic is then that of its item's own call
    const TcPlan plan = plan_tc(item_rows > 0 ? item_rows : M, N, K, num_sms, bn_step(bits, transpose),
                                bn_step2(bits, transpose));
    const int bn = plan.bn;
    const int ms = plan.ms;
    CUtensorMap map_x, map_c;
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
        cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(BM * ms)};
        cuuint32_t es[2] = {1, 1};
        if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    if (!transpose) {
        // weights [K, N]: boxes of 64 k-rows x bn columns (bn * bits / 32 words)
        const int64_t wpr = N * bits / 32;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(K)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(wpr) * 4};
        cuuint32_t box[2] = {static_cast<cuuint32_t>(bn * bits / 32), static_cast<cuuint32_t>(BK)};
        cuuint32_t es[2] = {1, 1};
        if (enc(&map_c, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    } else {
        const int64_t wpr = K * bits / 32;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(wpr) * 4};
        cuuint32_t box[2] = {static_cast<cuuint32_t>(BK * bits / 32), static_cast<cuuint32_t>(bn)};
        cuuint32_t es[2] = {1, 1};
        // 32/64-byte swizzle of the code rows: the dequant threads' row reads
        // then fall on distinct banks
        const CUtensorMapSwizzle swz = bits == 4   ? CU_TENSOR_MAP_SWIZZLE_32B
                                       : bits == 8 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_NONE;
        if (enc(&map_c, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    // scales and biases: blocks of 8 groups x bn rows, when rows are 16-byte multiples
    CUtensorMap map_s, map_b;
    const int64_t gpr = K / gs;
    const bool sb_tma = fmt == 0 && transpose && (gpr * 2) % 16 == 0;  // else loaded directly
    if (sb_tma) {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(gpr), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(gpr) * 2};
        cuuint32_t box[2] = {8, static_cast<cuuint32_t>(bn)};
        cuuint32_t es[2] = {1, 1};
        for (int i = 0; i < 2; ++i)
            if (enc(i ? &map_b : &map_s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(i ? biases : scales), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
    } else {
        map_s = map_c;
        map_b = map_c;
    }
    TcParams prm{};
    prm.sb_tma = sb_tma ? 1 : 0;
    prm.m2 = 2;
    prm.m4 = 4;
    prm.m6 = 6;
    prm.lg_gs = gs == 16 ? 4 : gs == 32 ? 5 : gs == 64 ? 6 : 7;
    prm.y = static_cast<uint16_t*>(y);
    prm.scales = static_cast<const uint16_t*>(scales);
    prm.biases = static_cast<const uint16_t*>(biases);
    prm.M = M;
    prm.N = N;
    prm.K = K;
    prm.gs = gs;
    prm.bn = bn;
    prm.m_tiles = static_cast<int>((M + BM * ms - 1) / (BM * ms));
    prm.n_tiles = static_cast<int>((N + bn - 1) / bn);
    const uint32_t a_stage = BM * BK * 2 * ms;                    // 16 KB per row subtile, 1024-aligned
    const uint32_t b_stage = static_cast<uint32_t>(bn) * BK * 2;  // bn * 128
    const uint32_t c_stage = (static_cast<uint32_t>(bn) * BK * bits / 8 + 1023) / 1024 * 1024;
    const uint32_t per_stage = a_stage + b_stage + c_stage;
    const uint32_t sb_ring = 2u * 2u * static_cast<uint32_t>(bn) * 16u;  // 2 slots x (s, b)
    const uint32_t budget = 227 * 1024 - 1024 - 512 - sb_ring;
    int stages = static_cast<int>(budget / per_stage);
    if (stages > 6) stages = 6;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    prm.stages = stages;
    prm.a_off = 0;
    prm.b_off = a_stage * stages;
    prm.c_off = prm.b_off + b_stage * stages;
    prm.sb_off = prm.c_off + c_stage * stages;
    prm.bar_off = prm.sb_off + sb_ring;
    prm.b_stage_bytes = b_stage;
    prm.c_stage_bytes = c_stage;
    prm.tmem_cols = 2 * ms * bn <= 256 ? 256 : 512;
    prm.splits = plan.splits;
    const size_t smem = prm.bar_off + (4 * stages + 8) * 8 + 16 + 1024;  // + alignment slack
    const int tiles = prm.m_tiles * prm.n_tiles;
    using Kern = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                          const TcParams);
    if (plan.splits == 1) {
        const int grid = tiles < num_sms ? tiles : num_sms;
        Kern k;
        if (fmt != 0)
            k = ms == 2 ? (fmt == 1 ? tc_qmm_kernel<4, false, false, 2, 1>
                           : fmt == 2 ? tc_qmm_kernel<8, false, false, 2, 2>
                                      : tc_qmm_kernel<4, false, false, 2, 3>)
                        : (fmt == 1 ? tc_qmm_kernel<4, false, false, 1, 1>
                           : fmt == 2 ? tc_qmm_kernel<8, false, false, 1, 2>
                                      : tc_qmm_kernel<4, false, false, 1, 3>);
        else if (ms == 2)
            k = transpose ? (bits == 4 ? tc_qmm_kernel<4, false, false, 2>
                             : bits == 8 ? tc_qmm_kernel<8, false, false, 2>
                                         : tc_qmm_kernel<2, false, false, 2>)
                          : (bits == 4 ? tc_qmm_kernel<4, false, true, 2>
                             : bits == 8 ? tc_qmm_kernel<8, false, true, 2>
                                         : tc_qmm_kernel<2, false, true, 2>);
        else
            k = transpose ? (bits == 4 ? tc_qmm_kernel<4, false, false>
                             : bits == 8 ? tc_qmm_kernel<8, false, false>
                                         : tc_qmm_kernel<2, false, false>)
                          : (bits == 4 ? tc_qmm_kernel<4, false, true>
                             : bits == 8 ? tc_qmm_kernel<8, false, true>
                                         : tc_qmm_kernel<2, false, true>);
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        k<<<grid, kThreads, smem, stream>>>(map_x, map_c, map_s, map_b, prm);
        return cudaGetLastError();
    }
    // split-K: one cluster of `splits` CTAs per tile; the partial tile
    // ([128][bn] fp32) reuses the pipeline's stages in shared memory
    if (static_cast<size_t>(BM) * bn * 4 > prm.sb_off) return cudaErrorInvalidConfiguration;
    Kern k = fmt == 1   ? tc_qmm_kernel<4, true, false, 1, 1>
             : fmt == 2 ? tc_qmm_kernel<8, true, false, 1, 2>
             : fmt == 3 ? tc_qmm_kernel<4, true, false, 1, 3>
             : transpose ? (bits == 4 ? tc_qmm_kernel<4, true, false>
                            : bits == 8 ? tc_qmm_kernel<8, true, false>
                                        : tc_qmm_kernel<2, true, false>)
                         : (bits == 4 ? tc_qmm_kernel<4, true, true>
                            : bits == 8 ? tc_qmm_kernel<8, true, true>
                                        : tc_qmm_kernel<2, true, true>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * plan.splits), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(plan.splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k, map_x, map_c, map_s, map_b, prm);
}

// Floating-point modes on the tiled kernel (weights [N, K]; mode 1 = MXFP4,
// 2 = MXFP8, 3 = NVFP4).
bool qmm_fp_tiled_supported(int64_t K, int mode) {
    return K % BK == 0 && K >= BK && mode >= 1 && mode <= 3;
}

cudaError_t launch_tc_qmm_fp(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                             const uint8_t* scales, int mode, void* y, cudaStream_t stream, int num_sms) {
    const int bits = mode == 2 ? 8 : 4, gs = mode == 3 ? 16 : 32;
    return launch_tc_qmm(x, M, K, N, codes, scales, nullptr, gs, bits, y, stream, num_sms, 0, 1, mode);
}

}  // namespace nvq
