// Quantized vector-matrix products for 1 to 8 rows of bf16 activations with
// the weights stored [K, N], grouped along N: y = x . w, the transpose = false
// form of quantized_matmul ("Docs / Quantization", section "Affine";
// GatherQmm and quantized_matmul take a transpose flag, nuvec crate docs).
//
// Here the scale varies along the contraction (one per k-row and group of
// columns): every weight is dequantized first, w = s[k, g(n)] * code[k, n] +
// b[k, g(n)] (one fp32 fused multiply-add on the exact code), and then
// y[n] += x_k * w. Keeping scale * code and bias in one term matters: summed
// apart they can cancel (a weight that dequantizes to exactly 0 under a huge
// activation). Design (sm_100a):
//  * A thread owns TW consecutive code words of a k-row (one group) and walks
//    k-rows; a warp reads consecutive columns of one k-row (coalesced).
//  * Codes become exact fp32 values without int->float conversions: a field
//    masked into the mantissa of 2^23 gives 2^23 + c * 2^e exactly, and one
//    packed fma.rn.f32x2 per two codes rescales and removes the 2^23.
//  * Dequantization and multiply-adds use packed fma.rn.f32x2 (two columns
//    per instruction).
//  * K is split between the two CTAs of a cluster and over kp thread-rows of a
//    CTA (64, or 32 / 16 where a CTA spans many columns, so that one CTA per
//    SM covers the whole output in one wave); the partial sums are reduced in
//    a fixed order (thread-rows through shared memory, then the cluster's two
//    halves through distributed shared memory), so results are deterministic.
//    kp follows N, bits and the group size only, so every output is computed
//    by the same operations whatever M is (row exactness).
#include <algorithm>
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace nvq {
namespace {

constexpr int KP = 64;          // most thread-rows (k-parts) per CTA
constexpr int KP_ROUND = 16;    // thread-rows reduced per shared-memory round (kp >= 16)
constexpr int kClusterK = 2;    // CTAs per cluster, splitting K

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t pack2u(uint32_t lo, uint32_t hi) {
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

template <int BITS>
struct Codes {
    static constexpr int PER = 32 / BITS;
    static constexpr int PAIRS = PER / 2;
    // Column (within the word) of the low / high element of pair j.
    __device__ static constexpr int col(int j, int h) {
        if constexpr (BITS == 4) return h ? j + 4 : j;
        else if constexpr (BITS == 8) return h ? j + 2 : j;
        else return h ? j + 8 : j;
    }
    // Exact codes of a word as fp32 pairs (col(j,0), col(j,1)).
    __device__ static __forceinline__ void to_f32(uint32_t w, uint64_t* c) {
        constexpr uint32_t MAGIC = 0x4B000000u;  // 2^23
        if constexpr (BITS == 4) {
            const uint32_t w2 = w >> 12;         // nibbles 3..7 at bits 0..19
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t lo = (w & (0xFu << (4 * j))) | MAGIC;         // 2^23 + c_j 2^(4j)
                const uint32_t hi = (w2 & (0xFu << (4 * j + 4))) | MAGIC;    // 2^23 + c_(j+4) 2^(4j+4)
                const float slo = __uint_as_float((127u - 4 * j) << 23);
                const float shi = __uint_as_float((127u - 4 * j - 4) << 23);
                const float olo = -__uint_as_float((127u + 23 - 4 * j) << 23);
                const float ohi = -__uint_as_float((127u + 19 - 4 * j) << 23);
                c[j] = fma2(pack2u(lo, hi), pack2(slo, shi), pack2(olo, ohi));
            }
        } else if constexpr (BITS == 8) {
            const uint32_t w2 = w >> 16;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t lo = (w & (0xFFu << (8 * j))) | MAGIC;
                const uint32_t hi = (w2 & (0xFFu << (8 * j))) | MAGIC;
                const float sc = __uint_as_float((127u - 8 * j) << 23);
                const float of = -__uint_as_float((127u + 23 - 8 * j) << 23);
                c[j] = fma2(pack2u(lo, hi), pack2(sc, sc), pack2(of, of));
            }
        } else {
            const uint32_t w2 = w >> 16;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t lo = (w & (0x3u << (2 * j))) | MAGIC;
                const uint32_t hi = (w2 & (0x3u << (2 * j))) | MAGIC;
                const float sc = __uint_as_float((127u - 2 * j) << 23);
                const float of = -__uint_as_float((127u + 23 - 2 * j) << 23);
                c[j] = fma2(pack2u(lo, hi), pack2(sc, sc), pack2(of, of));
            }
        }
    }
};

template <int TW>
__device__ __forceinline__ void load_tw(const uint32_t* p, uint32_t* w) {
    if constexpr (TW == 1) {
        w[0] = __ldg(p);
    } else if constexpr (TW == 2) {
        uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = v.x; w[1] = v.y;
    } else {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    }
}

struct QmvtParams {
    const uint16_t* x;  // bf16 [M, K]
    const uint32_t* codes;   // [K, N*bits/32]
    const uint16_t* scales;  // [K, N/gs]
    const uint16_t* biases;
    uint16_t* y;             // bf16 [M, N]
    int64_t N, K;
    int M;
    int gs;
    int64_t ncols;           // column units (TW words each)
    int ranges;              // CTAs along the columns
    int ctm;                 // max column units per CTA
    int kp;                  // thread-rows (k-parts) per CTA: 64, 32 or 16
};

constexpr int kMaxThreads = 512;  // column units per CTA x thread-rows

template <int BITS, int TW, int MT>
__global__ void __cluster_dims__(1, kClusterK, 1) __launch_bounds__(kMaxThreads)
qmvt_kernel(const QmvtParams prm) {
    // launched as the programmatic dependent of the previous kernel: the next
    // product may launch at once; this one waits for the previous grid before
    // its first read (x or the weights may come from it)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    using C = Codes<BITS>;
    constexpr int COLS_T = TW * C::PER;   // columns a thread owns
    extern __shared__ float smem[];       // [KP_ROUND][MT][ctm * COLS_T], then [MT][ctm * COLS_T]
    cg::cluster_group cluster = cg::this_cluster();

    const int ctm = prm.ctm;
    const int ct = threadIdx.x % ctm;
    const int p = threadIdx.x / ctm;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * prm.ncols / prm.ranges;
    const int64_t c1 = static_cast<int64_t>(blockIdx.x + 1) * prm.ncols / prm.ranges;
    const int ncol = static_cast<int>(c1 - c0);
    const int rank = static_cast<int>(cluster.block_rank());
    const int64_t K = prm.K, N = prm.N;
    const int64_t kr0 = rank * K / kClusterK, kr1 = (rank + 1) * K / kClusterK;
    const int64_t wpr = N * BITS / 32;  // words per k-row
    const int64_t gpr = N / prm.gs;     // groups per k-row
    const int M = prm.M;
    const int kp = prm.kp;
    const bool active = ct < ncol && p < kp;

    uint64_t acc[MT][TW][C::PAIRS];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int w = 0; w < TW; ++w)
#pragma unroll
            for (int j = 0; j < C::PAIRS; ++j) acc[m][w][j] = 0ull;

    if (active) {
        const int64_t word0 = (c0 + ct) * TW;
        const int64_t grp = word0 * C::PER / prm.gs;
        const uint32_t* cp = prm.codes + word0;
        const uint16_t* sp = prm.scales + grp;
        const uint16_t* bp = prm.biases + grp;
        // Loads in flight per thread; halved where 64 accumulators fill the registers.
        constexpr int U = MT * COLS_T >= 64 ? 2 : MT * COLS_T > 32 ? 4 : 8;
        int64_t k = kr0 + p;
        for (; k + (U - 1) * kp < kr1; k += U * kp) {
            uint32_t wv[U][TW];
            float sv[U], bv[U], xv[U][MT];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t kk = k + u * kp;
                load_tw<TW>(cp + kk * wpr, wv[u]);
                sv[u] = bf16_bits_to_f32(__ldg(sp + kk * gpr));
                bv[u] = bf16_bits_to_f32(__ldg(bp + kk * gpr));
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    xv[u][m] = m < M ? bf16_bits_to_f32(__ldg(prm.x + m * K + kk)) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint64_t s2 = pack2(sv[u], sv[u]), b2 = pack2(bv[u], bv[u]);
#pragma unroll
                for (int w = 0; w < TW; ++w) {
                    uint64_t cv[C::PAIRS];
                    C::to_f32(wv[u][w], cv);
#pragma unroll
                    for (int j = 0; j < C::PAIRS; ++j) cv[j] = fma2(s2, cv[j], b2);  // the weights
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const uint64_t x2 = pack2(xv[u][m], xv[u][m]);
#pragma unroll
                        for (int j = 0; j < C::PAIRS; ++j) acc[m][w][j] = fma2(x2, cv[j], acc[m][w][j]);
                    }
                }
            }
        }
        for (; k < kr1; k += kp) {
            uint32_t wv[TW];
            load_tw<TW>(cp + k * wpr, wv);
            const float s = bf16_bits_to_f32(__ldg(sp + k * gpr));
            const float b = bf16_bits_to_f32(__ldg(bp + k * gpr));
            float xv[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) xv[m] = m < M ? bf16_bits_to_f32(__ldg(prm.x + m * K + k)) : 0.f;
            const uint64_t s2 = pack2(s, s), b2 = pack2(b, b);
#pragma unroll
            for (int w = 0; w < TW; ++w) {
                uint64_t cv[C::PAIRS];
                C::to_f32(wv[w], cv);
#pragma unroll
                for (int j = 0; j < C::PAIRS; ++j) cv[j] = fma2(s2, cv[j], b2);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint64_t x2 = pack2(xv[m], xv[m]);
#pragma unroll
                    for (int j = 0; j < C::PAIRS; ++j) acc[m][w][j] = fma2(x2, cv[j], acc[m][w][j]);
                }
            }
        }
    }

    // ---- fixed-order reduction over the kp thread-rows, 16 per round ----
    const int cols_cta = ctm * COLS_T;            // columns of the CTA's buffer
    const int entries = MT * cols_cta;
    float* buf = smem;                            // [KP_ROUND][MT][cols_cta]
    float* out = smem + KP_ROUND * entries;       // [MT][cols_cta]
    const int nthreads = blockDim.x;
    // each thread owns entries e = threadIdx.x + i * nthreads
    constexpr int kMaxOwn = 4;
    float run[kMaxOwn];
#pragma unroll
    for (int i = 0; i < kMaxOwn; ++i) run[i] = 0.f;
    for (int r0 = 0; r0 < kp; r0 += KP_ROUND) {
        if (p >= r0 && p < r0 + KP_ROUND && ct < ctm) {
            float* dst = buf + (p - r0) * entries;
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int w = 0; w < TW; ++w)
#pragma unroll
                    for (int j = 0; j < C::PAIRS; ++j) {
                        float lo, hi;
                        unpack2(acc[m][w][j], lo, hi);
                        const int cb = ct * COLS_T + w * C::PER;
                        dst[m * cols_cta + cb + C::col(j, 0)] = lo;
                        dst[m * cols_cta + cb + C::col(j, 1)] = hi;
                    }
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kMaxOwn; ++i) {
            const int e = threadIdx.x + i * nthreads;
            if (e < entries)
                for (int q = 0; q < KP_ROUND; ++q) run[i] += buf[q * entries + e];
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < kMaxOwn; ++i) {
        const int e = threadIdx.x + i * nthreads;
        if (e < entries) out[e] = run[i];
    }

    // ---- the two K halves of the cluster: rank 0 adds rank 1's sums ----
    cluster.sync();
    if (rank == 0) {
        const float* other = cluster.map_shared_rank(out, 1);
        const int ncols_n = ncol * COLS_T;
        const int64_t n_base = c0 * TW * C::PER;
        for (int i = threadIdx.x; i < M * ncols_n; i += nthreads) {
            const int m = i / ncols_n, c = i % ncols_n;
            const float v = out[m * cols_cta + c] + other[m * cols_cta + c];
            prm.y[m * N + n_base + c] = f32_to_bf16_bits(v);
        }
    }
    cluster.sync();
}

template <int BITS, int TW, int MT>
cudaError_t launch_one(const QmvtParams& prm0, int num_sms, cudaStream_t stream) {
    QmvtParams prm = prm0;
    using C = Codes<BITS>;
    const int cols_t = TW * C::PER;
    // Column ranges: one cluster (two CTAs) per two SMs, each CTA at most
    // kMaxThreads / kp column units wide; wider outputs take more ranges.
    int64_t ranges = std::max<int64_t>(1, num_sms / kClusterK);
    ranges = std::min<int64_t>(ranges, prm.ncols);
    const int64_t max_units = kMaxThreads / prm.kp;
    while ((prm.ncols + ranges - 1) / ranges > max_units) ranges *= 2;
    prm.ranges = static_cast<int>(ranges);
    prm.ctm = static_cast<int>((prm.ncols + ranges - 1) / ranges);
    const int threads = prm.ctm * prm.kp;
    const size_t entries = static_cast<size_t>(MT) * prm.ctm * cols_t;
    if ((entries + threads - 1) / threads > 4) return cudaErrorInvalidConfiguration;
    const size_t smem = (KP_ROUND + 1) * entries * sizeof(float);
    auto k = qmvt_kernel<BITS, TW, MT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ranges), kClusterK, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, prm);
}

// Words per thread: as many as fit 64 accumulators per thread, within a group.
int tw_for(int bits, int gs, int mt) {
    const int per = 32 / bits;
    const int gw = gs * bits / 32;
    int tw = 4;
    while (tw > 1 && (mt * tw * per > 64 || tw > gw)) tw /= 2;
    if (mt * tw * per > 64 || tw > gw) return 0;
    return tw;
}

template <int BITS, int MT>
cudaError_t dispatch_tw(int tw, const QmvtParams& prm, int num_sms, cudaStream_t s) {
    constexpr int PER = 32 / BITS;
    if constexpr (MT * 4 * PER <= 64) {
        if (tw == 4) return launch_one<BITS, 4, MT>(prm, num_sms, s);
    }
    if constexpr (MT * 2 * PER <= 64) {
        if (tw == 2) return launch_one<BITS, 2, MT>(prm, num_sms, s);
    }
    if constexpr (MT * PER <= 64) {
        if (tw == 1) return launch_one<BITS, 1, MT>(prm, num_sms, s);
    }
    return cudaErrorInvalidValue;
}

template <int BITS>
cudaError_t dispatch_m(int mt, int tw, const QmvtParams& prm, int num_sms, cudaStream_t s) {
    switch (mt) {
        case 1: return dispatch_tw<BITS, 1>(tw, prm, num_sms, s);
        case 2: return dispatch_tw<BITS, 2>(tw, prm, num_sms, s);
        case 4: return dispatch_tw<BITS, 4>(tw, prm, num_sms, s);
        default:
            if constexpr (BITS != 2) return dispatch_tw<BITS, 8>(tw, prm, num_sms, s);
            return cudaErrorInvalidValue;
    }
}

int mt_for(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

// Thread-rows per CTA: 64 unless the one-row plan's CTAs would span more
// column units than 512 threads hold at 64 rows each. A function of N, bits
// and the group size only, so every M sums each output in the same order.
int kp_for(int64_t N, int bits, int gs, int num_sms) {
    const int tw = tw_for(bits, gs, 1);
    const int64_t ncols = N * bits / 32 / tw;
    const int64_t ranges = std::max<int64_t>(1, std::min<int64_t>(num_sms / kClusterK, ncols));
    const int64_t ctm = (ncols + ranges - 1) / ranges;
    int kp = KP;
    while (kp > KP_ROUND && ctm * kp > kMaxThreads) kp /= 2;
    return kp;
}

}  // namespace

bool qmvt_supported(int bits, int gs) {
    return (bits == 2 || bits == 4 || bits == 8) && (gs == 32 || gs == 64 || gs == 128);
}

bool qmvt_supported_m(int bits, int gs, int64_t M) {
    return qmvt_supported(bits, gs) && tw_for(bits, gs, mt_for(M)) > 0;
}

cudaError_t launch_qmvt(const void* x, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                        const void* scales, const void* biases, int gs, int bits, void* y,
                        cudaStream_t stream, int num_sms) {
    const int mt = mt_for(M);
    const int tw = tw_for(bits, gs, mt);
    if (tw == 0) return cudaErrorInvalidValue;
    QmvtParams prm{};
    prm.x = static_cast<const uint16_t*>(x);
    prm.codes = codes;
    prm.scales = static_cast<const uint16_t*>(scales);
    prm.biases = static_cast<const uint16_t*>(biases);
    prm.y = static_cast<uint16_t*>(y);
    prm.N = N;
    prm.K = K;
    prm.M = static_cast<int>(M);
    prm.gs = gs;
    prm.ncols = N * bits / 32 / tw;
    prm.kp = kp_for(N, bits, gs, num_sms);
    switch (bits) {
        case 2: return dispatch_m<2>(mt, tw, prm, num_sms, stream);
        case 4: return dispatch_m<4>(mt, tw, prm, num_sms, stream);
        case 8: return dispatch_m<8>(mt, tw, prm, num_sms, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace nvq
