// Routing for gather_qmm ("Docs / Quantization", section "Mixture of experts":
// with rows sorted by expert a grouped kernel reads each expert's weights once).
//
// One CTA turns the pair list (lhs token, rhs expert) into:
//   * offsets[E + 2]: where each expert's pairs start in expert order (bucket E
//     collects pairs whose expert or token id is out of range; they get zeros);
//   * perm[R]: the pairs stably sorted by expert (a counting sort, so pairs of
//     one expert keep their input order and the result is deterministic);
//   * problems: (expert, first sorted position, count <= 8) work items for the
//     grouped matrix-vector kernel, expert by expert;
//   * flags: out-of-range ids, and a broken "sorted" promise.
// Ranks inside a warp come from __match_any_sync; warps own contiguous pair
// segments and get their per-expert bases from a scan of per-warp histograms.
#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace nvq {
namespace {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive scan of one value per thread over the CTA; returns the total too.
__device__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = warp_sums[lane];
        uint32_t si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t n = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += n;
        }
        warp_sums[lane] = si - s;  // exclusive
        if (lane == 31) warp_sums[32] = si;
    }
    __syncthreads();
    const uint32_t r = warp_sums[warp] + inc - v;
    total = warp_sums[32];
    __syncthreads();
    return r;
}

// Pairs per lane whose keys stay in registers between the histogram and the
// scatter (a warp's segment of up to 32 * kKeyRegs pairs is read once; longer
// segments read the rest again in the scatter).
constexpr int kKeyRegs = 4;

__global__ void __launch_bounds__(kRouteThreads, 1) gather_route_kernel(
    const uint32_t* __restrict__ lhs, const uint32_t* __restrict__ rhs, int64_t R, int E,
    int64_t x_rows, int sorted, int want_problems, uint32_t* __restrict__ flags_out,
    uint32_t* __restrict__ num_problems, uint32_t* __restrict__ offsets_out,
    uint32_t* __restrict__ perm, uint32_t* __restrict__ problems) {
    extern __shared__ uint32_t hist[];  // [kRouteWarps][E + 1], then bucket offsets [E + 1]
    __shared__ uint32_t warp_sums[33];
    __shared__ uint32_t s_flags;
    const int NB = E + 1;  // buckets: experts, then "invalid"
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the grouped product may launch now; it waits for this grid to finish
    // before it reads the tables
    pdl_launch_dependents();
    // launched as a programmatic dependent itself: the previous kernel (the
    // last call's grouped product, which may still read tables of a shared
    // workspace, or the kernel that wrote the ids) ends before any access here
    pdl_wait();

    for (int i = threadIdx.x; i < kRouteWarps * NB; i += kRouteThreads) hist[i] = 0;
    if (threadIdx.x == 0) s_flags = 0;

    const int64_t seg0 = warp * R / kRouteWarps, seg1 = (warp + 1) * R / kRouteWarps;
    uint32_t my_flags = 0;
    auto key_of = [&](int64_t r, bool check) -> int {
        const uint32_t e = __ldg(rhs + r);
        const int64_t t = lhs ? static_cast<int64_t>(__ldg(lhs + r)) : r;
        if (check) {
            if (e >= static_cast<uint32_t>(E)) my_flags |= NV_FLAG_EXPERT_OUT_OF_RANGE;
            if (t >= x_rows) my_flags |= NV_FLAG_TOKEN_OUT_OF_RANGE;
            if (sorted && r > 0 && e < __ldg(rhs + r - 1)) my_flags |= NV_FLAG_NOT_SORTED;
        }
        return (e < static_cast<uint32_t>(E) && t < x_rows) ? static_cast<int>(e) : E;
    };
    // the first kKeyRegs chunks of the segment: all loads issued before any use
    int key[kKeyRegs];
#pragma unroll
    for (int i = 0; i < kKeyRegs; ++i) {
        const int64_t r = seg0 + 32 * i + lane;
        key[i] = r < seg1 ? key_of(r, true) : NB;
    }
    __syncthreads();  // histograms zeroed

    // Phase 1: per-warp histograms.
    auto count_key = [&](int k) {
        const uint32_t mask = __match_any_sync(0xffffffffu, k);
        if (k < NB && lane == __ffs(mask) - 1) hist[warp * NB + k] += __popc(mask);
        __syncwarp();
    };
#pragma unroll
    for (int i = 0; i < kKeyRegs; ++i) count_key(key[i]);
    for (int64_t c = seg0 + 32 * kKeyRegs; c < seg1; c += 32) {
        const int64_t r = c + lane;
        count_key(r < seg1 ? key_of(r, true) : NB);
    }
    if (my_flags) atomicOr(&s_flags, my_flags);
    __syncthreads();

    // Phase 2: per-bucket totals and per-warp bases within a bucket (warp w
    // scans buckets w, w + 32, ...: lane l holds warp l's count), then the
    // bucket offsets.
    uint32_t* cnt = hist + kRouteWarps * NB;  // bucket totals, then offsets
    for (int bk = warp; bk < NB; bk += kRouteWarps) {
        const uint32_t h = hist[lane * NB + bk];
        uint32_t inc = h;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += n;
        }
        hist[lane * NB + bk] = inc - h;
        if (lane == 31) cnt[bk] = inc;
    }
    __syncthreads();
    const int b = threadIdx.x;  // NB <= kRouteThreads
    const uint32_t count = b < NB ? cnt[b] : 0u;
    uint32_t total;
    const uint32_t off = block_exclusive_scan(count, warp_sums, total);
    if (b < NB) {
        offsets_out[b] = off;
        cnt[b] = off;  // bucket offsets for phase 3 (each thread rewrites its own entry)
    }
    if (b == 0) offsets_out[NB] = total;
    if (want_problems) {
        // Problems: ceil(count / 8) per bucket, bucket by bucket.
        const uint32_t np = (count + 7) / 8;
        uint32_t np_total;
        const uint32_t poff = block_exclusive_scan(b < NB ? np : 0u, warp_sums, np_total);
        if (b < NB) {
            for (uint32_t i = 0; i < np; ++i) {
                uint32_t* pr = problems + 4 * (poff + i);
                pr[0] = static_cast<uint32_t>(b);
                pr[1] = off + 8 * i;
                pr[2] = min(8u, count - 8 * i);
                pr[3] = 0;
            }
        }
        if (b == 0) *num_problems = np_total;
    }
    __syncthreads();

    // Phase 3: stable scatter into expert order.
    auto place = [&](int64_t r, int k) {
        const uint32_t mask = __match_any_sync(0xffffffffu, k);
        if (k < NB) perm[cnt[k] + hist[warp * NB + k] + __popc(mask & lanemask_lt())] = static_cast<uint32_t>(r);
        __syncwarp();
        if (k < NB && lane == __ffs(mask) - 1) hist[warp * NB + k] += __popc(mask);
        __syncwarp();
    };
#pragma unroll
    for (int i = 0; i < kKeyRegs; ++i) place(seg0 + 32 * i + lane, key[i]);
    for (int64_t c = seg0 + 32 * kKeyRegs; c < seg1; c += 32) {
        const int64_t r = c + lane;
        place(r, r < seg1 ? key_of(r, false) : NB);
    }
    if (threadIdx.x == 0) *flags_out = s_flags;
}

size_t pad16(size_t b) { return (b + 15) & ~static_cast<size_t>(15); }

}  // namespace

size_t gather_workspace_bytes(int64_t R, int64_t E) {
    const int64_t max_problems = (R + 7) / 8 + E + 1;
    return 16 + pad16((E + 2) * 4) + pad16(R * 4) + static_cast<size_t>(max_problems) * 16;
}

GatherWorkspace gather_workspace_carve(void* base, int64_t R, int64_t E) {
    GatherWorkspace ws;
    char* p = static_cast<char*>(base);
    ws.flags = reinterpret_cast<uint32_t*>(p);
    ws.num_problems = reinterpret_cast<uint32_t*>(p + 4);
    p += 16;
    ws.offsets = reinterpret_cast<uint32_t*>(p);
    p += pad16((E + 2) * 4);
    ws.perm = reinterpret_cast<uint32_t*>(p);
    p += pad16(R * 4);
    ws.problems = reinterpret_cast<uint32_t*>(p);
    ws.max_problems = (R + 7) / 8 + E + 1;
    return ws;
}

cudaError_t launch_gather_route(const uint32_t* lhs, const uint32_t* rhs, int64_t R, int64_t E,
                                int64_t x_rows, int sorted, const GatherWorkspace& ws,
                                cudaStream_t stream, bool want_problems) {
    const int NB = static_cast<int>(E) + 1;
    // per-warp histograms plus one row of bucket offsets
    const size_t smem = static_cast<size_t>(kRouteWarps + 1) * NB * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(gather_route_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(kRouteThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gather_route_kernel, lhs, rhs, R, static_cast<int>(E), x_rows, sorted,
                              want_problems ? 1 : 0, ws.flags, ws.num_problems, ws.offsets, ws.perm,
                              ws.problems);
}

}  // namespace nvq
