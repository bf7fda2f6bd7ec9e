// The routed SwiGLU mixture-of-experts block over quantized experts
// ("Docs / Quantization", section "Mixture of experts": every row is
// multiplied by its own expert's quantized weights, read in place; the block
// around gather_qmm is gate and up products, silu(gate) * up, the down
// product, and the routing weights' sum over each token's experts).
//
// One routed pass, all on the GPU:
//   1. pair r = t * topk + j of token t and its j-th expert ids[t, j]; a small
//      kernel writes the pairs' token ids, the router (the same one
//      gather_qmm uses) sorts the pairs by expert once for the three products;
//   2. gate: the grouped tensor-core kernel, x rows -> g [R, I] (bf16);
//   3. up: the same kernel with its SwiGLU epilogue: h = silu(g) * (x . w_up)
//      written over g in place;
//   4. down: the grouped kernel on the pairs' own h rows -> d [R, K] (bf16);
//   5. combine: y[t] = sum_j rw[t, j] * d[t * topk + j], fp32 in j order,
//      rounded once to bf16.
// Every step has a fixed order, so results are deterministic. Pairs whose
// expert id is out of range get zero rows (and a flag) in every product, so
// they add nothing to y.
#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace nvq {
namespace {

__global__ void pair_tokens_kernel(uint32_t* __restrict__ lhs, int64_t R, int topk) {
    // a programmatic dependent: waits for the previous grid before writing
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < R;
         r += static_cast<int64_t>(gridDim.x) * blockDim.x)
        lhs[r] = static_cast<uint32_t>(r / topk);
}

// y[t, n] = sum_j rw[t, j] * d[t * topk + j, n]: eight columns per thread
// (16-byte loads and stores), j in order.
__global__ void combine_kernel(const uint16_t* __restrict__ d, const float* __restrict__ rw,
                               int64_t T, int64_t K, int topk, uint16_t* __restrict__ y) {
    // a programmatic dependent of the down product: waits for it before reading d
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t chunks = K / 8;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < T * chunks;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / chunks, c = i - t * chunks;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < topk; ++j) {
            const float w = __ldg(rw + t * topk + j);
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(d + (t * topk + j) * K) + c);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                acc[2 * h] = fmaf(w, bf16_bits_to_f32(u[h] & 0xFFFFu), acc[2 * h]);
                acc[2 * h + 1] = fmaf(w, bf16_bits_to_f32(u[h] >> 16), acc[2 * h + 1]);
            }
        }
        uint4 o;
        o.x = f32_to_bf16_bits(acc[0]) | (static_cast<uint32_t>(f32_to_bf16_bits(acc[1])) << 16);
        o.y = f32_to_bf16_bits(acc[2]) | (static_cast<uint32_t>(f32_to_bf16_bits(acc[3])) << 16);
        o.z = f32_to_bf16_bits(acc[4]) | (static_cast<uint32_t>(f32_to_bf16_bits(acc[5])) << 16);
        o.w = f32_to_bf16_bits(acc[6]) | (static_cast<uint32_t>(f32_to_bf16_bits(acc[7])) << 16);
        reinterpret_cast<uint4*>(y + t * K)[c] = o;
    }
}

size_t pad256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct MoeWorkspace {
    void* route;      // gather_workspace_bytes(R, E); the flags come first
    uint32_t* lhs;    // [R]
    uint16_t* gh;     // [R, I]: gate, then silu(gate) * up
    uint16_t* d;      // [R, K]
    size_t bytes;
};

MoeWorkspace moe_carve(void* base, int64_t R, int64_t E, int64_t I, int64_t K) {
    MoeWorkspace w{};
    char* p = static_cast<char*>(base);
    size_t off = 0;
    w.route = p + off;
    off += pad256(gather_workspace_bytes(R, E));
    w.lhs = reinterpret_cast<uint32_t*>(p + off);
    off += pad256(static_cast<size_t>(R) * 4);
    w.gh = reinterpret_cast<uint16_t*>(p + off);
    off += pad256(static_cast<size_t>(R) * I * 2);
    w.d = reinterpret_cast<uint16_t*>(p + off);
    off += pad256(static_cast<size_t>(R) * K * 2);
    w.bytes = off;
    return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace nvq

extern "C" {

size_t nv_moe_swiglu_workspace_size(int64_t T, int64_t topk, int64_t E, int64_t I, int64_t K) {
    if (T < 0 || topk < 1 || E < 1 || I < 1 || K < 1) return 0;
    return nvq::moe_carve(nullptr, T * topk, E, I, K).bytes;
}

nv_status nv_moe_swiglu(const void* x, nv_dtype dt, int64_t T, int64_t K, const uint32_t* ids,
                        const float* rw, int topk, int64_t E, int64_t I,
                        const uint32_t* gate_codes, const void* gate_scales,
                        const void* gate_biases, const uint32_t* up_codes, const void* up_scales,
                        const void* up_biases, const uint32_t* down_codes,
                        const void* down_scales, const void* down_biases, int group_size,
                        int bits, void* workspace, size_t workspace_bytes, void* y,
                        nv_stream_t stream) {
    using nvq::aligned16;
    if (dt != NV_BF16 && dt != NV_F32) return NV_ERR_UNSUPPORTED;
    if (bits == 3 || bits == 5 || bits == 6 || bits == 1) return NV_ERR_UNSUPPORTED;
    if (bits != 2 && bits != 4 && bits != 8) return NV_ERR_INVALID_ARG;
    if (group_size != 32 && group_size != 64 && group_size != 128) return NV_ERR_INVALID_ARG;
    if (T < 0 || K <= 0 || I <= 0 || E <= 0 || topk < 1 || topk > 64) return NV_ERR_INVALID_ARG;
    if (K % group_size || I % group_size) return NV_ERR_INVALID_ARG;
    if (E > nvq::kMaxExperts) return NV_ERR_UNSUPPORTED;
    if (T > (int64_t(1) << 31) / topk) return NV_ERR_INVALID_ARG;
    // the grouped tensor-core kernels run every product: bf16 only, K and I
    // multiples of 128 with 16-byte rows of scales, K a multiple of 8 for the combine
    if (dt != NV_BF16 || !nvq::tc_gather_supported(K, I, bits, group_size) ||
        !nvq::tc_gather_supported(I, K, bits, group_size) || K % 8)
        return NV_ERR_UNSUPPORTED;
    const int64_t R = T * topk;
    if (R * (K > I ? K : I) >= (int64_t(1) << 35)) return NV_ERR_UNSUPPORTED;  // 16-byte offsets
    if (!workspace || !aligned16(workspace)) return NV_ERR_WORKSPACE;
    const nvq::MoeWorkspace w = nvq::moe_carve(workspace, R, E, I, K);
    if (workspace_bytes < w.bytes) return NV_ERR_WORKSPACE;
    if (T == 0) return NV_OK;
    if (!x || !ids || !rw || !y || !gate_codes || !gate_scales || !gate_biases || !up_codes ||
        !up_scales || !up_biases || !down_codes || !down_scales || !down_biases)
        return NV_ERR_INVALID_ARG;
    for (const void* p : {x, static_cast<const void*>(ids), static_cast<const void*>(rw),
                          static_cast<const void*>(y), static_cast<const void*>(gate_codes),
                          gate_scales, gate_biases, static_cast<const void*>(up_codes), up_scales,
                          up_biases, static_cast<const void*>(down_codes), down_scales,
                          down_biases})
        if (!aligned16(p)) return NV_ERR_INVALID_ARG;

    cudaStream_t s = stream;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((R + 255) / 256 < 4 * sms ? (R + 255) / 256 : 4 * sms), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, nvq::pair_tokens_kernel, w.lhs, R, topk);
    if (e != cudaSuccess) return NV_ERR_CUDA;
    const nvq::GatherWorkspace rt = nvq::gather_workspace_carve(w.route, R, E);
    e = nvq::launch_gather_route(w.lhs, ids, R, E, T, 0, rt, s, false);
    if (e != cudaSuccess) return NV_ERR_CUDA;
    // gate, then up with silu(gate) * up over the gate values, then down
    e = nvq::launch_tc_gather(x, T, K, w.lhs, rt.perm, rt.offsets, E, I, gate_codes, gate_scales,
                              gate_biases, group_size, bits, w.gh, s, sms);
    if (e != cudaSuccess) return NV_ERR_CUDA;
    e = nvq::launch_tc_gather(x, T, K, w.lhs, rt.perm, rt.offsets, E, I, up_codes, up_scales,
                              up_biases, group_size, bits, w.gh, s, sms, w.gh);
    if (e != cudaSuccess) return NV_ERR_CUDA;
    e = nvq::launch_tc_gather(w.gh, R, I, nullptr, rt.perm, rt.offsets, E, K, down_codes,
                              down_scales, down_biases, group_size, bits, w.d, s, sms);
    if (e != cudaSuccess) return NV_ERR_CUDA;
    const int64_t items = T * (K / 8);
    const int64_t blocks = (items + 255) / 256 < 8 * sms ? (items + 255) / 256 : 8 * sms;
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    e = cudaLaunchKernelEx(&cfg, nvq::combine_kernel, static_cast<const uint16_t*>(w.d), rw, T, K, topk,
                           static_cast<uint16_t*>(y));
    return e == cudaSuccess ? NV_OK : NV_ERR_CUDA;
}

}  // extern "C"
