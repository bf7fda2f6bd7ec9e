// The C ABI (include/nvq.h): argument checks on the host, then a pure routing
// decision (a function of shapes, dtype, group size, bits, layout and
// row_exact only, nuvec crate docs, "Determinism": "Routing is pure") and the
// launches. Nothing here allocates device memory or synchronises a stream,
// except nv_gather_qmm_flags, whose job is to read a result back.
#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Widths the quantizer and dequantizer take: 1, 2, 4, 8 (they divide 32).
nv_status check_codes(int gs, int bits) {
    if (bits == 3 || bits == 5 || bits == 6) return NV_ERR_UNSUPPORTED;
    if (bits != 1 && bits != 2 && bits != 4 && bits != 8) return NV_ERR_INVALID_ARG;
    if (gs != 32 && gs != 64 && gs != 128) return NV_ERR_INVALID_ARG;
    return NV_OK;
}

// Widths the products take: 2, 4, 8 (1-bit codes have no product kernels).
nv_status check_quant(int gs, int bits) {
    if (bits == 1) return NV_ERR_UNSUPPORTED;
    return check_codes(gs, bits);
}

bool valid_dtype(nv_dtype dt) { return dt == NV_F32 || dt == NV_BF16; }

// The last CUDA error a call of this thread returned as NV_ERR_CUDA
// (diagnostics for nv_last_cuda_error).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

nv_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return NV_OK;
    t_last_cuda_error = e;
    return NV_ERR_CUDA;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

}  // namespace

extern "C" {

const char* nv_status_string(nv_status s) {
    switch (s) {
        case NV_OK: return "NV_OK: success";
        case NV_ERR_INVALID_ARG: return "NV_ERR_INVALID_ARG: a shape, pointer or alignment is invalid";
        case NV_ERR_UNSUPPORTED: return "NV_ERR_UNSUPPORTED: valid combination not implemented (bit width or dtype)";
        case NV_ERR_WORKSPACE: return "NV_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case NV_ERR_CUDA: return "NV_ERR_CUDA: a CUDA launch or call failed";
    }
    return "unknown nv_status";
}

nv_status nv_quantize_affine(const void* w, nv_dtype dt, int64_t rows, int64_t cols,
                             int group_size, int bits, uint32_t* codes, void* scales,
                             void* biases, nv_stream_t stream) {
    if (!valid_dtype(dt)) return NV_ERR_UNSUPPORTED;
    nv_status st = check_codes(group_size, bits);
    if (st != NV_OK) return st;
    if (rows < 0 || cols <= 0 || cols % group_size != 0) return NV_ERR_INVALID_ARG;
    if (rows == 0) return NV_OK;
    if (!w || !codes || !scales || !biases) return NV_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases))
        return NV_ERR_INVALID_ARG;
    return from_cuda(nvq::launch_quantize_affine(w, dt, rows, cols, group_size, bits, codes,
                                                 scales, biases, stream, sm_count()));
}

nv_status nv_dequantize_affine(const uint32_t* codes, const void* scales, const void* biases,
                               nv_dtype dt, int64_t rows, int64_t cols, int group_size,
                               int bits, void* w, nv_stream_t stream) {
    if (!valid_dtype(dt)) return NV_ERR_UNSUPPORTED;
    nv_status st = check_codes(group_size, bits);
    if (st != NV_OK) return st;
    if (rows < 0 || cols <= 0 || cols % group_size != 0) return NV_ERR_INVALID_ARG;
    if (rows == 0) return NV_OK;
    if (!w || !codes || !scales || !biases) return NV_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases))
        return NV_ERR_INVALID_ARG;
    return from_cuda(nvq::launch_dequantize_affine(codes, scales, biases, dt, rows, cols,
                                                   group_size, bits, w, stream, sm_count()));
}

nv_status nv_qmm(const void* x, nv_dtype dt, int64_t M, int64_t K, int64_t N,
                 const uint32_t* codes, const void* scales, const void* biases, int group_size,
                 int bits, int transpose, int row_exact, void* y, nv_stream_t stream) {
    if (!valid_dtype(dt)) return NV_ERR_UNSUPPORTED;
    nv_status st = check_quant(group_size, bits);
    if (st != NV_OK) return st;
    if (M < 0 || K <= 0 || N < 0) return NV_ERR_INVALID_ARG;
    if ((transpose ? K : N) % group_size != 0) return NV_ERR_INVALID_ARG;
    if (row_exact && M > NV_ROW_INDEPENDENT_ROWS) return NV_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return NV_OK;
    if (!x || !codes || !scales || !biases || !y) return NV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases) ||
        !aligned16(y))
        return NV_ERR_INVALID_ARG;

    cudaStream_t s = stream;
    const int sms = sm_count();
    if (dt == NV_BF16) {
        if (transpose) {
            if (M <= NV_ROW_INDEPENDENT_ROWS && nvq::qmv_supported(bits, group_size))
                return from_cuda(nvq::launch_qmv(x, M, K, N, codes, scales, biases, group_size,
                                                 bits, y, s, sms));
            if (M > NV_ROW_INDEPENDENT_ROWS && nvq::tc_supported(M, K, N, bits, group_size))
                return from_cuda(nvq::launch_tc_qmm(x, M, K, N, codes, scales, biases,
                                                    group_size, bits, y, s, sms));
        } else {
            if (M <= NV_ROW_INDEPENDENT_ROWS && nvq::qmvt_supported_m(bits, group_size, 1)) {
                // Rows go through in chunks the kernel holds in registers; every
                // row's arithmetic is the same in any chunk, so the chunking keeps
                // each row's bits equal to its one-row product.
                int64_t chunk = M;
                while (chunk > 1 && !nvq::qmvt_supported_m(bits, group_size, chunk)) --chunk;
                for (int64_t m0 = 0; m0 < M; m0 += chunk) {
                    const int64_t mc = M - m0 < chunk ? M - m0 : chunk;
                    cudaError_t e = nvq::launch_qmvt(
                        static_cast<const uint16_t*>(x) + m0 * K, mc, K, N, codes, scales, biases,
                        group_size, bits, static_cast<uint16_t*>(y) + m0 * N, s, sms);
                    if (e != cudaSuccess) return from_cuda(e);
                }
                return NV_OK;
            }
            if (M > NV_ROW_INDEPENDENT_ROWS && nvq::tc_supported_t0(M, K, N, bits, group_size))
                return from_cuda(nvq::launch_tc_qmm(x, M, K, N, codes, scales, biases, group_size,
                                                    bits, y, s, sms, 0, 0));
        }
    }
    return from_cuda(nvq::launch_qmm_simt(x, dt, M, K, N, codes, scales, biases, group_size, bits,
                                          transpose, y, s));
}

nv_status nv_qmm_batched(const void* x, nv_dtype dt, int64_t B, int64_t L, int64_t K, int64_t N,
                         const uint32_t* codes, const void* scales, const void* biases,
                         int group_size, int bits, int transpose, void* y, nv_stream_t stream) {
    if (!valid_dtype(dt)) return NV_ERR_UNSUPPORTED;
    nv_status st = check_quant(group_size, bits);
    if (st != NV_OK) return st;
    if (B < 0 || L < 0 || K <= 0 || N < 0) return NV_ERR_INVALID_ARG;
    if ((transpose ? K : N) % group_size != 0) return NV_ERR_INVALID_ARG;
    if (L > 0 && B > (int64_t(1) << 40) / L) return NV_ERR_INVALID_ARG;
    const int64_t M = B * L;
    if (M == 0 || N == 0) return NV_OK;
    if (!x || !codes || !scales || !biases || !y) return NV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases) ||
        !aligned16(y))
        return NV_ERR_INVALID_ARG;
    // Routing by one item's rows L (crate docs, "Determinism": batch items of
    // quantized products get their solo bits, the split-K partitions counted
    // per item). Every route below computes each row with the same operations
    // as the item's own call, whatever the batch around it.
    cudaStream_t s = stream;
    const int sms = sm_count();
    if (dt == NV_BF16) {
        if (transpose) {
            if (L <= NV_ROW_INDEPENDENT_ROWS && nvq::qmv_supported(bits, group_size)) {
                for (int64_t m0 = 0; m0 < M; m0 += NV_ROW_INDEPENDENT_ROWS) {
                    const int64_t mc = M - m0 < NV_ROW_INDEPENDENT_ROWS ? M - m0 : NV_ROW_INDEPENDENT_ROWS;
                    cudaError_t e = nvq::launch_qmv(static_cast<const uint16_t*>(x) + m0 * K, mc, K, N,
                                                    codes, scales, biases, group_size, bits,
                                                    static_cast<uint16_t*>(y) + m0 * N, s, sms);
                    if (e != cudaSuccess) return from_cuda(e);
                }
                return NV_OK;
            }
            if (L > NV_ROW_INDEPENDENT_ROWS && nvq::tc_supported(M, K, N, bits, group_size))
                return from_cuda(nvq::launch_tc_qmm(x, M, K, N, codes, scales, biases, group_size,
                                                    bits, y, s, sms, L));
        } else if (L > NV_ROW_INDEPENDENT_ROWS && nvq::tc_supported_t0(M, K, N, bits, group_size)) {
            return from_cuda(nvq::launch_tc_qmm(x, M, K, N, codes, scales, biases, group_size, bits,
                                                y, s, sms, L, 0));
        } else if (L <= NV_ROW_INDEPENDENT_ROWS && nvq::qmvt_supported_m(bits, group_size, 1)) {
            int64_t chunk = NV_ROW_INDEPENDENT_ROWS;
            while (chunk > 1 && !nvq::qmvt_supported_m(bits, group_size, chunk)) --chunk;
            for (int64_t m0 = 0; m0 < M; m0 += chunk) {
                const int64_t mc = M - m0 < chunk ? M - m0 : chunk;
                cudaError_t e = nvq::launch_qmvt(static_cast<const uint16_t*>(x) + m0 * K, mc, K, N,
                                                 codes, scales, biases, group_size, bits,
                                                 static_cast<uint16_t*>(y) + m0 * N, s, sms);
                if (e != cudaSuccess) return from_cuda(e);
            }
            return NV_OK;
        }
    }
    return from_cuda(nvq::launch_qmm_simt(x, dt, M, K, N, codes, scales, biases, group_size, bits,
                                          transpose, y, s));
}

int nv_qmm_splits(int64_t M, int64_t K, int64_t N, int bits, int group_size, int transpose,
                  nv_dtype dt) {
    if (dt != NV_BF16 || M <= NV_ROW_INDEPENDENT_ROWS) return 1;
    if (transpose ? !nvq::tc_supported(M, K, N, bits, group_size)
                  : !nvq::tc_supported_t0(M, K, N, bits, group_size))
        return 1;
    return nvq::tc_splits(M, K, N, sm_count(), bits, transpose);
}

size_t nv_gather_qmm_workspace_size(int64_t R, int64_t E) {
    if (R < 0 || E < 0) return 0;
    return nvq::gather_workspace_bytes(R, E);
}

nv_status nv_gather_qmm(const void* x, nv_dtype dt, int64_t x_rows, int64_t K,
                        const uint32_t* lhs_idx, const uint32_t* rhs_idx, int64_t R, int64_t E,
                        int64_t N, const uint32_t* codes, const void* scales, const void* biases,
                        int group_size, int bits, int transpose, int sorted, int row_exact,
                        void* workspace, size_t workspace_bytes, void* y, nv_stream_t stream) {
    if (!valid_dtype(dt)) return NV_ERR_UNSUPPORTED;
    nv_status st = check_quant(group_size, bits);
    if (st != NV_OK) return st;
    if (x_rows < 0 || K <= 0 || R < 0 || E <= 0 || N < 0) return NV_ERR_INVALID_ARG;
    if ((transpose ? K : N) % group_size != 0) return NV_ERR_INVALID_ARG;
    if (R > (int64_t(1) << 31) - 1) return NV_ERR_INVALID_ARG;
    if (E > nvq::kMaxExperts) return NV_ERR_UNSUPPORTED;
    if (!workspace || !aligned16(workspace)) return NV_ERR_WORKSPACE;
    if (workspace_bytes < nvq::gather_workspace_bytes(R, E)) return NV_ERR_WORKSPACE;
    if (R == 0) return NV_OK;
    if (!x || !rhs_idx || !codes || !scales || !biases || !y) return NV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases) ||
        !aligned16(y) || !aligned16(rhs_idx) || (lhs_idx && !aligned16(lhs_idx)))
        return NV_ERR_INVALID_ARG;

    cudaStream_t s = stream;
    const int sms = sm_count();
    // Tensor-core routes: each expert's weights are read once for all its rows
    // (the kernels keep 32-bit offsets into x in 16-byte units).
    const bool tc = dt == NV_BF16 && !row_exact && x_rows * K < (int64_t(1) << 35) &&
                    (transpose ? nvq::tc_gather_supported(K, N, bits, group_size)
                               : nvq::tc_gather_t0_supported(K, N, bits, group_size));
    // Matrix-vector route (row_exact): every pair's output is bitwise equal to
    // nv_qmm(M = 1) of that row with its expert's weights.
    const bool mv = !tc && dt == NV_BF16 && transpose && nvq::qmv_supported(bits, group_size);
    nvq::GatherWorkspace ws = nvq::gather_workspace_carve(workspace, R, E);
    cudaError_t e = nvq::launch_gather_route(lhs_idx, rhs_idx, R, E, x_rows, sorted, ws, s, mv);
    if (e != cudaSuccess) return from_cuda(e);
    if (N == 0) return NV_OK;
    if (tc && transpose)
        return from_cuda(nvq::launch_tc_gather(x, x_rows, K, lhs_idx, ws.perm, ws.offsets, E, N,
                                               codes, scales, biases, group_size, bits, y, s, sms));
    if (tc)
        return from_cuda(nvq::launch_tc_gather_t0(x, x_rows, K, lhs_idx, ws.perm, ws.offsets, E, N,
                                                  codes, scales, biases, group_size, bits, y, s, sms));
    if (mv)
        return from_cuda(nvq::launch_qmv_gather(x, K, N, codes, scales, biases, group_size, bits,
                                                lhs_idx, ws.perm, ws.problems, ws.num_problems,
                                                ws.max_problems, E, y, s, sms));
    return from_cuda(nvq::launch_gather_simt(x, dt, x_rows, K, lhs_idx, rhs_idx, R, E, N, codes,
                                             scales, biases, group_size, bits, transpose, y, s));
}

nv_status nv_gather_mm(const void* x, nv_dtype dt, int64_t x_rows, int64_t K,
                       const uint32_t* lhs_idx, const uint32_t* rhs_idx, int64_t R, int64_t E,
                       int64_t N, const void* w, int sorted, void* workspace,
                       size_t workspace_bytes, void* y, nv_stream_t stream) {
    if (!valid_dtype(dt)) return NV_ERR_UNSUPPORTED;
    if (x_rows < 0 || K <= 0 || R < 0 || E <= 0 || N < 0) return NV_ERR_INVALID_ARG;
    if (R > (int64_t(1) << 31) - 1) return NV_ERR_INVALID_ARG;
    if (E > nvq::kMaxExperts) return NV_ERR_UNSUPPORTED;
    if (dt != NV_BF16 || !nvq::tc_gather_mm_supported(K, N > 0 ? N : 1)) return NV_ERR_UNSUPPORTED;
    if (x_rows * K >= (int64_t(1) << 35)) return NV_ERR_UNSUPPORTED;  // 32-bit 16-byte offsets into x
    if (!workspace || !aligned16(workspace)) return NV_ERR_WORKSPACE;
    if (workspace_bytes < nvq::gather_workspace_bytes(R, E)) return NV_ERR_WORKSPACE;
    if (R == 0) return NV_OK;
    if (!x || !rhs_idx || !w || !y) return NV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(y) || !aligned16(rhs_idx) ||
        (lhs_idx && !aligned16(lhs_idx)))
        return NV_ERR_INVALID_ARG;
    cudaStream_t s = stream;
    nvq::GatherWorkspace ws = nvq::gather_workspace_carve(workspace, R, E);
    cudaError_t e = nvq::launch_gather_route(lhs_idx, rhs_idx, R, E, x_rows, sorted, ws, s, false);
    if (e != cudaSuccess) return from_cuda(e);
    if (N == 0) return NV_OK;
    return from_cuda(nvq::launch_tc_gather_mm(x, x_rows, K, lhs_idx, ws.perm, ws.offsets, E, N, w,
                                              y, s, sm_count()));
}

nv_status nv_gather_qmm_flags(const void* workspace, uint32_t* host_flags, nv_stream_t stream) {
    if (!workspace || !aligned16(workspace) || !host_flags) return NV_ERR_INVALID_ARG;
    cudaStream_t s = stream;
    if (cudaMemcpyAsync(host_flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return NV_ERR_CUDA;
    return from_cuda(cudaStreamSynchronize(s));
}

const char* nv_last_cuda_error(void) {
    return cudaGetErrorName(t_last_cuda_error);
}

nv_status nv_pipeline_error(uint32_t* host_code) {
    if (!host_code) return NV_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return NV_ERR_CUDA;
    const unsigned int a = nvq::qmv_error_take();
    const unsigned int b = nvq::tc_error_take();
    const unsigned int c = nvq::tc_gather_error_take();
    const unsigned int d = nvq::tc_gather_mm_error_take();
    const unsigned int g = nvq::tc_gather_t0_error_take();
    const unsigned int t = nvq::selftest_error_take();
    if (a == 0xFFFFFFFFu || b == 0xFFFFFFFFu || c == 0xFFFFFFFFu || d == 0xFFFFFFFFu ||
        g == 0xFFFFFFFFu || t == 0xFFFFFFFFu)
        return NV_ERR_CUDA;
    *host_code = a ? a : b ? b : c ? c : d ? d : g ? g : t;
    return NV_OK;
}

nv_status nv_pipeline_selftest(uint32_t limit_us, nv_stream_t stream) {
    if (limit_us == 0 || limit_us > 2000000u) return NV_ERR_INVALID_ARG;
    return from_cuda(nvq::launch_pipeline_selftest(static_cast<uint64_t>(limit_us) * 1000u, stream));
}

}  // extern "C"
