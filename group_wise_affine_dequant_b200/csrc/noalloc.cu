// nv_gather_qmm_noalloc: the mixture-of-experts product for callers that
// cannot allocate device memory, e.g. code that runs inside another runtime's
// pre-planned memory arena (an inference server that forbids allocation on the
// decode path), plugin hosts that hand out no allocator, or real-time loops
// where a cudaMalloc could block or fragment. nv_gather_qmm needs a caller-
// provided workspace for its routing tables; this entry point keeps those
// tables in one fixed array compiled into the library instead.
//
// The array is a file-scope __device__ object of kNoAllocScratchBytes, so every
// GPU that loads the library holds it until the process exits. Host code
// cannot pass the symbol itself to a kernel (on the host it names a stand-in,
// not a device address), so its device address is looked up once per device
// with cudaGetSymbolAddress, with that device current, on the first call made
// on the device; that first call should therefore come before any stream
// capture. The looked-up address is kept for the life of the process: after
// a cudaDeviceReset it would be stale, so a device this entry point has used
// must not be reset. All calls share the array: calls that overlap on the GPU
// (two streams, or two devices' worth of host threads on one device) race on
// it. Nothing in it needs to start at zero: the routing kernel writes every
// entry a call reads. Each call leaves its routing tables (and its anomaly
// flags, which no entry point reads back from here) behind, overwritten by
// the next call.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

// Capacity: up to 32768 (row, expert) pairs and 256 experts.
constexpr int64_t kNoAllocMaxPairs = 32768;
constexpr int64_t kNoAllocMaxExperts = 256;
constexpr size_t kNoAllocScratchBytes = 16 + 16 * ((kNoAllocMaxExperts + 2) * 4 / 16 + 1) +
                                        kNoAllocMaxPairs * 4 +
                                        ((kNoAllocMaxPairs + 7) / 8 + kNoAllocMaxExperts + 1) * 16;

}  // namespace

// One copy per device; internal to this file.
static __device__ __align__(256) unsigned char g_gather_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gather_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" nv_status nv_gather_qmm_noalloc(const void* x, nv_dtype dt, int64_t x_rows, int64_t K,
                                           const uint32_t* lhs_idx, const uint32_t* rhs_idx,
                                           int64_t R, int64_t E, int64_t N, const uint32_t* codes,
                                           const void* scales, const void* biases,
                                           int group_size, int bits, int transpose, int sorted,
                                           int row_exact, void* y, nv_stream_t stream) {
    if (R > kNoAllocMaxPairs || E > kNoAllocMaxExperts) return NV_ERR_WORKSPACE;
    if (nv_gather_qmm_workspace_size(R, E) > kNoAllocScratchBytes) return NV_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return NV_ERR_CUDA;
    return nv_gather_qmm(x, dt, x_rows, K, lhs_idx, rhs_idx, R, E, N, codes, scales, biases,
                         group_size, bits, transpose, sorted, row_exact, scratch,
                         kNoAllocScratchBytes, y, stream);
}
