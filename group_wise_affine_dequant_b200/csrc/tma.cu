// Host-side helpers of the TMA pipelines and the device error word, and the
// self-test of the bounded waits.
#include "kernels.cuh"
#include "tma.cuh"

namespace nvq {

EncodeTiled tensor_map_encoder() {
    static EncodeTiled fn = []() -> EncodeTiled {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiled>(p);
    }();
    return fn;
}

namespace {

// One thread waits, through the same bounded wait the pipelines use, on an
// mbarrier that nothing ever completes: the wait gives up after limit_ns,
// records `code` in this file's error word and the kernel returns.
__global__ void pipeline_selftest_kernel(uint64_t limit_ns, unsigned code) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
        mbar_wait(&bar, 0, code, limit_ns);
    }
}

}  // namespace

cudaError_t launch_pipeline_selftest(uint64_t limit_ns, cudaStream_t stream) {
    pipeline_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, kSelftestWaitCode);
    return cudaGetLastError();
}

unsigned int selftest_error_take() { return pipeline_error_take(); }

}  // namespace nvq
