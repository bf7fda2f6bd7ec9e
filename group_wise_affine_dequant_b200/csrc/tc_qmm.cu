#include "tc.cuh"

namespace nvq {

bool tc_supported(int64_t, int64_t, int64_t, int, int) { return false; }

cudaError_t launch_tc_qmm(const void*, int64_t, int64_t, int64_t, const uint32_t*, const void*,
                          const void*, int, int, void*, cudaStream_t, int) {
    return cudaErrorNotSupported;
}

}  // namespace nvq
