// gemm.cu -- placeholder until the tcgen05 prefill GEMM lands.
#include "common.cuh"
namespace bitnet {
cudaError_t launch_gemm(const void *, int64_t, int64_t, bool, const int8_t *, const float *, int64_t,
                        float *, int32_t *, const DeviceGlobals &, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace bitnet
