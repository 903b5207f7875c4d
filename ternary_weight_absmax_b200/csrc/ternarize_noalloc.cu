// ternarize_noalloc.cu -- an allocation-free variant of the device absmean
// ternariser.
//
// bitnet_ternarize_absmean_device needs a small device workspace for its
// per-tensor reduction, and expects the caller to provide it.  Some callers
// cannot provide one: a host that has already handed out all device memory
// through its own fixed pool and forbids further allocation, a foreign-language
// binding with no device allocator at all, or a latency-sensitive loop that
// must not call cudaMalloc (which may synchronise the whole device and stall
// other work).  For them this file keeps the scratch in a file-scope device
// array instead, sized for the largest workspace the ternariser can ever ask
// for (2048 fp64 partial sums plus one 256-byte slot for gamma).
//
// The array is a device symbol: every GPU that loads the library holds one
// copy until the process exits.  Host code cannot use the symbol's name as a
// device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it.
#include <mutex>

#include "common.cuh"

namespace bitnet {
namespace {

constexpr size_t kNoAllocPartials = 2048;  // upper bound of absmean_num_partials()
constexpr size_t kNoAllocScratchBytes = kNoAllocPartials * sizeof(double) + 256;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64];

// Device address of this device's scratch array (looked up once per device).
cudaError_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace bitnet

extern "C" bitnet_status bitnet_ternarize_absmean_device_noalloc(const float *w_dev, int64_t rows, int64_t cols,
                                                                 int mode, uint8_t *codes_out_dev,
                                                                 float *scales_out_dev, bitnet_stream_t stream) {
    using namespace bitnet;
    const size_t need = bitnet_ternarize_workspace_bytes(rows, cols);
    if (need == 0)  // invalid shape: the regular entry point reports it, without touching the GPU
        return bitnet_ternarize_absmean_device(w_dev, rows, cols, mode, codes_out_dev, scales_out_dev, nullptr, 0,
                                               stream);
    if (need > kNoAllocScratchBytes)
        return set_error_detail(BITNET_ERR_BUFSIZE, "needs %zu bytes of scratch; the static array holds %zu", need,
                                kNoAllocScratchBytes);
    void *scratch = nullptr;
    const cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess)
        return set_error_detail(BITNET_ERR_CUDA, "cudaGetSymbolAddress of the scratch array: %s",
                                cudaGetErrorString(e));
    // No part of the scratch has to start at zero: the reduction writes every
    // partial it later reads, and gamma, within this same call.
    return bitnet_ternarize_absmean_device(w_dev, rows, cols, mode, codes_out_dev, scales_out_dev, scratch,
                                           kNoAllocScratchBytes, stream);
}
