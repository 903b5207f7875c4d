// quant_act.cu -- per-token absmax int8 activation quantisation.
//
// The pages make the activations of the W2A8 layer 8-bit with a scale
// derived from them ("5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构对决",
// section "GPU内核突破"; "浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍
// 提速实操", section "查表（LUT）内核") without printing the formula; the
// library uses s = 127 / max(absmax, 1e-5) and q = rint(x * s), ties to even.
//
// One CTA per token row.  Pass 1 reads the row as float4 and reduces |x| with
// warp shuffles then shared memory; pass 2 re-reads the row (now L1/L2
// resident), multiplies by s in fp32, rounds half to even and stores four
// int8 per thread per step.  Each warp step covers 32 float4 = one 128-wide
// block, so the optional per-block sums of q are one warp reduction each.
// Bound: HBM for prefill-sized T (4 B read + 1 B written per element), launch
// latency for decode.  Launched with programmatic dependent launch so the
// next kernel (the GEMV) can start streaming its weights meanwhile.
#include <atomic>

#include "common.cuh"

namespace bitnet {
namespace {

constexpr int kThreads = 256;  // 8 warps
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ int quant_one(float x, float s) {
    float p = __fmul_rn(x, s);          // single fp32 multiply, never fused
    int v = __float2int_rn(p);          // round half to even
    v = v > 127 ? 127 : v;
    v = v < -127 ? -127 : v;
    return v;
}

template <bool kBlockSum>
__global__ void __launch_bounds__(kThreads)
quant_act_kernel(const float4 *__restrict__ x, int64_t K, int8_t *__restrict__ q,
                 float *__restrict__ s, int32_t *__restrict__ blocksum) {
    // x may be produced by the kernel just before on the stream: wait for it
    // (a no-op without programmatic dependent launch), then let the next
    // kernel launch so it can prefetch its weights while this one runs.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t row = blockIdx.x;
    const int64_t n4 = K / 4;
    const float4 *xr = x + row * n4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    float m = 0.0f;
    for (int64_t i = tid; i < n4; i += kThreads) {
        float4 v = __ldg(xr + i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[kWarps];
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; w++) m = fmaxf(m, red[w]);

    const float scale = __fdiv_rn(127.0f, m > kEps ? m : kEps);  // IEEE fp32 divide
    if (tid == 0) s[row] = scale;

    uint32_t *qr = reinterpret_cast<uint32_t *>(q + row * K);
    const int64_t nb = K / 128;
    // Step it covers float4 [it*256, it*256+256); warp w of it covers block it*8 + w.
    for (int64_t base = 0; base < n4; base += kThreads) {
        int64_t i = base + tid;
        int sum = 0;
        if (i < n4) {
            float4 v = __ldg(xr + i);
            int a = quant_one(v.x, scale), b = quant_one(v.y, scale);
            int c = quant_one(v.z, scale), d = quant_one(v.w, scale);
            qr[i] = (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) |
                    ((uint32_t)(c & 0xff) << 16) | ((uint32_t)(d & 0xff) << 24);
            sum = a + b + c + d;
        }
        if (kBlockSum) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            int64_t blk = (base >> 5) + warp;
            if (lane == 0 && blk < nb) blocksum[row * nb + blk] = sum;
        }
    }
}

}  // namespace

cudaError_t launch_quant_act(const float *x, int64_t T, int64_t K, int8_t *q, float *s,
                             int32_t *blocksum, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    static std::atomic<bool> configured[64];  // set once per device; a repeat is harmless
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        // Same shared-memory carveout as the decode kernel, so the two can share
        // an SM under programmatic dependent launch without a reconfiguration.
        for (auto k : {quant_act_kernel<true>, quant_act_kernel<false>}) {
            e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
        }
        configured[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)T);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float4 *x4 = reinterpret_cast<const float4 *>(x);
    if (blocksum) return cudaLaunchKernelEx(&cfg, quant_act_kernel<true>, x4, K, q, s, blocksum);
    return cudaLaunchKernelEx(&cfg, quant_act_kernel<false>, x4, K, q, s, (int32_t *)nullptr);
}

}  // namespace bitnet
