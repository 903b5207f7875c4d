// quant_act.cu -- per-token absmax int8 activation quantisation.
//
// The pages make the activations of the W2A8 layer 8-bit with a scale
// derived from them ("5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构对决",
// section "GPU内核突破"; "浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍
// 提速实操", section "查表（LUT）内核") without printing the formula; the
// library uses s = 127 / max(absmax, 1e-5) and q = rint(x * s), ties to even.
//
// One CTA per token row, sized to the row: thread i holds float4 elements i,
// i + threads, ... (up to NPER of them) in registers, so x is read from HBM
// exactly once; |x| is reduced with warp shuffles then shared memory, and the
// row is quantised from the registers (one fp32 multiply, round half to
// even) into four int8 per float4.  The elements of a 128-wide block are 32
// float4 held by one warp at one register index, so the optional per-block
// sums of q are one warp reduction each.  Bound: HBM at prefill sizes (4 B
// read + 1 B written per element), launch latency at decode.  Launched with
// programmatic dependent launch so the next kernel (the GEMV or GEMM) can
// start fetching its weights meanwhile.
#include <atomic>

#include "common.cuh"
#include "expand.cuh"

namespace bitnet {
namespace {

constexpr int kMaxThreads = 512;

__device__ __forceinline__ int quant_one(float x, float s) {
    float p = __fmul_rn(x, s);          // single fp32 multiply, never fused
    int v = __float2int_rn(p);          // round half to even
    v = v > 127 ? 127 : v;
    v = v < -127 ? -127 : v;
    return v;
}

// Row `row` of x by the whole CTA (red: kMaxThreads / 32 floats of shared memory).
template <int NPER, bool kBlockSum>
__device__ __forceinline__ void quant_row(const float4 *__restrict__ x, int64_t K, int8_t *__restrict__ q,
                                          float *__restrict__ s, int32_t *__restrict__ blocksum, int64_t row,
                                          float *red) {
    const int n4 = (int)(K / 4);
    const float4 *xr = x + row * n4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;

    float4 v[NPER];
    float m = 0.0f;
#pragma unroll
    for (int u = 0; u < NPER; u++) {
        const int i = u * nt + tid;
        v[u] = i < n4 ? __ldg(xr + i) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
    for (int w = 1; w < (nt >> 5); w++) m = fmaxf(m, red[w]);

    const float scale = __fdiv_rn(127.0f, m > kEps ? m : kEps);  // IEEE fp32 divide
    if (tid == 0) s[row] = scale;

    uint32_t *qr = reinterpret_cast<uint32_t *>(q + row * K);
#pragma unroll
    for (int u = 0; u < NPER; u++) {
        const int i = u * nt + tid;
        int sum = 0;
        if (i < n4) {
            const int a = quant_one(v[u].x, scale), b = quant_one(v[u].y, scale);
            const int c = quant_one(v[u].z, scale), d = quant_one(v[u].w, scale);
            qr[i] = (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
                    ((uint32_t)(d & 0xff) << 24);
            sum = a + b + c + d;
        }
        if (kBlockSum) {
            // float4 elements u*nt + 32*warp .. +31 form block (u*nt)/32 + warp
            // (nt is a multiple of 32).
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const int blk = (u * nt >> 5) + warp;
            if (lane == 0 && blk * 32 < n4) blocksum[row * (K / 128) + blk] = sum;
        }
    }
}

template <int NPER, bool kBlockSum>
__global__ void __launch_bounds__(kMaxThreads)
quant_act_kernel(const float4 *__restrict__ x, int64_t K, int8_t *__restrict__ q,
                 float *__restrict__ s, int32_t *__restrict__ blocksum) {
    // x may be produced by the kernel just before on the stream: wait for it
    // (a no-op without programmatic dependent launch), then let the next
    // kernel launch so it can prefetch its weights while this one runs.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ float red[kMaxThreads / 32];
    quant_row<NPER, kBlockSum>(x, K, q, s, blocksum, blockIdx.x, red);
}

// The prefill linear's pre-pass: CTAs 0 .. T-1 quantise the token rows (as
// quant_act_kernel), the others expand the weights to int8 for the GEMM, one
// warp per 512-byte code tile (expand.cuh), so the two run side by side.
// Both write only after griddepcontrol.wait (x may come from the previous
// kernel, which may also still read the workspace); the code words are read
// before it.
template <int NPER>
__global__ void __launch_bounds__(kMaxThreads)
prefill_prep_kernel(const float4 *__restrict__ x, int64_t K, int8_t *__restrict__ q, float *__restrict__ s,
                    int64_t T, const uint4 *__restrict__ tiles, int8_t *__restrict__ wout, int64_t ntiles,
                    int nb) {
    __shared__ float red[kMaxThreads / 32];
    __shared__ uint4 stage[kMaxThreads / 32][32];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if ((int64_t)blockIdx.x < T) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        quant_row<NPER, false>(x, K, q, s, nullptr, blockIdx.x, red);
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tj = ((int64_t)blockIdx.x - T) * (blockDim.x >> 5) + warp;  // tile tr * nb + j
    const bool has = tj < ntiles;
    const uint4 v = has ? __ldcs(tiles + tj * 32 + lane) : make_uint4(0, 0, 0, 0);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (has) expand_tile(v, stage[warp], wout, tj, nb, K);
}

// Rows longer than 16 float4 per thread of 512 threads (K > 32768): two
// passes over the row (the second hits L1 / L2).
template <bool kBlockSum>
__global__ void __launch_bounds__(kMaxThreads)
quant_act_long_kernel(const float4 *__restrict__ x, int64_t K, int8_t *__restrict__ q,
                      float *__restrict__ s, int32_t *__restrict__ blocksum) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t row = blockIdx.x;
    const int64_t n4 = K / 4;
    const float4 *xr = x + row * n4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ float red[kMaxThreads / 32];
    float m = 0.0f;
    for (int64_t i = tid; i < n4; i += kMaxThreads) {
        const float4 v = __ldg(xr + i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
    for (int w = 1; w < kMaxThreads / 32; w++) m = fmaxf(m, red[w]);
    const float scale = __fdiv_rn(127.0f, m > kEps ? m : kEps);
    if (tid == 0) s[row] = scale;
    uint32_t *qr = reinterpret_cast<uint32_t *>(q + row * K);
    for (int64_t base = 0; base < n4; base += kMaxThreads) {
        const int64_t i = base + tid;
        int sum = 0;
        if (i < n4) {
            const float4 v = __ldg(xr + i);
            const int a = quant_one(v.x, scale), b = quant_one(v.y, scale);
            const int c = quant_one(v.z, scale), d = quant_one(v.w, scale);
            qr[i] = (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
                    ((uint32_t)(d & 0xff) << 24);
            sum = a + b + c + d;
        }
        if (kBlockSum) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const int64_t blk = (base >> 5) + warp;
            if (lane == 0 && blk * 32 < n4) blocksum[row * (K / 128) + blk] = sum;
        }
    }
}

template <int NPER>
cudaError_t launch_one(const cudaLaunchConfig_t &cfg, const float4 *x4, int64_t K, int8_t *q, float *s,
                       int32_t *blocksum) {
    if (blocksum) return cudaLaunchKernelEx(&cfg, quant_act_kernel<NPER, true>, x4, K, q, s, blocksum);
    return cudaLaunchKernelEx(&cfg, quant_act_kernel<NPER, false>, x4, K, q, s, (int32_t *)nullptr);
}

template <int NPER>
cudaError_t launch_prep(const cudaLaunchConfig_t &cfg, const float4 *x4, int64_t K, int8_t *q, float *s, int64_t T,
                        const uint4 *tiles, int8_t *wout, int64_t ntiles, int nb) {
    return cudaLaunchKernelEx(&cfg, prefill_prep_kernel<NPER>, x4, K, q, s, T, tiles, wout, ntiles, nb);
}

}  // namespace

bool prefill_prep_supported(int64_t K) { return K / 4 <= 16 * (int64_t)kMaxThreads; }

cudaError_t launch_prefill_prep(const float *x, int64_t T, int64_t K, int8_t *q, float *s, const void *data,
                                int64_t rows, int8_t *expanded, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int64_t n4 = K / 4;
    int nper = 1;
    while (nper < 16 && n4 > (int64_t)nper * kMaxThreads) nper *= 2;
    if (n4 > (int64_t)nper * kMaxThreads) return cudaErrorInvalidValue;  // rows of K > 32768: not taken
    int64_t threads = (n4 + nper - 1) / nper;
    threads = (threads + 31) / 32 * 32;
    const Layout L = layout_of(rows, K);
    const int64_t ntiles = L.ntr * L.nb;
    const int64_t warps = threads / 32;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(T + (ntiles + warps - 1) / warps));
    cfg.blockDim = dim3((unsigned)threads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float4 *x4 = reinterpret_cast<const float4 *>(x);
    const uint4 *tiles = reinterpret_cast<const uint4 *>(static_cast<const char *>(data) + L.off_tiles);
    const int nb = (int)L.nb;
    switch (nper) {
        case 1: return launch_prep<1>(cfg, x4, K, q, s, T, tiles, expanded, ntiles, nb);
        case 2: return launch_prep<2>(cfg, x4, K, q, s, T, tiles, expanded, ntiles, nb);
        case 4: return launch_prep<4>(cfg, x4, K, q, s, T, tiles, expanded, ntiles, nb);
        case 8: return launch_prep<8>(cfg, x4, K, q, s, T, tiles, expanded, ntiles, nb);
        default: return launch_prep<16>(cfg, x4, K, q, s, T, tiles, expanded, ntiles, nb);
    }
}

cudaError_t launch_quant_act(const float *x, int64_t T, int64_t K, int8_t *q, float *s,
                             int32_t *blocksum, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    // float4 per thread: the smallest of 1, 2, 4, 8, 16 that fits the row in
    // 512 threads; threads: a multiple of 32 covering the row.
    const int64_t n4 = K / 4;
    int nper = 1;
    while (nper < 16 && n4 > (int64_t)nper * kMaxThreads) nper *= 2;
    const bool long_rows = n4 > (int64_t)nper * kMaxThreads;
    int64_t threads = long_rows ? kMaxThreads : (n4 + nper - 1) / nper;
    threads = (threads + 31) / 32 * 32;
    static std::atomic<bool> configured[64];  // set once per device; a repeat is harmless
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        // Same shared-memory carveout as the decode kernels, so the two can
        // share an SM under programmatic dependent launch without a
        // reconfiguration.
        const void *ks[] = {(const void *)quant_act_kernel<1, false>, (const void *)quant_act_kernel<1, true>,
                            (const void *)quant_act_kernel<2, false>, (const void *)quant_act_kernel<2, true>,
                            (const void *)quant_act_kernel<4, false>, (const void *)quant_act_kernel<4, true>,
                            (const void *)quant_act_kernel<8, false>, (const void *)quant_act_kernel<8, true>,
                            (const void *)quant_act_kernel<16, false>, (const void *)quant_act_kernel<16, true>,
                            (const void *)quant_act_long_kernel<false>, (const void *)quant_act_long_kernel<true>};
        for (const void *k : ks) {
            e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
        }
        configured[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)T);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float4 *x4 = reinterpret_cast<const float4 *>(x);
    if (long_rows) {
        if (blocksum) return cudaLaunchKernelEx(&cfg, quant_act_long_kernel<true>, x4, K, q, s, blocksum);
        return cudaLaunchKernelEx(&cfg, quant_act_long_kernel<false>, x4, K, q, s, (int32_t *)nullptr);
    }
    switch (nper) {
        case 1: return launch_one<1>(cfg, x4, K, q, s, blocksum);
        case 2: return launch_one<2>(cfg, x4, K, q, s, blocksum);
        case 4: return launch_one<4>(cfg, x4, K, q, s, blocksum);
        case 8: return launch_one<8>(cfg, x4, K, q, s, blocksum);
        default: return launch_one<16>(cfg, x4, K, q, s, blocksum);
    }
}

}  // namespace bitnet
