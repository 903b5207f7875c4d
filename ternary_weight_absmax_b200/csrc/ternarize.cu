// ternarize.cu -- absmean ternarisation of fp32 weights and i2_s packing, on
// the device.
//
// The pages constrain weights to {-1, 0, +1} with absmean quantisation
// ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操", section
// "为什么是 WASM"; "BitRun v0.2 实测", section "三值权重与 1.58-bit 的由来")
// and pack them as i2_s (same article, section "i2_s 到底是什么").  The
// library's reading: gamma = mean |W| accumulated in fp64 and rounded once to
// fp32 (floored at 1e-5), t = clamp(rint(W / gamma), -1, 1) with an fp32
// divide, code = t + 1, byte b of a 128-weight block holds weights b, b+32,
// b+64, b+96 at shifts 6, 4, 2, 0.
//
// Per-tensor mode: a deterministic two-pass fp64 reduction.  Pass 1: a fixed
// grid of CTAs each sums a fixed contiguous slice of |W| and writes one fp64
// partial into the caller's workspace; pass 2: one CTA adds the partials in
// index order and writes gamma.  The grid does not depend on the device, so
// the result is reproducible bit for bit.
// Per-block mode: each 128-weight block gets the mean of its own |W|, summed
// in index order by one thread (no workspace needed).
// Pass 3 (both modes): one thread per packed 32-bit word (16 weights of one
// row), writing codes and, from the first word of each block, the scale.
#include "common.cuh"

namespace bitnet {
namespace {

constexpr int kRedThreads = 256;

__global__ void __launch_bounds__(kRedThreads)
absmean_partial_kernel(const float *__restrict__ w, int64_t n, int64_t per_cta,
                       double *__restrict__ partial) {
    const int64_t begin = blockIdx.x * per_cta;
    const int64_t end = min(n, begin + per_cta);
    double acc = 0.0;
    for (int64_t i = begin + threadIdx.x; i < end; i += kRedThreads) acc += fabs((double)__ldg(w + i));
    __shared__ double red[kRedThreads];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int s = kRedThreads / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

__global__ void __launch_bounds__(kRedThreads)
absmean_final_kernel(const double *__restrict__ partial, int nparts, int64_t n,
                     float *__restrict__ gamma_out) {
    double acc = 0.0;
    for (int i = threadIdx.x; i < nparts; i += kRedThreads) acc += partial[i];
    __shared__ double red[kRedThreads];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int s = kRedThreads / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        float g = n > 0 ? (float)(red[0] / (double)n) : 0.0f;
        if (!(g >= kEps)) g = kEps;
        *gamma_out = g;
    }
}

__device__ __forceinline__ uint32_t code_of(float w, float gamma) {
    const float r = __fdiv_rn(w, gamma);
    float n = rintf(r);
    n = fminf(fmaxf(n, -1.0f), 1.0f);
    return (uint32_t)((int)n + 1);
}

// One thread per packed word: row o, block j, byte positions 4p .. 4p+3.
template <bool kPerBlock>
__global__ void ternarize_pack_kernel(const float *__restrict__ w, int64_t rows, int64_t cols,
                                      const float *__restrict__ gamma_tensor,
                                      uint32_t *__restrict__ codes, float *__restrict__ scales) {
    const int64_t nb = cols / kQK;
    const int64_t words = rows * nb * 8;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < words;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int p = (int)(idx & 7);
        const int64_t blk = idx >> 3;  // o * nb + j
        const float *wb = w + blk * kQK;
        float gamma;
        if (kPerBlock) {
            double acc = 0.0;
            for (int i = 0; i < kQK; i++) acc += fabs((double)__ldg(wb + i));
            gamma = (float)(acc / (double)kQK);
            if (!(gamma >= kEps)) gamma = kEps;
        } else {
            gamma = __ldg(gamma_tensor);
        }
        uint32_t word = 0;
#pragma unroll
        for (int byte = 0; byte < 4; byte++) {
            const int b = 4 * p + byte;
            uint32_t v = 0;
#pragma unroll
            for (int grp = 0; grp < 4; grp++) v |= code_of(__ldg(wb + grp * 32 + b), gamma) << (6 - 2 * grp);
            word |= v << (8 * byte);
        }
        codes[idx] = word;
        if (p == 0) scales[blk] = gamma;
    }
}

unsigned grid_cap(int64_t work, int threads) {
    int64_t g = (work + threads - 1) / threads;
    if (g < 1) g = 1;
    if (g > 148 * 32) g = 148 * 32;
    return (unsigned)g;
}

}  // namespace

int absmean_num_partials(int64_t n) {
    // Fixed by n alone: about 64K elements per CTA, at most 2048 CTAs.
    int64_t parts = (n + 65535) / 65536;
    if (parts < 1) parts = 1;
    if (parts > 2048) parts = 2048;
    return (int)parts;
}

cudaError_t launch_ternarize(const float *w, int64_t rows, int64_t cols, bool per_block, uint32_t *codes,
                             float *scales, double *partials, float *gamma_slot, cudaStream_t st) {
    const int64_t n = rows * cols;
    if (!per_block) {
        const int parts = absmean_num_partials(n);
        const int64_t per_cta = (n + parts - 1) / parts;
        absmean_partial_kernel<<<parts, kRedThreads, 0, st>>>(w, n, per_cta, partials);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        absmean_final_kernel<<<1, kRedThreads, 0, st>>>(partials, parts, n, gamma_slot);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ternarize_pack_kernel<false><<<grid_cap(n / 16, 256), 256, 0, st>>>(w, rows, cols, gamma_slot, codes,
                                                                           scales);
    } else {
        ternarize_pack_kernel<true><<<grid_cap(n / 16, 256), 256, 0, st>>>(w, rows, cols, nullptr, codes,
                                                                          scales);
    }
    return cudaGetLastError();
}

}  // namespace bitnet
