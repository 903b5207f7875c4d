// dp4a.cuh -- device helpers shared by the GEMV kernels: the masked dp4a
// products on i2_s code words, lane-group reductions, streaming loads and the
// per-token absmax quantisation of four activations.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnet {

static __device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

static __device__ __forceinline__ int dp4a_ss(int a, int b, int c) { return __dp4a(a, b, c); }

// Streaming 16-byte load of weights (read once: bypass L1).  volatile keeps the
// compiler from sinking it below griddepcontrol.wait.
static __device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Four masked-and-scaled group sums -> sum of code*q.
static __device__ __forceinline__ int combine4(const int a[4]) {
    return a[3] + (a[2] >> 2) + (a[1] >> 4) + (a[0] >> 6);
}

template <typename T>
__device__ __forceinline__ T tig_reduce(T v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

// q = clamp(rint(x * s), -127, 127) for four activations (IEEE fp32 multiply,
// round half to even), packed as four int8 bytes.
static __device__ __forceinline__ uint32_t quant4(float4 v, float s) {
    auto one = [&](float x) {
        int q = __float2int_rn(__fmul_rn(x, s));
        q = q > 127 ? 127 : (q < -127 ? -127 : q);
        return (uint32_t)(q & 0xff);
    };
    return one(v.x) | (one(v.y) << 8) | (one(v.z) << 16) | (one(v.w) << 24);
}

}  // namespace bitnet
