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

// Shared-memory word of activation word m (bytes 4m .. 4m+3 of q): lane-part t
// of block j, slot 2*group + half, so that lane t's words qa0 qb0 qa1 qb1 qa2
// qb2 qa3 qb3 of a block are contiguous.
__device__ __forceinline__ int perm_word(int m) {
    const int w = m & 31;
    return (m & ~31) | ((w & 3) << 3) | ((w >> 3) << 1) | ((w >> 2) & 1);
}

// Exact int -> fp32 for |v| < 2^22 with one integer add and one fp32 add:
// the bits 0x4B400000 + v encode 1.5 * 2^23 + v.
__device__ __forceinline__ float int_to_float(int v) {
    return __fsub_rn(__int_as_float(0x4B400000 + v), 12582912.0f);
}

// The activation quantiser's q = rint(x * s) (one fp32 multiply, ties to
// even) for four activations of a row with |x| <= absmax: then
// |x * s| <= 127 * (1 + 2^-24)^2 < 127.5, so q lies in [-127, 127] and the
// clamp never acts for finite x.  Adding 1.5 * 2^23 (round-to-nearest-even)
// leaves rint(v) in the low mantissa bits, and the low byte of those bits is q
// as an int8; three byte permutes pack the four bytes.  (NaN or Inf in x give
// unspecified bytes here.)
__device__ __forceinline__ uint32_t quant4_fast(float4 v, float s) {
    const uint32_t b0 = __float_as_uint(__fadd_rn(__fmul_rn(v.x, s), 12582912.0f));
    const uint32_t b1 = __float_as_uint(__fadd_rn(__fmul_rn(v.y, s), 12582912.0f));
    const uint32_t b2 = __float_as_uint(__fadd_rn(__fmul_rn(v.z, s), 12582912.0f));
    const uint32_t b3 = __float_as_uint(__fadd_rn(__fmul_rn(v.w, s), 12582912.0f));
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

}  // namespace bitnet
