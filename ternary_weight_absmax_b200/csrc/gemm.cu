// gemm.cu -- prefill W2A8 GEMM on the tcgen05 int8 tensor cores.
//
// y[t][o] = (sum_j scale[o][j] * acc[t][o][j]) / s[t],
// acc = int32 block dot products of the ternary weights and the int8
// activations.  The pages time the same i2_s x int8 semantics as a CPU GEMM
// ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操", section
// "性能与内存的取舍"); on B200 the prefill case is a dense int8 contraction,
// so it runs on the tensor cores.
//
// One CTA computes a 128-token x BN-output tile, stepping through K one
// 128-wide i2_s block per pipeline stage:
//   warp 0      TMA producer: the stage's 128x128 int8 activation tile
//               (128-byte swizzle) and the BN/16 packed 512-byte code tiles.
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma
//               (M=128, N=BN, K=32, s8 x s8 -> s32), four per stage, and
//               commits each stage back to the producer.
//   warps 2-5   decoders: 2-bit codes -> signed int8 {-1,0,+1} written into
//               the B operand in the 128-byte-swizzled K-major layout the
//               MMA descriptor expects (c - 1 per byte without carries:
//               (c + 0x7F) ^ 0x80).
//   warps 6-9   epilogue: tcgen05.ld of the int32 accumulator, scale, store.
// Uniform weights (all block scales of a row equal): the accumulator sums the
// whole K in int32 (|acc| <= 127*K < 2^31) and the epilogue multiplies once.
// Otherwise (and for the accumulator-export test variant) each block is
// accumulated fresh into one of two tensor-memory buffers and the epilogue
// folds scale[o][j] * acc_j into fp64 registers while the next block runs.
// Every mbarrier wait is bounded; on a timeout the kernel latches an error
// bit, waits (bounded) for its own copies and MMAs in flight, frees tensor
// memory and returns.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace bitnet {
namespace {

constexpr int kBM = 128;
constexpr int kThreads = 320;  // 10 warps
constexpr uint32_t kDrainLimit = 1u << 22;

template <int BN, bool BLOCKWISE>
struct Cfg {
    static constexpr int kStages = BLOCKWISE ? 4 : 3;
    static constexpr int kABytes = kBM * 128;        // activations, 128 x 128 int8
    static constexpr int kBBytes = BN * 128;         // decoded weights, BN x 128 int8
    static constexpr int kCBytes = BN / 16 * 512;    // packed code tiles
    static constexpr int kStageBytes = kABytes + kBBytes + kCBytes;
    static constexpr int kTmemCols = BLOCKWISE ? 2 * BN : BN;
    static constexpr int kBarBytes = 256;
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + kBarBytes;
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kTmemCols >= 32 && (kTmemCols & (kTmemCols - 1)) == 0, "tmem cols power of two");
};

struct GemmArgs {
    const float *tscales;   // [ntr][nb][16]
    const float *rowscale;  // [ntr*16]
    const float *s;         // [T]
    float *y;               // [T][rows]
    int32_t *acc;           // [T][rows][nb] or null
    unsigned *err;
    const unsigned *wait_limit;
    int64_t T, rows;
    int nb;
};

__device__ __forceinline__ uint32_t sw128_offset(int n, int k) {
    return (uint32_t)((n >> 3) * 1024 + (n & 7) * 128 + ((((k >> 4) ^ (n & 7)) << 4) | (k & 15)));
}

__device__ __forceinline__ uint32_t decode_group(uint32_t w, int grp) {
    const uint32_t c = (w >> (6 - 2 * grp)) & 0x03030303u;
    return (c + 0x7F7F7F7Fu) ^ 0x80808080u;
}

// Bounded wait by lane 0 only, result broadcast to the warp, so every lane of a
// warp takes the same branch (the tcgen05.ld and __syncwarp that follow need
// the whole warp).  __syncwarp orders lane 0's acquire before the other lanes'
// reads of the data the barrier guards.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint32_t limit,
                                          const volatile int *abort) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, limit, abort) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

template <int BN, bool BLOCKWISE, bool ACC>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_c,
            const GemmArgs args) {
    using C = Cfg<BN, BLOCKWISE>;
    constexpr int S = C::kStages;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *gbase = smem_raw + (base - raw);
    const uint32_t bars = base + S * C::kStageBytes;
    // barrier words: full[S], dec[S], empty[S], accf[2], acce[2], drain
    auto full = [&](int s) { return bars + 8u * s; };
    auto decb = [&](int s) { return bars + 8u * (S + s); };
    auto empty = [&](int s) { return bars + 8u * (2 * S + s); };
    auto accf = [&](int a) { return bars + 8u * (3 * S + a); };
    auto acce = [&](int a) { return bars + 8u * (3 * S + 2 + a); };
    const uint32_t drain = bars + 8u * (3 * S + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + S * C::kStageBytes + 8 * (3 * S + 5));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.x * kBM;
    const int64_t n0 = (int64_t)blockIdx.y * BN;
    const int nb = args.nb;
    const uint32_t limit = *args.wait_limit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(decb(s), 4);
            ptx::mbar_init(empty(s), 1);
        }
        for (int a = 0; a < 2; a++) {
            ptx::mbar_init(accf(a), 1);
            ptx::mbar_init(acce(a), 4);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&map_a);
        ptx::prefetch_tmap(&map_c);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(args.err, kErrTimeout);
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued[S];
            for (int s = 0; s < S; s++) issued[s] = 0;
            for (int kb = 0; kb < nb; kb++) {
                const int s = kb % S, round = kb / S;
                if (round > 0 && !ptx::mbar_wait(empty(s), (round - 1) & 1, limit, abort_flag)) {
                    give_up();
                    break;
                }
                const uint32_t sa = base + s * C::kStageBytes;
                ptx::mbar_arrive_expect_tx(full(s), C::kABytes + C::kCBytes);
                ptx::tma_load_2d(sa, &map_a, full(s), kb * 128, (int)m0);
                ptx::tma_load_3d(sa + C::kABytes + C::kBBytes, &map_c, full(s), 0, kb, (int)(n0 / 16));
                issued[s]++;
            }
            // Drain: every load this thread issued has landed before shared
            // memory can be released.
            for (int s = 0; s < S; s++)
                if (issued[s] > 0) ptx::mbar_wait(full(s), (issued[s] - 1) & 1, kDrainLimit, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_i8(kBM, BN);
            for (int kb = 0; kb < nb; kb++) {
                const int s = kb % S, round = kb / S;
                if (!ptx::mbar_wait(decb(s), round & 1, limit, abort_flag) ||
                    !ptx::mbar_wait(full(s), round & 1, limit, abort_flag)) {
                    give_up();
                    break;
                }
                uint32_t d = tmem;
                if (BLOCKWISE) {
                    const int a = kb & 1;
                    if (kb >= 2 && !ptx::mbar_wait(acce(a), ((kb >> 1) - 1) & 1, limit, abort_flag)) {
                        give_up();
                        break;
                    }
                    d = tmem + (uint32_t)(a * BN);
                }
                ptx::tc_fence_after();
                const uint32_t sa = base + s * C::kStageBytes;
                const uint64_t da = ptx::desc_k_sw128(sa);
                const uint64_t db = ptx::desc_k_sw128(sa + C::kABytes);
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    const uint32_t accum = BLOCKWISE ? (kk > 0) : (kb > 0 || kk > 0);
                    ptx::mma_i8(d, da + 2u * kk, db + 2u * kk, idesc, accum);
                }
                ptx::mma_commit(empty(s));
                if (BLOCKWISE) ptx::mma_commit(accf(kb & 1));
            }
            if (!BLOCKWISE) ptx::mma_commit(accf(0));
            // Drain: all MMAs done before tensor memory is freed.
            ptx::mma_commit(drain);
            ptx::mbar_wait(drain, 0, kDrainLimit, nullptr);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------ decoders
        const int d = threadIdx.x - 64;  // 0..127
        constexpr int kSlots = BN / 16 * 32;
        for (int kb = 0; kb < nb; kb++) {
            const int s = kb % S, round = kb / S;
            if (!warp_wait(full(s), round & 1, limit, abort_flag)) {
                if (lane == 0) give_up();
                break;
            }
            const unsigned char *cs = gbase + s * C::kStageBytes + C::kABytes + C::kBBytes;
            unsigned char *bs = gbase + s * C::kStageBytes + C::kABytes;
            for (int slot = d; slot < kSlots; slot += 128) {
                const uint4 c = reinterpret_cast<const uint4 *>(cs)[slot];
                const int tile = slot >> 5, L = slot & 31, g = L >> 2, t = L & 3;
                const int na = tile * 16 + g, nbr = na + 8;
#pragma unroll
                for (int grp = 0; grp < 4; grp++) {
                    const int k0 = 32 * grp + 4 * t, k1 = k0 + 16;
                    *reinterpret_cast<uint32_t *>(bs + sw128_offset(na, k0)) = decode_group(c.x, grp);
                    *reinterpret_cast<uint32_t *>(bs + sw128_offset(nbr, k0)) = decode_group(c.y, grp);
                    *reinterpret_cast<uint32_t *>(bs + sw128_offset(na, k1)) = decode_group(c.z, grp);
                    *reinterpret_cast<uint32_t *>(bs + sw128_offset(nbr, k1)) = decode_group(c.w, grp);
                }
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(decb(s));
        }
    } else {
        // ------------------------------------------------ epilogue
        const int sp = warp & 3;                 // tensor-memory lane quarter
        const int m = sp * 32 + lane;            // row of the tile
        const int64_t tok = m0 + m;
        const bool tok_ok = tok < args.T;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const int64_t rows = args.rows;
        float *yrow = args.y + (tok_ok ? tok : 0) * rows;
        const bool vec_ok = (rows & 3) == 0;
        if (!BLOCKWISE) {
            const float inv_s = tok_ok ? (float)(1.0 / (double)args.s[tok]) : 0.0f;
            if (!warp_wait(accf(0), 0, limit, abort_flag)) {
                if (lane == 0) give_up();
            } else {
                ptx::tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(trow + (uint32_t)c0, v);
                    ptx::tmem_wait_ld();
                    const int64_t o0 = n0 + c0;
                    float outv[32];
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const int64_t o = o0 + i;
                        const float g = o < rows ? __ldg(args.rowscale + o) : 0.0f;
                        outv[i] = __fmul_rn(__fmul_rn((float)(int)v[i], g), inv_s);
                    }
                    if (tok_ok) {
                        if (vec_ok && o0 + 32 <= rows) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                __stcs(reinterpret_cast<float4 *>(yrow + o0 + i),
                                       make_float4(outv[i], outv[i + 1], outv[i + 2], outv[i + 3]));
                        } else {
                            for (int i = 0; i < 32; i++)
                                if (o0 + i < rows) yrow[o0 + i] = outv[i];
                        }
                    }
                }
            }
        } else {
            const double inv_s = tok_ok ? 1.0 / (double)args.s[tok] : 0.0;
            double sum[BN];
#pragma unroll
            for (int i = 0; i < BN; i++) sum[i] = 0.0;
            bool ok = true;
            for (int kb = 0; kb < nb && ok; kb++) {
                const int a = kb & 1;
                if (!warp_wait(accf(a), (kb >> 1) & 1, limit, abort_flag)) {
                    if (lane == 0) give_up();
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(trow + (uint32_t)(a * BN + c0), v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const int64_t o = n0 + c0 + i;
                        const int64_t ot = o < rows ? o : 0;
                        const float sc = __ldg(args.tscales + ((ot >> 4) * nb + kb) * 16 + (ot & 15));
                        sum[c0 + i] += (double)sc * (double)(int)v[i];
                        if (ACC && tok_ok && o < rows) args.acc[(tok * rows + o) * nb + kb] = (int)v[i];
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(acce(a));
            }
            if (ok && tok_ok) {
#pragma unroll
                for (int i = 0; i < BN; i++) {
                    const int64_t o = n0 + i;
                    if (o < rows) yrow[o] = (float)(sum[i] * inv_s);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, C::kTmemCols);
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

template <int BN, bool BLOCKWISE, bool ACC>
cudaError_t run(const void *data, const Layout &L, const int8_t *q, const GemmArgs &a, cudaStream_t st) {
    using C = Cfg<BN, BLOCKWISE>;
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap ma, mc;
    {
        cuuint64_t dims[2] = {(cuuint64_t)L.cols, (cuuint64_t)a.T};
        cuuint64_t strides[1] = {(cuuint64_t)L.cols};
        cuuint32_t box[2] = {128, kBM};
        cuuint32_t es[2] = {1, 1};
        if (enc(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(q), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const char *tiles = static_cast<const char *>(data) + L.off_tiles;
        cuuint64_t dims[3] = {128, (cuuint64_t)L.nb, (cuuint64_t)L.ntr};
        cuuint64_t strides[2] = {512, (cuuint64_t)L.nb * 512};
        cuuint32_t box[3] = {128, 1, BN / 16};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<char *>(tiles), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    auto k = gemm_kernel<BN, BLOCKWISE, ACC>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    const int64_t gy = (L.rows + BN - 1) / BN;
    if (gy > 65535) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)((a.T + kBM - 1) / kBM), (unsigned)gy);
    k<<<grid, kThreads, C::kSmem, st>>>(ma, mc, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const void *data, int64_t rows, int64_t cols, bool uniform, const int8_t *q,
                        const float *s, int64_t T, float *y, int32_t *acc, const DeviceGlobals &g,
                        cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    const char *base = static_cast<const char *>(data);
    GemmArgs a;
    a.tscales = reinterpret_cast<const float *>(base + L.off_tscales);
    a.rowscale = reinterpret_cast<const float *>(base + L.off_rowscale);
    a.s = s;
    a.y = y;
    a.acc = acc;
    a.err = g.err;
    a.wait_limit = g.wait_limit;
    a.T = T;
    a.rows = rows;
    a.nb = (int)L.nb;
    if (acc) return run<64, true, true>(data, L, q, a, st);
    if (uniform) return run<256, false, false>(data, L, q, a, st);
    return run<64, true, false>(data, L, q, a, st);
}

}  // namespace bitnet
