// gemm.cu -- prefill W2A8 GEMM on the tcgen05 int8 tensor cores.
//
// y[t][o] = (sum_j scale[o][j] * acc[t][o][j]) / s[t],
// acc = int32 block dot products of the ternary weights and the int8
// activations.  The pages time the same i2_s x int8 semantics as a CPU GEMM
// ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操", section
// "性能与内存的取舍"); on B200 the prefill case is a dense int8 contraction,
// so it runs on the tensor cores.
//
// Persistent kernel: one CTA per SM walks output tiles of 128 tokens x BN
// outputs (token tile fastest, so concurrent CTAs share weight tiles in L2),
// stepping through K one 128-wide i2_s block per pipeline stage:
//   warp 0      TMA producer: the stage's 128x128 int8 activation tile
//               (128-byte swizzle) and the BN/16 packed 512-byte code tiles.
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma
//               (M=128, N=BN, K=32, s8 x s8 -> s32), four per stage.
//   warps 2..   decoders (8 warps; 4 on the block-scale path): 2-bit codes ->
//               signed int8 {-1,0,+1} written into the B operand in the
//               128-byte-swizzled K-major layout the MMA descriptor expects
//               (c - 1 per byte without carries: (c + 0x7F) ^ 0x80).
//   last 4      epilogue: tcgen05.ld of the int32 accumulator, scale, and
//               y through 128-byte-swizzled shared staging + TMA stores.
// Two tensor-memory accumulators alternate between tiles, so the epilogue of
// one tile overlaps the main loop of the next.
// Uniform weights (all block scales of a row equal): the accumulator sums the
// whole K in int32 (|acc| <= 127*K < 2^31) and the epilogue multiplies once:
// y = float(acc) * scale_o * (1/s_t) in fp32 (three roundings, <= 2e-7 rel.).
// Otherwise (and for the accumulator-export test variant) each block is
// accumulated fresh into one of two tensor-memory buffers and the epilogue
// folds scale[o][j] * acc_j into fp64 registers while the next block runs.
// Every mbarrier wait is bounded; on a timeout the kernel latches an error
// bit, waits (bounded) for its own copies and MMAs in flight, frees tensor
// memory and returns.  Launched with programmatic dependent launch: set-up
// overlaps the previous kernel; q and s are read only after it has finished.
//
// With a caller's workspace, from kGemmExpandMinT tokens on uniform rows, the
// weights are instead expanded to int8 once per call (expand_weights_kernel
// below) and the pair kernel of gemm_pair.cu multiplies with both operands
// loaded by TMA: here every 128-token tile decodes its weights again, which
// at 2048 tokens is sixteen decodes of each weight.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "expand.cuh"
#include "tcgen05.cuh"

namespace bitnet {
namespace {

constexpr int kBM = 128;
constexpr int kEpiWarps = 4;
constexpr uint32_t kDrainLimit = 1u << 22;
constexpr unsigned kIdleSleepNs = 128;

template <int BN, bool BLOCKWISE>
struct Cfg {
    // Decode warps: 8 on the uniform path (2% faster at T = 2048 than 4; the
    // block-scale epilogue's fp64 sums need the registers 4 leave).
    static constexpr int kDecWarps = BLOCKWISE ? 4 : 8;
    static constexpr int kEpiWarp0 = 2 + kDecWarps;
    static constexpr int kThreads = 32 * (2 + kDecWarps + kEpiWarps);
    static constexpr int kStages = BLOCKWISE ? 4 : 3;
    static constexpr int kABytes = kBM * 128;        // activations, 128 x 128 int8
    static constexpr int kBBytes = BN * 128;         // decoded weights, BN x 128 int8
    static constexpr int kCBytes = BN / 16 * 512;    // packed code tiles
    static constexpr int kStageBytes = kABytes + kBBytes + kCBytes;
    static constexpr int kTmemCols = 2 * BN;         // two accumulators
    static constexpr int kOutBytes = BLOCKWISE ? 0 : kEpiWarps * 2 * 4096;  // y staging, 2 per warp
    static constexpr int kScaleBytes = kEpiWarps * BN * 4;                // scales, one copy per warp
    static constexpr int kBarBytes = 256;
    static constexpr int kOffOut = kStages * kStageBytes;
    static constexpr int kOffScale = kOffOut + kOutBytes;
    static constexpr int kOffBar = kOffScale + kScaleBytes;
    static constexpr size_t kSmem = 1024 + (size_t)kOffBar + kBarBytes;
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0, "tmem cols");
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
    int tiles_m;
    int64_t ntiles;
    int tma_store;          // y written with TMA stores (rows % 4 == 0)
};

__device__ __forceinline__ uint32_t sw128_offset(int n, int k) {
    return (uint32_t)((n >> 3) * 1024 + (n & 7) * 128 + ((((k >> 4) ^ (n & 7)) << 4) | (k & 15)));
}

// Bounded wait by lane 0 only, result broadcast to the warp, so every lane of a
// warp takes the same branch (the tcgen05.ld and __syncwarp that follow need
// the whole warp).  __syncwarp orders lane 0's acquire before the other lanes'
// reads of the data the barrier guards.
template <bool SLEEP>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint32_t limit,
                                          const volatile int *abort) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = (SLEEP ? ptx::mbar_wait_sleep(bar, parity, limit, abort, kIdleSleepNs)
                    : ptx::mbar_wait(bar, parity, limit, abort))
                 ? 1
                 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

template <int BN, bool BLOCKWISE, bool ACC>
__global__ void __launch_bounds__(Cfg<BN, BLOCKWISE>::kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_c,
            const __grid_constant__ CUtensorMap map_y, const GemmArgs args) {
    using C = Cfg<BN, BLOCKWISE>;
    constexpr int S = C::kStages;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *gbase = smem_raw + (base - raw);
    const uint32_t bars = base + C::kOffBar;
    // barrier words: full[S], dec[S], empty[S], accf[2], acce[2], drain
    auto full = [&](int s) { return bars + 8u * s; };
    auto decb = [&](int s) { return bars + 8u * (S + s); };
    auto empty = [&](int s) { return bars + 8u * (2 * S + s); };
    auto accf = [&](int a) { return bars + 8u * (3 * S + a); };
    auto acce = [&](int a) { return bars + 8u * (3 * S + 2 + a); };
    const uint32_t drain = bars + 8u * (3 * S + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::kOffBar + 8 * (3 * S + 5));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = args.nb;
    const uint32_t limit = *args.wait_limit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(decb(s), C::kDecWarps);
            ptx::mbar_init(empty(s), 1);
        }
        for (int a = 0; a < 2; a++) {
            ptx::mbar_init(accf(a), 1);
            ptx::mbar_init(acce(a), kEpiWarps);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&map_a);
        ptx::prefetch_tmap(&map_c);
        if (!BLOCKWISE && args.tma_store) ptx::prefetch_tmap(&map_y);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Everything read from here on (q, s) may be produced by the previous kernel.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(args.err, kErrTimeout);
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued[S];
            for (int s = 0; s < S; s++) issued[s] = 0;
            uint32_t it = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < args.ntiles && ok; tile += gridDim.x) {
                const int m0 = (int)(tile % args.tiles_m) * kBM;
                const int n0 = (int)(tile / args.tiles_m) * BN;
                for (int kb = 0; kb < nb; kb++, it++) {
                    const int s = (int)(it % S);
                    const uint32_t round = it / S;
                    if (round > 0 && !ptx::mbar_wait(empty(s), (round - 1) & 1, limit, abort_flag)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    const uint32_t sa = base + s * C::kStageBytes;
                    ptx::mbar_arrive_expect_tx(full(s), C::kABytes + C::kCBytes);
                    ptx::tma_load_2d(sa, &map_a, full(s), kb * 128, m0);
                    ptx::tma_load_3d(sa + C::kABytes + C::kBBytes, &map_c, full(s), 0, kb, n0 / 16);
                    issued[s]++;
                }
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
            uint32_t it = 0, ti = 0, bi = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < args.ntiles && ok; tile += gridDim.x, ti++) {
                int buf = (int)(ti & 1);
                if (!BLOCKWISE && ti >= 2 && !ptx::mbar_wait(acce(buf), ((ti >> 1) - 1) & 1, limit, abort_flag)) {
                    give_up();
                    break;
                }
                for (int kb = 0; kb < nb; kb++, it++) {
                    const int s = (int)(it % S);
                    const uint32_t round = it / S;
                    if (!ptx::mbar_wait(decb(s), round & 1, limit, abort_flag) ||
                        !ptx::mbar_wait(full(s), round & 1, limit, abort_flag)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    if (BLOCKWISE) {
                        buf = (int)(bi & 1);
                        if (bi >= 2 && !ptx::mbar_wait(acce(buf), ((bi >> 1) - 1) & 1, limit, abort_flag)) {
                            give_up();
                            ok = false;
                            break;
                        }
                    }
                    ptx::tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(buf * BN);
                    const uint32_t sa = base + s * C::kStageBytes;
                    const uint64_t da = ptx::desc_k_sw128(sa);
                    const uint64_t db = ptx::desc_k_sw128(sa + C::kABytes);
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        const uint32_t accum = BLOCKWISE ? (kk > 0) : (kb > 0 || kk > 0);
                        ptx::mma_i8(d, da + 2u * kk, db + 2u * kk, idesc, accum);
                    }
                    ptx::mma_commit(empty(s));
                    if (BLOCKWISE) {
                        ptx::mma_commit(accf(buf));
                        bi++;
                    }
                }
                if (!BLOCKWISE && ok) ptx::mma_commit(accf(buf));
            }
            // Drain: all MMAs done before tensor memory is freed.
            ptx::mma_commit(drain);
            ptx::mbar_wait(drain, 0, kDrainLimit, nullptr);
        }
        __syncwarp();
    } else if (warp < C::kEpiWarp0) {
        // ------------------------------------------------ decoders
        const int d = threadIdx.x - 64;
        constexpr int kSlots = BN / 16 * 32;
        uint32_t it = 0;
        bool ok = true;
        for (int64_t tile = blockIdx.x; tile < args.ntiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < nb; kb++, it++) {
                const int s = (int)(it % S);
                const uint32_t round = it / S;
                if (!warp_wait<false>(full(s), round & 1, limit, abort_flag)) {
                    if (lane == 0) give_up();
                    ok = false;
                    break;
                }
                const unsigned char *cs = gbase + s * C::kStageBytes + C::kABytes + C::kBBytes;
                unsigned char *bs = gbase + s * C::kStageBytes + C::kABytes;
                for (int slot = d; slot < kSlots; slot += 32 * C::kDecWarps) {
                    const uint4 c = reinterpret_cast<const uint4 *>(cs)[slot];
                    const int tile16 = slot >> 5, L = slot & 31, g = L >> 2, t = L & 3;
                    const int na = tile16 * 16 + g, nbr = na + 8;
#pragma unroll
                    for (int grp = 0; grp < 4; grp++) {
                        const int k0 = 32 * grp + 4 * t, k1 = k0 + 16;
                        *reinterpret_cast<uint32_t *>(bs + sw128_offset(na, k0)) = expand_group(c.x, grp);
                        *reinterpret_cast<uint32_t *>(bs + sw128_offset(nbr, k0)) = expand_group(c.y, grp);
                        *reinterpret_cast<uint32_t *>(bs + sw128_offset(na, k1)) = expand_group(c.z, grp);
                        *reinterpret_cast<uint32_t *>(bs + sw128_offset(nbr, k1)) = expand_group(c.w, grp);
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(decb(s));
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int e = warp - C::kEpiWarp0;       // 0..3
        const int sp = warp & 3;                 // tensor-memory lane quarter
        const int64_t rows = args.rows;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        float *scs = reinterpret_cast<float *>(gbase + C::kOffScale) + e * BN;
        if (!BLOCKWISE) {
            const uint32_t out_base = base + C::kOffOut + e * 8192;
            unsigned char *out_gen = gbase + C::kOffOut + e * 8192;
            uint32_t ti = 0, nstores = 0;
            for (int64_t tile = blockIdx.x; tile < args.ntiles; tile += gridDim.x, ti++) {
                const int64_t m0 = (tile % args.tiles_m) * kBM;
                const int64_t n0 = (tile / args.tiles_m) * BN;
                const int buf = (int)(ti & 1);
                const int64_t tok = m0 + sp * 32 + lane;
                const bool tok_ok = tok < args.T;
                for (int i = lane; i < BN; i += 32)
                    scs[i] = n0 + i < rows ? __ldg(args.rowscale + n0 + i) : 0.0f;
                const float inv_s = tok_ok ? (float)(1.0 / (double)args.s[tok]) : 0.0f;
                if (!warp_wait<true>(accf(buf), (ti >> 1) & 1, limit, abort_flag)) {
                    if (lane == 0) give_up();
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(trow + (uint32_t)(buf * BN + c0), v);
                    ptx::tmem_wait_ld();
                    if (c0 + 32 == BN) {  // accumulator fully read: hand it back to the MMA warp
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(acce(buf));
                    }
                    float o[32];
#pragma unroll
                    for (int i = 0; i < 32; i++) o[i] = __fmul_rn(__fmul_rn((float)(int)v[i], scs[c0 + i]), inv_s);
                    // A box wholly outside y (ragged last tiles) is not stored at all.
                    const bool in_range = (n0 + c0 < rows) && (m0 + sp * 32 < args.T);
                    if (args.tma_store && in_range) {
                        const uint32_t sb = nstores & 1;
                        if (nstores >= 2) {
                            if (lane == 0) ptx::bulk_wait_read<1>();
                            __syncwarp();
                        }
                        unsigned char *row = out_gen + sb * 4096 + lane * 128;
#pragma unroll
                        for (int c = 0; c < 8; c++)
                            *reinterpret_cast<float4 *>(row + ((c ^ (lane & 7)) << 4)) =
                                make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                        ptx::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            ptx::tma_store_2d(&map_y, out_base + sb * 4096, (int)(n0 + c0), (int)(m0 + sp * 32));
                            ptx::bulk_commit();
                        }
                        nstores++;
                    } else if (!args.tma_store && tok_ok) {
                        float *yrow = args.y + tok * rows;
                        for (int i = 0; i < 32; i++)
                            if (n0 + c0 + i < rows) yrow[n0 + c0 + i] = o[i];
                    }
                }
                __syncwarp();  // every lane is done with this tile's scale copy
            }
            if (lane == 0) ptx::bulk_wait<0>();
            __syncwarp();
        } else {
            uint32_t bi = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < args.ntiles && ok; tile += gridDim.x) {
                const int64_t m0 = (tile % args.tiles_m) * kBM;
                const int64_t n0 = (tile / args.tiles_m) * BN;
                const int64_t tok = m0 + sp * 32 + lane;
                const bool tok_ok = tok < args.T;
                const double inv_s = tok_ok ? 1.0 / (double)args.s[tok] : 0.0;
                double sum[BN];
#pragma unroll
                for (int i = 0; i < BN; i++) sum[i] = 0.0;
                for (int kb = 0; kb < nb; kb++, bi++) {
                    const int buf = (int)(bi & 1);
                    for (int i = lane; i < BN; i += 32) {
                        const int64_t o = n0 + i;
                        const int64_t ot = o < rows ? o : 0;
                        scs[i] = __ldg(args.tscales + ((ot >> 4) * nb + kb) * 16 + (ot & 15));
                    }
                    if (!warp_wait<true>(accf(buf), (bi >> 1) & 1, limit, abort_flag)) {
                        if (lane == 0) give_up();
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < BN; c0 += 32) {
                        uint32_t v[32];
                        ptx::tmem_ld_32x32b_x32(trow + (uint32_t)(buf * BN + c0), v);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            sum[c0 + i] += (double)scs[c0 + i] * (double)(int)v[i];
                            const int64_t o = n0 + c0 + i;
                            if (ACC && tok_ok && o < rows) args.acc[(tok * rows + o) * nb + kb] = (int)v[i];
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(acce(buf));
                }
                if (ok && tok_ok) {
                    float *yrow = args.y + tok * rows;
#pragma unroll
                    for (int i = 0; i < BN; i++)
                        if (n0 + i < rows) yrow[n0 + i] = (float)(sum[i] * inv_s);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, C::kTmemCols);
}

// Expands the repacked code tiles to int8 t = c - 1, row-major [ntr * 16]
// [cols], one warp per tile (expand.cuh).  The code words are read before
// griddepcontrol.wait (no kernel writes weights); the output, which the
// previous kernel may still be reading, is written after it.
constexpr int kExpandWarps = 8;
__global__ void __launch_bounds__(32 * kExpandWarps) expand_weights_kernel(const uint4 *tiles, int8_t *out,
                                                                           int64_t ntiles, int nb, int64_t cols) {
    __shared__ uint4 stage[kExpandWarps][32];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tj = (int64_t)blockIdx.x * kExpandWarps + warp;  // tile tr * nb + j
    const bool has = tj < ntiles;
    const uint4 v = has ? __ldcs(tiles + tj * 32 + lane) : make_uint4(0, 0, 0, 0);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (has) expand_tile(v, stage[warp], out, tj, nb, cols);
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
cudaError_t run(const void *data, const Layout &L, const int8_t *q, GemmArgs a, cudaStream_t st) {
    using C = Cfg<BN, BLOCKWISE>;
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap ma, mc, my;
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
    memset(&my, 0, sizeof(my));
    a.tma_store = 0;
    if (!BLOCKWISE && (L.rows % 4) == 0) {
        // y [T][rows] fp32; 32 x 32 boxes, 128-byte swizzle (rows*4 is a multiple of 16).
        cuuint64_t dims[2] = {(cuuint64_t)L.rows, (cuuint64_t)a.T};
        cuuint64_t strides[1] = {(cuuint64_t)L.rows * 4};
        cuuint32_t box[2] = {32, 32};
        cuuint32_t es[2] = {1, 1};
        if (enc(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.y, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        a.tma_store = 1;
    }
    auto k = gemm_kernel<BN, BLOCKWISE, ACC>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    a.tiles_m = (int)((a.T + kBM - 1) / kBM);
    const int64_t tiles_n = (L.rows + BN - 1) / BN;
    a.ntiles = (int64_t)a.tiles_m * tiles_n;
    const int64_t grid = a.ntiles < num_sms() ? a.ntiles : num_sms();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, ma, mc, my, a);
}

}  // namespace

size_t gemm_expanded_bytes(int64_t rows, int64_t cols) {
    const Layout L = layout_of(rows, cols);
    return (size_t)L.ntr * kTileRows * (size_t)L.cols;
}

cudaError_t launch_gemm(const void *data, int64_t rows, int64_t cols, bool uniform, const int8_t *q,
                        const float *s, int64_t T, float *y, int32_t *acc, const DeviceGlobals &g,
                        cudaStream_t st, int8_t *expanded) {
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
    a.tiles_m = 0;
    a.ntiles = 0;
    a.tma_store = 0;
    if (acc) return run<64, true, true>(data, L, q, a, st);
    if (uniform && expanded && T >= kGemmExpandMinT) {
        // Expand the weights once, then both operands stream in by TMA.
        const int64_t ntiles = L.ntr * L.nb;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((ntiles + kExpandWarps - 1) / kExpandWarps));
        cfg.blockDim = dim3(32 * kExpandWarps);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, expand_weights_kernel,
                                           reinterpret_cast<const uint4 *>(base + L.off_tiles), expanded, ntiles,
                                           (int)L.nb, (int64_t)L.cols);
        if (e != cudaSuccess) return e;
        return launch_gemm_pair(data, rows, cols, q, s, T, y, expanded, g, st);
    }
    if (uniform) return run<256, false, false>(data, L, q, a, st);
    return run<64, true, false>(data, L, q, a, st);
}

}  // namespace bitnet
