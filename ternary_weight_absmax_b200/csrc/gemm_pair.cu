// gemm_pair.cu -- prefill W2A8 GEMM on pairs of SMs (tcgen05.mma.cta_group::2)
// for weights already expanded to int8 (t = c - 1, [rows rounded up to 16]
// [cols], written once per call by expand_weights_kernel in gemm.cu).
//
// y[t][o] = float(acc[t][o]) * scale_o * (1/s_t) for weights with uniform rows,
// acc = the int32 dot product of the ternary weights and the int8 activations
// over all of K (|acc| <= 127 K < 2^31): the same three fp32 roundings as every
// other uniform-row kernel of the library, so the same bits.  The pages time
// the i2_s x int8 GEMM on a CPU ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的
// 50 倍提速实操", section "性能与内存的取舍"); on B200 the prefill case is a dense
// int8 contraction, so it runs on the tensor cores.
//
// Why pairs.  With both operands coming from L2 by TMA, a one-SM tile of 128
// tokens x 256 weight rows loads 48 KB per 128-wide K block and its MMAs read
// 48 KB of shared memory: the SM's shared-memory and L2 bandwidth, not the
// tensor pipe, set the pace.  An M = 256 MMA over a CTA pair (a 2-CTA
// cluster) computes 256 tokens x 256 rows; each SM loads its 128 tokens and
// 128 of the 256 weight rows (32 KB per K block) and the hardware shares the
// weight halves between the two SMs: a third less traffic per SM for the same
// MMA rate.
//
// Roles (192 threads in each CTA of the pair):
//   warp 0     TMA producer: the CTA's 128 x 128 int8 activation tile and the
//              128 x 128 int8 weight tile of its rows (both 128-byte swizzled,
//              the K-major layout the MMA descriptors expect) into one of six
//              stages.  Both CTAs' copies complete on the leader's "full"
//              barrier (the pair form of the tensor copy), whose expected
//              byte count the leader sets for the two of them, so no thread
//              hands a stage across the pair.
//   warp 1     allocates tensor memory with its peer (cta_group::2).  In the
//              even CTA (the leader) one lane issues the MMAs (M = 256, N = 256,
//              K = 32, s8 x s8 -> s32) once a stage is full, and commits them
//              to the barriers of both CTAs.  In the odd CTA lane 0 relays each
//              tile's "accumulator read" to the leader (one cluster-scope
//              arrive per tile).
//   warps 2-5  epilogue: tcgen05.ld of this CTA's 128 tokens of the
//              accumulator, scale, y through swizzled staging + TMA stores.
// Two 256-column accumulators alternate between tiles, so the epilogue of one
// tile overlaps the main loop of the next.  Every mbarrier wait is bounded
// (iteration cap; the cluster-scope ones acquire at cluster scope); on a
// timeout a thread latches the error word and its CTA stops, the peer's waits
// run out the same way, and every thread of both CTAs still reaches the final
// cluster barrier before tensor memory is freed, after the MMAs have drained.
// A producer does not leave before the MMAs released the last round it loaded
// (or a long bounded wait ran out), so no copy is in flight into a CTA that
// has exited.
// No TMA load uses cluster multicast.
#include <cudaTypedefs.h>

#include <atomic>

#include "common.cuh"
#include "tcgen05.cuh"

namespace bitnet {
namespace {

constexpr int kBM = 128;  // tokens per CTA (M = 256 per pair)
constexpr int kBN = 256;  // weight rows per pair tile (N)
constexpr int kBH = 128;  // weight rows each CTA loads
constexpr int kEpiWarps = 4;
constexpr int kEpiWarp0 = 2;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kStages = 6;
constexpr int kABytes = kBM * 128;  // activations, 128 x 128 int8
constexpr int kBBytes = kBH * 128;  // weights, 128 x 128 int8
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 2 * kBN;  // two accumulators
constexpr int kOutBytes = kEpiWarps * 4096;
constexpr int kScaleBytes = kEpiWarps * kBN * 4;
constexpr int kOffOut = kStages * kStageBytes;
constexpr int kOffScale = kOffOut + kOutBytes;
constexpr int kOffBar = kOffScale + kScaleBytes;
constexpr size_t kSmem = 1024 + (size_t)kOffBar + 256;
constexpr uint32_t kDrainLimit = 1u << 22;
constexpr long long kDrainCycles = 2000000;  // ~1 ms
constexpr unsigned kIdleSleepNs = 128;
static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(kSmem <= 227 * 1024, "shared memory");

struct PairArgs {
    const float *rowscale;  // [ntr*16]
    const float *s;         // [T]
    float *y;               // [T][rows]
    unsigned *err;
    const unsigned *wait_limit;
    int64_t T, rows;
    int nb;
    int tiles_m;            // 256-token tiles
    int64_t ntiles;
    int tma_store;          // y written with TMA stores (rows % 4 == 0)
};

// ---- pair-wide tcgen05 forms (every tcgen05 op of this kernel uses cta_group::2)
__device__ __forceinline__ void tmem_alloc2(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma2_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives once on the barrier at offset `bar` in every CTA of `mask` when the
// MMAs this thread issued so far are done.
__device__ __forceinline__ void commit2(uint32_t bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"(mask)
        : "memory");
}
// A tensor copy of this CTA's tile that completes on `bar_cluster`, a barrier
// of either CTA of the pair (the pair form; no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar_cluster, int c0,
                                                 int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(dst),
        "l"((uint64_t)m), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
// Arrive on a barrier of another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Bounded wait with acquire at cluster scope (for barriers the peer arrives on).
__device__ __forceinline__ bool wait_cluster(uint32_t bar, uint32_t parity, uint32_t limit, const volatile int *abort) {
    for (uint32_t i = 0; i < limit; i++) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (abort && *abort) return false;
    }
    return false;
}

// Bounded wait by lane 0 only, result broadcast to the warp (the tcgen05.ld
// and __syncwarp that follow need the whole warp).
__device__ __forceinline__ bool warp_wait_sleep(uint32_t bar, uint32_t parity, uint32_t limit,
                                                const volatile int *abort) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait_sleep(bar, parity, limit, abort, kIdleSleepNs) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const __grid_constant__ CUtensorMap map_y, const PairArgs args) {
    constexpr int S = kStages;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *gbase = smem_raw + (base - raw);
    const uint32_t bars = base + kOffBar;
    // barrier words: full[S] (the leader's: both CTAs' copies of a stage),
    // empty[S], accf[2], acce[2] (leader), acel[2] (the odd CTA's, relayed),
    // drain
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (S + s); };
    auto accf = [&](int a) { return bars + 8u * (2 * S + a); };
    auto acce = [&](int a) { return bars + 8u * (2 * S + 2 + a); };
    auto acel = [&](int a) { return bars + 8u * (2 * S + 4 + a); };
    const uint32_t drain = bars + 8u * (2 * S + 6);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + kOffBar + 8 * (2 * S + 7));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_rank();  // 0: the leader, 1: its peer
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int nb = args.nb;
    const uint32_t limit = *args.wait_limit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), 1);
        }
        for (int a = 0; a < 2; a++) {
            ptx::mbar_init(accf(a), 1);
            ptx::mbar_init(acce(a), kEpiWarps + 1);  // the leader's: its epilogue + the relay
            ptx::mbar_init(acel(a), kEpiWarps);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&map_a);
        ptx::prefetch_tmap(&map_b);
        if (args.tma_store) ptx::prefetch_tmap(&map_y);
    }
    if (warp == 1) {
        tmem_alloc2(ptx::smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish2();
    }
    // Both CTAs' barriers are initialised and tensor memory allocated before
    // any CTA arrives on, or issues MMAs into, its peer.
    ptx::tc_fence_before();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Everything read from here on (q, s, the expanded weights) may be
    // produced by the previous kernel.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(args.err, kErrTimeout);
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (each CTA)
        if (lane == 0) {
            int issued[S];
            for (int s = 0; s < S; s++) issued[s] = 0;
            uint32_t it = 0;
            bool ok = true;
            for (int64_t tile = pair; tile < args.ntiles && ok; tile += npairs) {
                const int m0 = (int)(tile % args.tiles_m) * (2 * kBM) + (int)rank * kBM;
                const int r0 = (int)(tile / args.tiles_m) * kBN + (int)rank * kBH;
                for (int kb = 0; kb < nb; kb++, it++) {
                    const int s = (int)(it % S);
                    const uint32_t round = it / S;
                    if (round > 0 && !ptx::mbar_wait(empty(s), (round - 1) & 1, limit, abort_flag)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    const uint32_t sa = base + s * kStageBytes;
                    const uint32_t fb = ptx::map_to_rank(full(s), 0);  // the leader's barrier
                    if (rank == 0) ptx::mbar_arrive_expect_tx(full(s), 2 * (kABytes + kBBytes));
                    tma_load_2d_pair(sa, &map_a, fb, kb * 128, m0);
                    tma_load_2d_pair(sa + kABytes, &map_b, fb, kb * 128, r0);
                    issued[s]++;
                }
            }
            // The MMAs release a round only after reading it, so once the last
            // round of every stage is released no copy of this CTA is in
            // flight.  After a timeout a round may never be released: the wait
            // then gives up after ~1 ms of SM clock, far longer than a copy.
            for (int s = 0; s < S; s++) {
                if (issued[s] == 0) continue;
                const long long t0 = clock64();
                while (!ptx::mbar_try_wait(empty(s), (uint32_t)(issued[s] - 1) & 1u))
                    if (clock64() - t0 > kDrainCycles) break;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // -------------------------------------------- MMA issuer (the leader)
            constexpr uint32_t idesc = ptx::idesc_i8(2 * kBM, kBN);
            uint32_t it = 0, ti = 0;
            bool ok = true;
            for (int64_t tile = pair; tile < args.ntiles && ok; tile += npairs, ti++) {
                const int buf = (int)(ti & 1);
                if (ti >= 2 && !wait_cluster(acce(buf), ((ti >> 1) - 1) & 1, limit, abort_flag)) {
                    give_up();
                    break;
                }
                for (int kb = 0; kb < nb; kb++, it++) {
                    const int s = (int)(it % S);
                    const uint32_t round = it / S;
                    if (!ptx::mbar_wait(full(s), round & 1, limit, abort_flag)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(buf * kBN);
                    const uint32_t sa = base + s * kStageBytes;
                    const uint64_t da = ptx::desc_k_sw128(sa);
                    const uint64_t db = ptx::desc_k_sw128(sa + kABytes);
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        mma2_i8(d, da + 2u * kk, db + 2u * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    commit2(empty(s), 0x3);
                }
                if (ok) commit2(accf(buf), 0x3);
            }
            commit2(drain, 0x3);  // both CTAs learn when every MMA is done
        } else if (rank == 1 && lane == 0) {
            // -------------------------------------------- the odd CTA's relay
            uint32_t ti = 0;
            for (int64_t tile = pair; tile < args.ntiles; tile += npairs, ti++) {
                const int buf = (int)(ti & 1);
                if (!ptx::mbar_wait(acel(buf), (ti >> 1) & 1, limit, abort_flag)) {
                    give_up();
                    break;
                }
                arrive_remote(ptx::map_to_rank(acce(buf), 0));
            }
        }
        // The tensor memory of both CTAs stays allocated until the MMAs drained.
        if (lane == 0) ptx::mbar_wait(drain, 0, kDrainLimit, nullptr);
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (each CTA)
        const int e = warp - kEpiWarp0;  // 0..3
        const int sp = warp & 3;         // tensor-memory lane quarter
        const int64_t rows = args.rows;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        float *scs = reinterpret_cast<float *>(gbase + kOffScale) + e * kBN;
        const uint32_t out_base = base + kOffOut + e * 4096;
        unsigned char *out_gen = gbase + kOffOut + e * 4096;
        uint32_t ti = 0, nstores = 0;
        for (int64_t tile = pair; tile < args.ntiles; tile += npairs, ti++) {
            const int64_t m0 = (tile % args.tiles_m) * (2 * kBM) + (int64_t)rank * kBM;
            const int64_t n0 = (tile / args.tiles_m) * kBN;
            const int buf = (int)(ti & 1);
            const int64_t tok = m0 + sp * 32 + lane;
            const bool tok_ok = tok < args.T;
            for (int i = lane; i < kBN; i += 32) scs[i] = n0 + i < rows ? __ldg(args.rowscale + n0 + i) : 0.0f;
            const float inv_s = tok_ok ? (float)(1.0 / (double)args.s[tok]) : 0.0f;
            if (!warp_wait_sleep(accf(buf), (ti >> 1) & 1, limit, abort_flag)) {
                if (lane == 0) give_up();
                break;
            }
            ptx::tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(trow + (uint32_t)(buf * kBN + c0), v);
                ptx::tmem_wait_ld();
                if (c0 + 32 == kBN) {  // accumulator fully read: hand it back
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(rank == 0 ? acce(buf) : acel(buf));
                }
                float o[32];
#pragma unroll
                for (int i = 0; i < 32; i++) o[i] = __fmul_rn(__fmul_rn((float)(int)v[i], scs[c0 + i]), inv_s);
                // A box wholly outside y (ragged last tiles) is not stored at all.
                const bool in_range = (n0 + c0 < rows) && (m0 + sp * 32 < args.T);
                if (args.tma_store && in_range) {
                    if (nstores >= 1) {  // the staging buffer's previous store has read it
                        if (lane == 0) ptx::bulk_wait_read<0>();
                        __syncwarp();
                    }
                    unsigned char *row = out_gen + lane * 128;
#pragma unroll
                    for (int c = 0; c < 8; c++)
                        *reinterpret_cast<float4 *>(row + ((c ^ (lane & 7)) << 4)) =
                            make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::tma_store_2d(&map_y, out_base, (int)(n0 + c0), (int)(m0 + sp * 32));
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
    }

    // No CTA of the pair leaves, or frees tensor memory, while its peer may
    // still arrive on its barriers or the MMAs read its shared memory.
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    if (warp == 1) tmem_dealloc2(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        fn.store(f, std::memory_order_release);
    }
    return f;
}

}  // namespace

cudaError_t launch_gemm_pair(const void *data, int64_t rows, int64_t cols, const int8_t *q, const float *s,
                             int64_t T, float *y, const int8_t *expanded, const DeviceGlobals &g,
                             cudaStream_t st) {
    static std::atomic<bool> configured[64];
    const Layout L = layout_of(rows, cols);
    const char *base = static_cast<const char *>(data);
    PairArgs a;
    a.rowscale = reinterpret_cast<const float *>(base + L.off_rowscale);
    a.s = s;
    a.y = y;
    a.err = g.err;
    a.wait_limit = g.wait_limit;
    a.T = T;
    a.rows = rows;
    a.nb = (int)L.nb;
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap ma, mb, my;
    {
        cuuint64_t dims[2] = {(cuuint64_t)L.cols, (cuuint64_t)T};
        cuuint64_t strides[1] = {(cuuint64_t)L.cols};
        cuuint32_t box[2] = {128, kBM};
        cuuint32_t es[2] = {1, 1};
        if (enc(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(q), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)L.cols, (cuuint64_t)(L.ntr * kTileRows)};
        cuuint64_t strides[1] = {(cuuint64_t)L.cols};
        cuuint32_t box[2] = {128, kBH};
        cuuint32_t es[2] = {1, 1};
        if (enc(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(expanded), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    memset(&my, 0, sizeof(my));
    a.tma_store = 0;
    if ((L.rows % 4) == 0) {
        // y [T][rows] fp32; 32 x 32 boxes, 128-byte swizzle (rows*4 is a multiple of 16).
        cuuint64_t dims[2] = {(cuuint64_t)L.rows, (cuuint64_t)T};
        cuuint64_t strides[1] = {(cuuint64_t)L.rows * 4};
        cuuint32_t box[2] = {32, 32};
        cuuint32_t es[2] = {1, 1};
        if (enc(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        a.tma_store = 1;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    a.tiles_m = (int)((T + 2 * kBM - 1) / (2 * kBM));
    const int64_t tiles_n = (rows + kBN - 1) / kBN;
    a.ntiles = (int64_t)a.tiles_m * tiles_n;
    const int64_t pairs_max = num_sms() / 2;
    const int64_t pairs = a.ntiles < pairs_max ? a.ntiles : pairs_max;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, gemm_pair_kernel, ma, mb, my, a);
}

}  // namespace bitnet
