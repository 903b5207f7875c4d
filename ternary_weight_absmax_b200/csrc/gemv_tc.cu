// gemv_tc.cu -- small-batch W2A8 GEMV (2..64 tokens, uniform rows) on the
// tcgen05 int8 tensor cores, weights on the M side ("swap AB").
//
// y[b][o] = rowscale[o] * (sum_k t[o][k] * q[b][k]) * (1/s[b])  in fp32, the
// same three roundings as the batch-1 and batched decode kernels, so all of
// them give the same bits.  The integer product is that of the pages (+1 adds,
// -1 subtracts, 0 skips: "BitRun v0.2 实测：1-bit LLM 终端驾驶舱与毫瓦级功耗
// 遥测", section "三值权重与 1.58-bit 的由来"; 2-bit weights x 8-bit
// activations: "5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构对决",
// section "GPU内核突破").
//
// Why tensor cores here and not at batch 1: with B tokens the dp4a kernels
// spend B dp4a per four weights and become ALU-bound from B ~ 4 on; an MMA
// spends the same decode work on every token count.  Layout of the work:
//   * a CTA owns a 128-row M tile (eight 16-row weight tiles) and a slice of
//     the K blocks; the CTAs that split one M tile's K form a cluster (1..8)
//     and add their int32 partial sums into the first CTA's shared memory
//     (distributed shared memory), which writes y; integer adds keep the
//     result independent of their order;
//   * warp 0 loads each K block's code tiles (4 KB) and the block's int8
//     activations (NT tokens x 128 bytes, 128-byte swizzle; rows past B are
//     zero-filled by the TMA) into one of S pipeline stages;
//   * warps 2..5 decode the 2-bit codes c = t + 1 of their 32 rows into
//     bytes (one shift and one mask per four weights) and store them into
//     tensor memory with tcgen05.st: the A operand of the MMA is read from
//     tensor memory, so decoded weights never take shared-memory bandwidth;
//     they also sum q per token over the CTA's K slice;
//   * warp 1 issues tcgen05.mma kind::i8 (M = 128, N = NT, K = 32; A = u8
//     codes from tensor memory, B = s8 activations from shared memory) into a
//     tensor-memory accumulator: D = sum c * q, and sum t * q = D - sum q;
//   * warps 2..5 then read the accumulator (thread = row), subtract sum q,
//     and either write y (no split) or add into the cluster's first CTA.
// Launched with programmatic dependent launch: the first stages' weight
// copies start before griddepcontrol.wait; q and s are read after it.  Every
// mbarrier wait is bounded; on a timeout the kernel latches the error word,
// stops, waits (bounded) for its own copies and MMAs, frees tensor memory and
// reaches the cluster barrier like every other thread, so nothing hangs.
#include <cudaTypedefs.h>

#include <atomic>

#include "common.cuh"
#include "dp4a.cuh"
#include "tcgen05.cuh"

namespace bitnet {
namespace {

constexpr int kDecSets = 2;       // decoder warp sets (4 warps each), taking K blocks in turn
constexpr int kDecBatch = 2;      // K blocks a set decodes per wait for its tensor-memory stores
constexpr int kThreads = 64 + 128 * kDecSets;  // producer, MMA, decoders (the first set also the epilogue)
constexpr int kTmemCols = 256;    // accumulator at [0, 64), A buffers at 64 + 32 * buffer
constexpr int kAcol = 64;
constexpr int kNA = 6;            // tensor-memory A buffers (one K block each)
constexpr uint32_t kDrainLimit = 1u << 22;

// NT tokens per CTA (16, 32 or 64).  The shared-memory ring is deeper than
// the tensor-memory one: a stage lives from its copy until its MMAs finish,
// most of it waiting on HBM, while an A buffer lives only from its decode to
// its MMAs.  About 96 KB of stages per CTA, two CTAs per SM.
template <int NT>
struct TcCfg {
    static constexpr int kStages = NT == 16 ? 16 : (NT == 32 ? 12 : 8);
    static constexpr int kQBytes = NT * 128;                  // activations of one block, 128-byte rows
    static constexpr int kCodeBytes = 8 * kTileBytes;         // eight 16-row code tiles of one block
    static constexpr int kStageBytes = kQBytes + kCodeBytes;  // multiple of 1024
    static constexpr int kPartStride = NT + 1;                // int32 partial sums [128][NT + 1] (+1: banks)
    static constexpr int kOffSq = kStages * kStageBytes;
    static constexpr int kOffInv = kOffSq + NT * 4;
    static constexpr int kOffBar = kOffInv + NT * 4;
    // At least 80 KB so that no more than two CTAs share an SM: two hold all
    // 512 tensor-memory columns, and a third would block in its allocation.
    static constexpr size_t kUsed = 1024 + (size_t)kOffBar + 512;
    static constexpr size_t kSmem = kUsed > 80 * 1024 ? kUsed : 80 * 1024;
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    static_assert(128 * kPartStride * 4 <= kOffSq, "partial sums fit in the stages they reuse");
    static_assert(kSmem <= 110 * 1024, "two CTAs per SM");
    static_assert(kAcol + 32 * kNA <= kTmemCols && NT <= kAcol, "tensor-memory columns");
};

struct TcArgs {
    const float *rowscale;  // [ntr * 16]
    const float *s;         // [B]
    float *y;               // [B][rows]
    unsigned *err;
    const unsigned *wait_limit;
    int64_t rows;
    int B, nb, splits;
};

// Decoded codes of one lane's 16 bytes of a tile, in the order of
// tmem_st_16x128b_x8: group gg of the 128-weight block (K = 32 gg .. 32 gg +
// 31) goes to columns 8 gg .. 8 gg + 7; within it, x (row g, bytes 4t..4t+3
// of the block's 32), y (row g + 8, same bytes), z (row g, bytes 16+4t..), w
// (row g + 8, bytes 16+4t..).  Byte b of a block holds weights b, b+32, b+64,
// b+96 at shifts 6, 4, 2, 0, so group gg of byte b is weight 32 gg + b.
__device__ __forceinline__ void decode_tile(const uint4 w, uint32_t (&v)[16]) {
#pragma unroll
    for (int gg = 0; gg < 4; gg++) {
        const int sh = 6 - 2 * gg;
        v[4 * gg + 0] = (w.x >> sh) & 0x03030303u;
        v[4 * gg + 1] = (w.y >> sh) & 0x03030303u;
        v[4 * gg + 2] = (w.z >> sh) & 0x03030303u;
        v[4 * gg + 3] = (w.w >> sh) & 0x03030303u;
    }
}

template <bool SLEEP>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint32_t limit, const volatile int *abort) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = (SLEEP ? ptx::mbar_wait_sleep(bar, parity, limit, abort, 64) : ptx::mbar_wait(bar, parity, limit, abort))
                 ? 1
                 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 2)
gemv_tc_kernel(const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_q, const TcArgs a) {
    using C = TcCfg<NT>;
    constexpr int S = C::kStages;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = a.splits > 1 ? ptx::cluster_rank() : 0u;
    const int mt = (int)(blockIdx.x / (unsigned)a.splits);
    const int bt = a.B;  // tokens (<= NT)
    const int j0 = (int)((int64_t)rank * a.nb / a.splits);
    const int nj = (int)((int64_t)(rank + 1) * a.nb / a.splits) - j0;
    const uint32_t bars = base + C::kOffBar;
    auto full = [&](int s) { return bars + 8u * s; };
    auto empty = [&](int s) { return bars + 8u * (S + s); };
    auto decb = [&](int b) { return bars + 8u * (2 * S + b); };
    auto afree = [&](int b) { return bars + 8u * (2 * S + kNA + b); };
    const uint32_t accf = bars + 8u * (2 * S + 2 * kNA);
    const uint32_t drain = accf + 8u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::kOffBar + 8 * (2 * S + 2 * kNA + 2));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *part = reinterpret_cast<int *>(gbase);  // [128][kPartStride], after the main loop
    int *sq = reinterpret_cast<int *>(gbase + C::kOffSq);
    float *inv = reinterpret_cast<float *>(gbase + C::kOffInv);
    const uint32_t limit = *a.wait_limit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), 1);
        }
        for (int b = 0; b < kNA; b++) {
            ptx::mbar_init(decb(b), 4);
            ptx::mbar_init(afree(b), 1);
        }
        ptx::mbar_init(accf, 1);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&map_c);
        ptx::prefetch_tmap(&map_q);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    for (int i = threadIdx.x; i < NT; i += kThreads) sq[i] = 0;
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(a.err, kErrTimeout);
    };
    const int npre = nj < S ? nj : S;
    // Weights do not depend on the previous kernel: their first copies go out now.
    if (warp == 0 && lane == 0) {
        for (int k = 0; k < npre; k++) {
            ptx::mbar_arrive_expect_tx(full(k), C::kCodeBytes + C::kQBytes);
            ptx::tma_load_3d(base + k * C::kStageBytes + C::kQBytes, &map_c, full(k), 0, j0 + k, mt * 8);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // q, s ready; y free
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < nj; it++) {
                const int s = it % S;
                if (it >= S) {
                    if (!ptx::mbar_wait(empty(s), ((it / S) - 1) & 1, limit, abort_flag)) {
                        give_up();
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(full(s), C::kCodeBytes + C::kQBytes);
                    ptx::tma_load_3d(base + s * C::kStageBytes + C::kQBytes, &map_c, full(s), 0, j0 + it, mt * 8);
                }
                ptx::tma_load_2d(base + s * C::kStageBytes, &map_q, full(s), 128 * (j0 + it), 0);
                issued = it + 1;
            }
            // Copies in flight (the last S stages issued) land before the CTA
            // can exit.  A give-up happens only from stage S on, so every stage
            // issued before it has both of its copies.
            for (int it = issued > S ? issued - S : 0; it < issued; it++)
                ptx::mbar_wait(full(it % S), (it / S) & 1, kDrainLimit, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_i8(128, NT, false);
            for (int it = 0; it < nj; it++) {
                const int s = it % S, ab = it % kNA;
                if (!ptx::mbar_wait(decb(ab), (it / kNA) & 1, limit, abort_flag)) {
                    give_up();
                    break;
                }
                ptx::tc_fence_after();
                const uint64_t bdesc = ptx::desc_k_sw128(base + s * C::kStageBytes);
                const uint32_t acol = tmem + (uint32_t)(kAcol + 32 * ab);
#pragma unroll
                for (int gg = 0; gg < 4; gg++)
                    ptx::mma_i8_ta(tmem, acol + 8u * gg, bdesc + 2u * gg, idesc, (it > 0 || gg > 0) ? 1u : 0u);
                ptx::mma_commit(empty(s));
                ptx::mma_commit(afree(ab));
            }
            ptx::mma_commit(accf);
            ptx::mma_commit(drain);
            ptx::mbar_wait(drain, 0, kDrainLimit, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ decoders, then epilogue
        // Set `set` decodes K blocks it = (kDecSets * m + set) * kDecBatch + u;
        // within a set, kDecBatch blocks share one wait for the tensor-memory
        // stores before they are handed to the MMA warp.
        const int set = (warp - 2) >> 2;
        const int quarter = warp & 3;  // tensor-memory lanes 32 * quarter ..
        const uint32_t tlane = (uint32_t)(quarter * 32) << 16;
        const int d = (threadIdx.x - 64) & 127;  // 0..127 within the set
        constexpr int kPer = 128 / NT;   // threads per token for sum(q)
        const int tok = d / kPer, part_i = d % kPer;
        if (set == 0 && d < bt) inv[d] = __frcp_rn(a.s[d]);
        const int row = quarter * 32 + lane;
        const int64_t o = (int64_t)mt * 128 + row;
        const float rs = a.splits == 1 && o < a.rows ? __ldg(a.rowscale + o) : 0.0f;
        int sqa = 0;
        bool ok = true;
        for (int it0 = set * kDecBatch; it0 < nj && ok; it0 += kDecSets * kDecBatch) {
            const int nd = min(kDecBatch, nj - it0);
            for (int u = 0; u < nd; u++) {
                const int it = it0 + u;
                const int s = it % S, ab = it % kNA;
                if (!warp_wait<false>(full(s), (it / S) & 1, limit, abort_flag) ||
                    (it >= kNA && !warp_wait<false>(afree(ab), ((it / kNA) - 1) & 1, limit, abort_flag))) {
                    if (lane == 0) give_up();
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const unsigned char *st = gbase + s * C::kStageBytes;
                const uint4 *cs = reinterpret_cast<const uint4 *>(st + C::kQBytes);
                const uint32_t acol = tmem + tlane + (uint32_t)(kAcol + 32 * ab);
                uint32_t v[16];
                decode_tile(cs[(2 * quarter) * 32 + lane], v);
                ptx::tmem_st_16x128b_x8(acol, v);
                decode_tile(cs[(2 * quarter + 1) * 32 + lane], v);
                ptx::tmem_st_16x128b_x8(acol + (16u << 16), v);
                // sum(q) of token `tok`: its 128-byte row of the stage (the
                // swizzle permutes 16-byte chunks within the row), NT bytes per
                // thread.
                const uint4 *qr = reinterpret_cast<const uint4 *>(st + tok * 128 + part_i * NT);
#pragma unroll
                for (int c = 0; c < NT / 16; c++) {
                    const uint4 qv = qr[c];
                    sqa = dp4a_ss((int)qv.x, 0x01010101, sqa);
                    sqa = dp4a_ss((int)qv.y, 0x01010101, sqa);
                    sqa = dp4a_ss((int)qv.z, 0x01010101, sqa);
                    sqa = dp4a_ss((int)qv.w, 0x01010101, sqa);
                }
            }
            if (!ok) break;
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int u = 0; u < nd; u++) ptx::mbar_arrive(decb((it0 + u) % kNA));
        }
        atomicAdd(sq + tok, sqa);
        asm volatile("bar.sync 1, %0;" ::"n"(128 * kDecSets) : "memory");  // sum(q), 1/s complete (decoders)
        if (set == 0) {  // the first set writes the results
            // The accumulator, 16 token columns at a time (thread = row):
            // sum t*q = sum c*q - sum q; then y (no split) or this CTA's partial
            // sums (the stages are free once every MMA has completed).
            const bool have = ok && warp_wait<true>(accf, 0, limit, abort_flag);
            if (ok && !have && lane == 0) give_up();
            if (have) ptx::tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < NT && c0 < bt; c0 += 16) {
                uint32_t v[16];
                if (have) {
                    ptx::tmem_ld_32x32b_x16(tmem + tlane + (uint32_t)c0, v);
                    ptx::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 16; i++) v[i] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const int b = c0 + i;
                    if (b >= bt) break;
                    const int val = (int)v[i] - sq[b];
                    if (a.splits == 1) {
                        if (o < a.rows) a.y[(int64_t)b * a.rows + o] = __fmul_rn(__fmul_rn(rs, (float)val), inv[b]);
                    } else {
                        part[row * C::kPartStride + b] = val;
                    }
                }
            }
        }
    }

    if (a.splits > 1) {
        // Every CTA's partial sums are in its shared memory; CTA r sums rows
        // [r R, r R + R) over the cluster (R = 128 / splits) and writes y.
        ptx::cluster_sync();
        if (warp >= 2 && warp < 6) {
            const int d = threadIdx.x - 64;
            const int R = 128 / a.splits;
            const int row = (int)rank * R + d % R;
            const int64_t o = (int64_t)mt * 128 + row;
            if (o < a.rows) {
                const float rs = __ldg(a.rowscale + o);
                const uint32_t loc = ptx::smem_u32(part + row * C::kPartStride);
                for (int b = d / R; b < bt; b += 128 / R) {
                    int v = 0;
                    for (int k = 0; k < a.splits; k++) v += ld_cluster_s32(ptx::map_to_rank(loc + 4u * b, (uint32_t)k));
                    a.y[(int64_t)b * a.rows + o] = __fmul_rn(__fmul_rn(rs, (float)v), inv[b]);
                }
            }
        }
        ptx::cluster_sync();  // no CTA leaves while another reads its partial sums
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
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

template <int NT>
cudaError_t run_tc(const void *data, const Layout &L, const int8_t *q, TcArgs a, cudaStream_t st) {
    using C = TcCfg<NT>;
    static std::atomic<bool> configured[64];
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap mc, mq;
    {
        const char *tiles = static_cast<const char *>(data) + L.off_tiles;
        cuuint64_t dims[3] = {128, (cuuint64_t)L.nb, (cuuint64_t)L.ntr};
        cuuint64_t strides[2] = {512, (cuuint64_t)L.nb * 512};
        cuuint32_t box[3] = {128, 1, 8};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<char *>(tiles), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)L.cols, (cuuint64_t)a.B};
        cuuint64_t strides[1] = {(cuuint64_t)L.cols};
        cuuint32_t box[2] = {128, (cuuint32_t)NT};
        cuuint32_t es[2] = {1, 1};
        if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(q), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    auto k = gemv_tc_kernel<NT>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    const int64_t mtiles = (L.rows + 127) / 128;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(mtiles * a.splits));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)a.splits;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k, mc, mq, a);
}

}  // namespace

bool gemv_tc_supported(int64_t rows, int64_t cols, int64_t B) {
    (void)rows;
    return B >= 1 && B <= 64 && cols >= kQK && cols <= (int64_t(1) << 17);
}

cudaError_t launch_gemv_tc(const void *data, int64_t rows, int64_t cols, const int8_t *q, const float *s,
                           int64_t B, float *y, const DeviceGlobals &g, cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    const unsigned char *base = static_cast<const unsigned char *>(data);
    TcArgs a;
    a.rowscale = reinterpret_cast<const float *>(base + L.off_rowscale);
    a.s = s;
    a.y = y;
    a.err = g.err;
    a.wait_limit = g.wait_limit;
    a.rows = rows;
    a.B = (int)B;
    a.nb = (int)L.nb;
    // K split over a cluster so that the grid fills two CTAs per SM in one
    // wave, keeping at least four K blocks per CTA.
    const int64_t mtiles = (rows + 127) / 128;
    int splits = 1;
    while (splits < 8 && a.nb / (splits * 2) >= 4 && mtiles * splits * 2 <= 2 * (int64_t)num_sms()) splits *= 2;
    a.splits = splits;
    if (B <= 16) return run_tc<16>(data, L, q, a, st);
    if (B <= 32) return run_tc<32>(data, L, q, a, st);
    return run_tc<64>(data, L, q, a, st);
}

}  // namespace bitnet
