// gemv_mma.cu -- small-batch W2A8 GEMV (8..64 tokens, uniform rows) on the
// warp-level int8 tensor-core MMA (mma.sync m16n8k32, u8 x s8 -> s32).
//
// y[b][o] = rowscale[o] * (sum_k t[o][k] * q[b][k]) * (1/s[b])  in fp32, the
// same three roundings as the batch-1 and batched decode kernels, so all of
// them give the same bits.  The integer product is that of the pages (+1 adds,
// -1 subtracts, 0 skips: "BitRun v0.2 实测：1-bit LLM 终端驾驶舱与毫瓦级功耗
// 遥测", section "三值权重与 1.58-bit 的由来"; 2-bit weights x 8-bit
// activations: "5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构对决",
// section "GPU内核突破").
//
// Why this MMA and not tcgen05 here.  With 8..64 tokens the product is a
// GEMV bound by the weight stream (2 bits a weight from HBM), and the tensor
// work is small: 16 tokens on 20480 x 3200 is 2.1 G int ops, under 2 us at
// the 1.1 POP/s measured for mma.sync m16n8k32 s8 on this GPU.  What decides
// the speed is the work per decoded weight.  A tcgen05.mma reads both
// operands from shared memory (or A from tensor memory), so the decoded
// weights take a store and a read through shared or tensor memory and every
// K block passes through mbarrier hand-offs between a decoder, a single MMA
// issuing thread (about 50 cycles of that thread per MMA, measured) and the
// producers; a tcgen05 version of this kernel measured 14.7 to 25 us for 16
// tokens on 20480 x 3200.  The warp-level MMA takes A from registers, and the
// repacked code tile is already in its A fragment layout: lane 4g+t of a
// 16-row tile holds bytes 4t..4t+3 of rows g (x) and g+8 (y) and bytes
// 16+4t.. of the same rows (z, w), and byte b of a 128-weight block holds
// weights b, b+32, b+64, b+96 at shifts 6, 4, 2, 0.  So ((x >> (6 - 2 grp))
// & 0x03030303, same for y, z, w) is exactly the A fragment (16 rows x 32 k)
// of the block's k slice grp, as unsigned codes c = t + 1: two operations per
// four weights, no shuffles, no shared memory.  sum t*q = sum c*q - sum q.
//
// Work layout: a CTA (4 warps) owns a 64-row M tile, one 16-row tile a warp,
// and a slice of the K blocks; the CTAs that split one M tile's K form a
// cluster (1..8) and sum their int32 partial sums through distributed shared
// memory (integer adds: the result does not depend on the split).  Each warp
// streams its tile's code words with 16-byte loads into registers, 4 to 8 K
// blocks ahead (the first ones before griddepcontrol.wait, since weights do
// not depend on the previous kernel).  The CTA gathers the activations of one
// chunk of K blocks at a time into shared memory in fragment order (lane
// 4g+t's eight words of a block and 8-token tile side by side, read with two
// conflict-free 16-byte loads) with 4-byte cp.async copies, three chunks
// ahead.  sum q of each token over the CTA's K slice is taken with dp4a from
// the B fragments the warps load anyway, each (block, 8-token tile) by one
// warp.  The only waits are CTA and cluster barriers.  A grid that fits in
// three CTAs per SM asks for enough shared memory that no SM holds a fourth:
// under programmatic dependent launch the CTAs start on the SMs the previous
// kernel leaves first, and without the cap they piled up four to an SM while
// other SMs stayed empty (16 tokens on 20480 x 3200: 13.8 -> 12.3 us; with the
// code-word registers used in rotating groups rather than shifted: 11.4 us).
// (A version that streamed the code words through per-warp bulk-copy rings in
// shared memory measured the same to 50% slower, depending on the shape.)
#include <atomic>

#include "common.cuh"
#include "tcgen05.cuh"

namespace bitnet {
namespace {

constexpr int kWarps = 4;  // 16-row tiles per CTA (a 64-row M tile)
constexpr int kThreads = 32 * kWarps;

template <int NT>
struct MmaCfg {
    static constexpr int kNTL = NT / 8;                    // 8-token tiles
    static constexpr int kCH = 64 / NT;                    // K blocks per activation chunk (8 KB)
    static constexpr int kPre = NT == 64 ? 4 : 8;          // K blocks of code words a warp holds
    static constexpr int kChunkBytes = kCH * kNTL * 1024;  // [block][ntile][half][lane][16 B]
    static constexpr int kQD = 4;                          // chunk buffers: copies run kQD - 1 chunks ahead
    static constexpr int kOffInv = kQD * kChunkBytes;      // the chunk buffers, then 1/s, sum q
    static constexpr int kOffSq = kOffInv + NT * 4;
    static constexpr size_t kSmem = (size_t)kOffSq + NT * 4;
    static constexpr int kPartStride = NT + 1;  // int32 partial sums [64][NT + 1] over the chunk buffers
    static_assert(64 * kPartStride * 4 <= kQD * kChunkBytes, "partial sums fit in the chunk buffers");
    static_assert(kSmem <= 56 * 1024, "four CTAs per SM");
};

struct MmaArgs {
    const uint4 *tiles;     // [ntr][nb][32 lanes] 16-byte code words
    const float *rowscale;  // [ntr * 16]
    const int8_t *q;        // [B][cols]
    const float *s;         // [B]
    float *y;               // [B][rows]
    int64_t rows, cols, ntr;
    int B, nb, splits;
};

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// Code words are read once: no L1 allocation, first out of L2.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p, uint64_t policy) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Gathers the activations of a chunk into buffer `buf` in fragment order.
// Region (block i, 8-token tile nt, half hf) of a chunk holds 128 words:
// word 4L + pos is lane L = 4g + t's B fragment register hb = pos & 1 of k
// slice grp = 2 hf + (pos >> 1), i.e. q[8 nt + g][128 j + 32 grp + 16 hb + 4t
// .. + 3].  Thread `tid` copies word `tid` of every region (consecutive
// threads, consecutive words: no bank conflicts); its source rows are fixed,
// so their addresses are set up once (`Gather`).  Token rows past B are never
// copied; the buffers are zeroed once.
template <int NT>
struct Gather {
    using C = MmaCfg<NT>;
    const int8_t *src[C::kNTL];  // this thread's word of block 0, per 8-token tile (null past B)
    __device__ __forceinline__ Gather(const MmaArgs &a, int j0, int tid) {
        const int L = tid >> 2, pos = tid & 3, g = L >> 2, t = L & 3;
        const int off = 128 * j0 + 32 * (pos >> 1) + 16 * (pos & 1) + 4 * t;
#pragma unroll
        for (int nt = 0; nt < C::kNTL; nt++) {
            const int n = 8 * nt + g;
            src[nt] = n < a.B ? a.q + (int64_t)n * a.cols + off : nullptr;
        }
    }
    // Blocks chunk * kCH .. of the CTA's K slice (those below nj) into `buf`.
    __device__ __forceinline__ void chunk(uint32_t buf, int nj, int chunk, int tid) const {
#pragma unroll
        for (int i = 0; i < C::kCH; i++) {
            const int jj = chunk * C::kCH + i;
            if (jj >= nj) break;
#pragma unroll
            for (int nt = 0; nt < C::kNTL; nt++) {
                if (src[nt]) {
                    const uint32_t dst = buf + (uint32_t)(((i * C::kNTL + nt) * 2) * 512 + 4 * tid);
                    const int8_t *sp = src[nt] + 128 * jj;
                    cp_async4(dst, sp);             // half 0: k slices 0, 1
                    cp_async4(dst + 512, sp + 64);  // half 1: k slices 2, 3
                }
            }
        }
    }
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 4) gemv_mma_kernel(const MmaArgs a) {
    using C = MmaCfg<NT>;
    constexpr int NTL = C::kNTL, CH = C::kCH;
    extern __shared__ __align__(128) unsigned char smem[];
    float *inv = reinterpret_cast<float *>(smem + C::kOffInv);
    int *sq = reinterpret_cast<int *>(smem + C::kOffSq);
    int *part = reinterpret_cast<int *>(smem);  // [64][kPartStride], after the main loop
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t rank = a.splits > 1 ? ptx::cluster_rank() : 0u;
    const int mt = (int)(blockIdx.x / (unsigned)a.splits);
    const int j0 = (int)((int64_t)rank * a.nb / a.splits);
    const int nj = (int)((int64_t)(rank + 1) * a.nb / a.splits) - j0;
    const int64_t tile = (int64_t)mt * kWarps + warp;
    const bool has_tile = tile < a.ntr;
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint4 *cw = a.tiles + ((has_tile ? tile : 0) * a.nb + j0) * 32 + lane;
    const uint64_t policy = ptx::policy_evict_first();

    // The first code words: weights do not depend on the previous kernel.
    constexpr int PRE = C::kPre;
    static_assert(PRE % CH == 0, "code words are held in whole chunks");
    uint4 pre[PRE];
#pragma unroll
    for (int i = 0; i < PRE; i++)
        pre[i] = has_tile && i < nj ? ld_stream(cw + (int64_t)i * 32, policy) : make_uint4(0, 0, 0, 0);
    // The rest of this warp's code words (one contiguous range of its tile)
    // into L2 now: the register loads above keep only 4..8 K blocks in flight.
    if (has_tile && lane == 0 && nj > PRE)
        prefetch_l2_bulk(cw - lane + (int64_t)PRE * 32, (uint32_t)(nj - PRE) * kTileBytes);
    if (a.B < NT) {  // token rows past B stay zero in every activation buffer
        for (int i = threadIdx.x; i < C::kQD * C::kChunkBytes / 16; i += kThreads)
            reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // q, s ready; y free
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (threadIdx.x < NT) {
        inv[threadIdx.x] = threadIdx.x < a.B ? __frcp_rn(a.s[threadIdx.x]) : 0.0f;
        sq[threadIdx.x] = 0;
    }
    __syncthreads();  // the zero fill lands before the gathers
    const int nch = (nj + CH - 1) / CH;
    const Gather<NT> gather(a, j0, threadIdx.x);
    // One cp.async group per activation chunk (empty past the last), kQD - 1 in flight.
#pragma unroll
    for (int c = 0; c < C::kQD - 1; c++) {
        if (c < nch) gather.chunk(sbase + (uint32_t)(c * C::kChunkBytes), nj, c, threadIdx.x);
        cp_async_commit();
    }
    cp_async_wait<C::kQD - 2>();  // chunk 0 landed (this thread's copies)
    __syncthreads();

    // AS accumulator sets (k slice grp goes to set grp % AS): eight
    // independent MMA chains per warp whatever the token count, so the MMA
    // latency is covered; summed after the loop.
    constexpr int AS = 4 / (NTL < 4 ? NTL : 4) ;
    int acc[AS][NTL][4], sqp[NTL];
#pragma unroll
    for (int n = 0; n < NTL; n++) {
        sqp[n] = 0;
#pragma unroll
        for (int u = 0; u < AS; u++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[u][n][i] = 0;
    }

    // The code words of chunk c sit in register group c % M (M = PRE / CH);
    // once used, the group is refilled with chunk c + M.  Unrolled over the
    // groups so that no word moves between registers.
    constexpr int M = PRE / CH;
#pragma unroll 1
    for (int c0 = 0; c0 < nch; c0 += M) {
#pragma unroll
        for (int u = 0; u < M; u++) {
            const int c = c0 + u;
            if (c >= nch) break;
            const int cn = c + C::kQD - 1;
            if (cn < nch) gather.chunk(sbase + (uint32_t)((cn % C::kQD) * C::kChunkBytes), nj, cn, threadIdx.x);
            cp_async_commit();
            const uint4 *qb = reinterpret_cast<const uint4 *>(smem + (c % C::kQD) * C::kChunkBytes) + lane;
#pragma unroll
            for (int i = 0; i < CH; i++) {
                if (c * CH + i < nj) {
                    const uint4 w = pre[u * CH + i];
#pragma unroll
                    for (int nt = 0; nt < NTL; nt++) {
                        const uint4 h0 = qb[((i * NTL + nt) * 2 + 0) * 32];
                        const uint4 h1 = qb[((i * NTL + nt) * 2 + 1) * 32];
                        if (has_tile && AS == 4) {
                            // One set per k slice: the codes are masked in place
                            // (bytes c * 4^(3 - grp) <= 128) and each set's sum is
                            // shifted back after the loop, exactly.
                            mma_u8s8(acc[0][nt], w.x & 0xC0C0C0C0u, w.y & 0xC0C0C0C0u, w.z & 0xC0C0C0C0u,
                                     w.w & 0xC0C0C0C0u, h0.x, h0.y);
                            mma_u8s8(acc[1 % AS][nt], w.x & 0x30303030u, w.y & 0x30303030u, w.z & 0x30303030u,
                                     w.w & 0x30303030u, h0.z, h0.w);
                            mma_u8s8(acc[2 % AS][nt], w.x & 0x0C0C0C0Cu, w.y & 0x0C0C0C0Cu, w.z & 0x0C0C0C0Cu,
                                     w.w & 0x0C0C0C0Cu, h1.x, h1.y);
                            mma_u8s8(acc[3 % AS][nt], w.x & 0x03030303u, w.y & 0x03030303u, w.z & 0x03030303u,
                                     w.w & 0x03030303u, h1.z, h1.w);
                        } else if (has_tile) {
                            mma_u8s8(acc[0][nt], (w.x >> 6) & 0x03030303u, (w.y >> 6) & 0x03030303u,
                                     (w.z >> 6) & 0x03030303u, (w.w >> 6) & 0x03030303u, h0.x, h0.y);
                            mma_u8s8(acc[1 % AS][nt], (w.x >> 4) & 0x03030303u, (w.y >> 4) & 0x03030303u,
                                     (w.z >> 4) & 0x03030303u, (w.w >> 4) & 0x03030303u, h0.z, h0.w);
                            mma_u8s8(acc[2 % AS][nt], (w.x >> 2) & 0x03030303u, (w.y >> 2) & 0x03030303u,
                                     (w.z >> 2) & 0x03030303u, (w.w >> 2) & 0x03030303u, h1.x, h1.y);
                            mma_u8s8(acc[3 % AS][nt], w.x & 0x03030303u, w.y & 0x03030303u, w.z & 0x03030303u,
                                     w.w & 0x03030303u, h1.z, h1.w);
                        }
                        if ((i * NTL + nt) % kWarps == warp) {  // this warp's share of sum q
                            int v = __dp4a((int)h0.x, 0x01010101, sqp[nt]);
                            v = __dp4a((int)h0.y, 0x01010101, v);
                            v = __dp4a((int)h0.z, 0x01010101, v);
                            v = __dp4a((int)h0.w, 0x01010101, v);
                            v = __dp4a((int)h1.x, 0x01010101, v);
                            v = __dp4a((int)h1.y, 0x01010101, v);
                            v = __dp4a((int)h1.z, 0x01010101, v);
                            sqp[nt] = __dp4a((int)h1.w, 0x01010101, v);
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < CH; i++) {
                const int jj = (c + M) * CH + i;
                pre[u * CH + i] =
                    has_tile && jj < nj ? ld_stream(cw + (int64_t)jj * 32, policy) : make_uint4(0, 0, 0, 0);
            }
            cp_async_wait<C::kQD - 2>();  // chunk c + 1 landed
            __syncthreads();
        }
    }
    cp_async_wait<0>();
    if (AS == 4) {  // undo the in-place scaling of the k slices' codes (exact shifts)
#pragma unroll
        for (int n = 0; n < NTL; n++)
#pragma unroll
            for (int i = 0; i < 4; i++) {
                acc[0][n][i] >>= 6;
                acc[1 % AS][n][i] >>= 4;
                acc[2 % AS][n][i] >>= 2;
            }
    }
#pragma unroll
    for (int u = 1; u < AS; u++)
#pragma unroll
        for (int n = 0; n < NTL; n++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[0][n][i] += acc[u][n][i];
    // Lane 4g+t holds part of token 8 nt + g's sum q.
#pragma unroll
    for (int nt = 0; nt < NTL; nt++) {
        int v = sqp[nt];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if (t == 0 && v != 0) atomicAdd(sq + 8 * nt + g, v);
    }
    __syncthreads();

    // acc[0][nt][e]: row g (e < 2) or g + 8 of the warp's tile, token
    // 8 nt + 2t + (e & 1); sum t*q = sum c*q - sum q.
    const int64_t o0 = tile * 16 + g, o1 = o0 + 8;
    if (a.splits == 1) {
        if (has_tile) {
            const float rs0 = o0 < a.rows ? __ldg(a.rowscale + o0) : 0.0f;
            const float rs1 = o1 < a.rows ? __ldg(a.rowscale + o1) : 0.0f;
#pragma unroll
            for (int nt = 0; nt < NTL; nt++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int b = 8 * nt + 2 * t + (e & 1);
                    const int64_t o = e < 2 ? o0 : o1;
                    if (b < a.B && o < a.rows) {
                        const int val = acc[0][nt][e] - sq[b];
                        a.y[(int64_t)b * a.rows + o] = __fmul_rn(__fmul_rn(e < 2 ? rs0 : rs1, (float)val), inv[b]);
                    }
                }
        }
    } else {
        // Partial sums into this CTA's shared memory (the chunk buffers are
        // free after the loop's last barrier); CTA r of the cluster then sums
        // rows [r R, r R + R) over the cluster (R = 64 / splits) and writes y.
#pragma unroll
        for (int nt = 0; nt < NTL; nt++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int b = 8 * nt + 2 * t + (e & 1);
                const int r = warp * 16 + g + (e < 2 ? 0 : 8);
                if (b < NT) part[r * C::kPartStride + b] = acc[0][nt][e] - sq[b];
            }
        ptx::cluster_sync();
        const int R = 64 / a.splits;
        const int row = (int)rank * R + threadIdx.x % R;
        const int64_t o = (int64_t)mt * 64 + row;
        if (o < a.rows) {
            const float rs = __ldg(a.rowscale + o);
            const uint32_t loc = ptx::smem_u32(part + row * C::kPartStride);
            for (int b = threadIdx.x / R; b < a.B; b += kThreads / R) {
                int v = 0;
                for (int k = 0; k < a.splits; k++) v += ld_cluster_s32(ptx::map_to_rank(loc + 4u * b, (uint32_t)k));
                a.y[(int64_t)b * a.rows + o] = __fmul_rn(__fmul_rn(rs, (float)v), inv[b]);
            }
        }
        ptx::cluster_sync();  // no CTA leaves while another reads its partial sums
    }
}

template <int NT>
cudaError_t run_mma(const MmaArgs &a, int64_t mtiles, cudaStream_t st) {
    using C = MmaCfg<NT>;
    static std::atomic<bool> configured[64];
    auto k = gemv_mma_kernel<NT>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 60 * 1024);
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(mtiles * a.splits));
    cfg.blockDim = dim3(kThreads);
    // A grid that fits in three CTAs per SM asks for enough shared memory
    // that no SM takes a fourth: when the previous kernel's CTAs leave the
    // SMs one by one, this spreads the CTAs over more SMs.
    cfg.dynamicSmemBytes = mtiles * a.splits <= 3 * (int64_t)num_sms() ? 60 * 1024 : C::kSmem;
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
    return cudaLaunchKernelEx(&cfg, k, a);
}

}  // namespace

bool gemv_mma_supported(int64_t rows, int64_t cols, int64_t B) {
    (void)rows;
    return B >= 1 && B <= 64 && cols >= kQK && cols <= (int64_t(1) << 17);
}

cudaError_t launch_gemv_mma(const void *data, int64_t rows, int64_t cols, const int8_t *q, const float *s, int64_t B,
                            float *y, cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    const unsigned char *base = static_cast<const unsigned char *>(data);
    MmaArgs a;
    a.tiles = reinterpret_cast<const uint4 *>(base + L.off_tiles);
    a.rowscale = reinterpret_cast<const float *>(base + L.off_rowscale);
    a.q = q;
    a.s = s;
    a.y = y;
    a.rows = rows;
    a.cols = cols;
    a.ntr = L.ntr;
    a.B = (int)B;
    a.nb = (int)L.nb;
    // K split over a cluster while the grid stays within one wave of four
    // CTAs per SM and every CTA keeps at least four K blocks.
    const int64_t mtiles = (L.ntr + kWarps - 1) / kWarps;
    int splits = 1;
    while (splits < 8 && a.nb / (splits * 2) >= 4 && mtiles * splits * 2 <= 4 * (int64_t)num_sms()) splits *= 2;
    a.splits = splits;
    if (B <= 16) return run_mma<16>(a, mtiles, st);
    if (B <= 32) return run_mma<32>(a, mtiles, st);
    return run_mma<64>(a, mtiles, st);
}

}  // namespace bitnet
