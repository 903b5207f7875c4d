// decode.cu -- batch-1 W2A8 linear for uniform rows (the per-tensor absmean
// case): the latency-critical call of token-by-token generation.
//
// y[o] = rowscale[o] * (sum_k t[o][k] * q[k]) / s,   q = per-token absmax int8
// activations ("5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构对决", section
// "GPU内核突破": 2-bit weights x 8-bit activations with dp4a).  The pages do not
// print the activation formula; the library reads it as s = 127 / max(absmax,
// 1e-5) and q = rint(x * s), ties to even (one fp32 multiply), the reading the
// quantiser documents.  q and the integer sums are exactly those of the general
// kernel; the epilogue runs in fp32 (below).
//
// A decode step is a chain of dependent linears of a few microseconds each, so
// what costs is the chain's latency: the time from the previous kernel's end
// to this kernel's last store.  Measured on B200, the pieces of that are the
// release of griddepcontrol.wait (~0.6 us after the previous grid ends), one
// L2 round trip for x, two CTA barriers around the activation quantisation,
// the dp4a work (ALU-pipe bound: one LOP3 mask and one IDP4A per four
// weights) and the epilogue.  Hence:
//
//  * one CTA of 16 warps per SM, at most half of the SM's registers, so the
//    next linear's CTA is resident beside this one (programmatic dependent
//    launch) and fetches its weights before its griddepcontrol.wait;
//  * the weights move by bulk copies (cp.async.bulk, one per two 512-byte
//    tiles, L2 evict-first: read once per step, they must not push the
//    activations out of L2) into shared memory, up to eight tiles per warp;
//    register loads could not keep enough bytes in flight per SM;
//  * the copies are waited for before griddepcontrol.wait, where the wait is
//    free; larger slices stream through the same slots after it;
//  * every shared-memory carveout request is the same (max shared), so CTAs
//    of consecutive linears share an SM without it being reconfigured;
//  * a CTA owns whole row tiles (no cross-CTA reduction) and its warps split
//    the (tile, block) items evenly in memory order, so a warp's tiles are one
//    contiguous range; index state is set up before the wait;
//  * after the wait: x is read once into registers, the absmax is combined
//    across warps through shared memory (barrier 1), x is quantised into
//    shared memory in the order the lanes read it (a lane's eight words of a
//    block are 32 contiguous bytes) and sum(q) is taken once per CTA
//    (barrier 2); the products run per row-tile run without per-item
//    branches, one shared-memory atomic per row and run; barrier 3, epilogue;
//  * the epilogue is fp32: rowscale * sum * (1/s), three roundings, relative
//    error below 2.4e-7 of the fp64 value (the fp64 product, divide and
//    conversions cost ~0.25 us per call on this path).
// Integer sums are exact, so the atomics leave the result independent of
// their order.  Every wait on a copy is bounded; on a timeout the kernel sets
// the device error word, waits (bounded) for its copies in flight and returns.
//
// Two more kernels share the weight ring (WeightRing below): the batched
// kernel for 2..16 tokens (decode_bn_kernel) and a table-lookup variant for
// comparison (decode_lut_kernel).
#include <atomic>

#include "common.cuh"
#include "dp4a.cuh"
#include "tcgen05.cuh"

namespace bitnet {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 2;     // tiles per bulk copy
constexpr int kMaxSlots = 4;  // copies in flight per warp
constexpr int kTile = kTileBytes;
constexpr uint32_t kDrainLimit = 1u << 26;  // tries while waiting out a copy after a timeout

struct DecArgs {
    const unsigned char *tiles;
    const float *rowscale;
    const int8_t *q;   // [K] (unfused)
    const float *s;    // [1] (unfused)
    const float *x;    // [K] fp32 (fused)
    int8_t *q_out;     // nullable (fused): written by CTA 0
    float *s_out;      // nullable (fused): written by CTA 0
    float *y;
    unsigned *err;
    const unsigned *wait_limit;
    int64_t rows;
    int K;
    int nb;
    int tiles_lo;  // every CTA owns tiles_lo or tiles_lo + 1 row tiles
    int extra;     // the first `extra` CTAs own tiles_lo + 1
    int wcap;      // tiles of shared memory per warp: kChunk * (copies in flight), a power of two
    uint32_t off_q, off_acc, off_rsc, off_red, off_bar;
    int B;         // tokens (batched kernel)
};

// One warp's share of a CTA's (row tile, block) items and the ring of
// shared-memory slots its tiles move through.  Items run in memory order:
// item i is row tile i / nb, block i % nb, 512-byte tile (r0 * nb + i).
struct WeightRing {
    int64_t r0;                // first row tile of the CTA
    int nr, n;                 // row tiles and items of the CTA
    int i0, nit;               // this warp's items
    int wcap, nslots, nchunks; // slots (a power of two, in tiles), copies of kChunk tiles
    unsigned char *wsm;        // this warp's slots
    uint32_t bars, rbar;       // this warp's slot barriers, the row-scale barrier
    const unsigned char *src;  // this warp's first tile
    uint64_t pol;

    __device__ __forceinline__ void init(const DecArgs &a, unsigned char *smem, int warp) {
        const int c = blockIdx.x;
        r0 = (int64_t)c * a.tiles_lo + min(c, a.extra);
        nr = a.tiles_lo + (c < a.extra ? 1 : 0);
        n = nr * a.nb;
        i0 = (int)(((int64_t)warp * n) / kWarps);
        nit = (int)(((int64_t)(warp + 1) * n) / kWarps) - i0;
        wcap = a.wcap;
        nslots = wcap / kChunk;
        nchunks = (nit + kChunk - 1) / kChunk;
        wsm = smem + (size_t)warp * wcap * kTile;
        bars = ptx::smem_u32(smem + a.off_bar) + 8u * (warp * kMaxSlots);
        rbar = ptx::smem_u32(smem + a.off_bar) + 8u * (kWarps * kMaxSlots);
        src = a.tiles + (size_t)(r0 * a.nb + i0) * kTile;
        pol = ptx::policy_evict_first();
    }
    // Lane 0: chunk k of this warp's tiles into slot k % nslots.
    __device__ __forceinline__ void issue(int k) const {
        const int s = k & (nslots - 1);
        const uint32_t bytes = (uint32_t)min(kChunk, nit - k * kChunk) * kTile;
        ptx::mbar_arrive_expect_tx(bars + 8u * s, bytes);
        ptx::bulk_g2s(ptx::smem_u32(wsm + s * kChunk * kTile), src + (size_t)k * kChunk * kTile, bytes,
                      bars + 8u * s, pol);
    }
    __device__ __forceinline__ int npre() const { return nchunks < nslots ? nchunks : nslots; }
    // Lane 0 of every warp: barriers, the first nslots copies, and (warp 0) the
    // CTA's row scales into rsc.
    __device__ __forceinline__ void start(const DecArgs &a, float *rsc, int warp) const {
        for (int s = 0; s < nslots; s++) ptx::mbar_init(bars + 8u * s, 1);
        if (warp == 0) ptx::mbar_init(rbar, 1);
        ptx::fence_mbar_init();
        for (int k = 0; k < npre(); k++) issue(k);
        if (warp == 0) {
            const uint32_t bytes = (uint32_t)nr * kTileRows * sizeof(float);
            ptx::mbar_arrive_expect_tx(rbar, bytes);
            ptx::bulk_g2s(ptx::smem_u32(rsc), a.rowscale + r0 * kTileRows, bytes, rbar, pol);
        }
    }
    // Lanes 0..15 of warp 0 wait for warp lane's first copies, lane 16 for the
    // row scales, sleeping between polls while the other warps block in the
    // barrier that follows (they take no issue slots from the kernel sharing
    // the SM).  A wait that runs out sets *bad.  Call only after a CTA barrier
    // that follows every warp's start(): the barriers polled here belong to
    // other warps.
    __device__ __forceinline__ void wait_started(const DecArgs &a, unsigned char *smem, int *bad, uint32_t limit,
                                                 int warp, int lane) const {
        if (warp != 0 || lane > kWarps) return;
        bool good;
        if (lane < kWarps) {
            const int wn = (int)(((int64_t)(lane + 1) * n) / kWarps) - (int)(((int64_t)lane * n) / kWarps);
            const int wc = (wn + kChunk - 1) / kChunk;
            const int wpre = wc < nslots ? wc : nslots;
            const uint32_t wb = ptx::smem_u32(smem + a.off_bar) + 8u * (lane * kMaxSlots);
            good = true;
            for (int k = 0; k < wpre && good; k++) good = ptx::mbar_wait_sleep(wb + 8u * k, 0u, limit, nullptr, 128);
        } else {
            good = ptx::mbar_wait_sleep(rbar, 0u, limit, nullptr, 128);
        }
        if (!good) *bad = 1;
    }
    // Runs item(w, j) over the warp's items (w = this lane's 16 bytes of the
    // tile, j = its block) and flush(r) whenever the row tile r ends or the
    // items run out.  Copies past the first nslots are waited for here and
    // refilled as slots free up.  On a timeout: error bit, bounded drain of the
    // warp's copies in flight, and ok = false.
    template <class Item, class Flush>
    __device__ __forceinline__ void run(const DecArgs &a, bool &ok, uint32_t limit, int warp, int lane, Item item,
                                        Flush flush) const {
        int r = i0 / a.nb, j = i0 - r * a.nb, it = 0;
        const uint4 *wl = reinterpret_cast<const uint4 *>(wsm) + lane;
        if (nit <= wcap) {
            // Every tile is in shared memory already: runs within one row tile.
            while (it < nit && ok) {
                const int len = min(nit - it, a.nb - j);
                const uint4 *wv = wl + it * 32;
#pragma unroll 2
                for (int e = 0; e < len; e++) item(wv[e * 32], j + e);
                it += len;
                j += len;
                if (j == a.nb) {
                    flush(r);
                    r++;
                    j = 0;
                }
            }
        } else {
            for (; it < nit && ok; it++) {
                if (it >= wcap && (it & (kChunk - 1)) == 0) {
                    const int k = it / kChunk;
                    int got = 0;
                    if (lane == 0)
                        got = ptx::mbar_wait(bars + 8u * (k & (nslots - 1)), (uint32_t)(k / nslots) & 1u, limit,
                                             nullptr) ? 1 : 0;
                    if (!__shfl_sync(0xffffffffu, got, 0)) {
                        ok = false;
                        break;
                    }
                }
                item(wl[(it & (wcap - 1)) * 32], j);
                if (++j == a.nb) {
                    flush(r);
                    r++;
                    j = 0;
                }
                if ((it & (kChunk - 1)) == kChunk - 1 && it / kChunk + nslots < nchunks) {
                    __syncwarp();  // every lane has read the chunk's slot
                    if (lane == 0) {
                        ptx::fence_proxy_async_smem();
                        issue(it / kChunk + nslots);
                    }
                }
            }
        }
        if (!ok) {
            // Timed out: record it, then wait out this warp's copies in flight
            // (chunks it / kChunk .. the last one issued).
            if (lane == 0) {
                atomicOr(a.err, kErrTimeout);
                const int k0 = it / kChunk;
                for (int k = k0; k < nchunks && k < k0 + nslots; k++)
                    ptx::mbar_wait(bars + 8u * (k & (nslots - 1)), (uint32_t)(k / nslots) & 1u, kDrainLimit,
                                   nullptr);
                if (warp == 0) ptx::mbar_wait(rbar, 0u, kDrainLimit, nullptr);
            }
            __syncwarp();
        }
        if (j != 0) flush(r);  // items since the last tile change (none if j == 0)
    }
};

// The batch-1 kernel inlines the weight ring's steps (the compiler keeps fewer
// values live across the products that way: measured 2% faster per step).
template <bool FUSED, int NX>
__global__ void __launch_bounds__(kThreads, 2) decode_b1_kernel(const DecArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int c = blockIdx.x;
    const int64_t r0 = (int64_t)c * a.tiles_lo + min(c, a.extra);
    const int nr = a.tiles_lo + (c < a.extra ? 1 : 0);
    const int n = nr * a.nb;
    const int i0 = (int)(((int64_t)warp * n) / kWarps);
    const int nit = (int)(((int64_t)(warp + 1) * n) / kWarps) - i0;
    const int wcap = a.wcap;  // a power of two, kChunk .. kChunk * kMaxSlots
    const int nslots = wcap / kChunk;
    const int nchunks = (nit + kChunk - 1) / kChunk;
    unsigned char *wsm = smem + (size_t)warp * wcap * kTile;
    uint32_t *qw = reinterpret_cast<uint32_t *>(smem + a.off_q);
    int *acc = reinterpret_cast<int *>(smem + a.off_acc);
    float *rsc = reinterpret_cast<float *>(smem + a.off_rsc);
    unsigned *amax_w = reinterpret_cast<unsigned *>(smem + a.off_red);  // absmax bits (atomic max)
    int *qsum_w = reinterpret_cast<int *>(smem + a.off_red + 4);          // sum(q) (atomic add)
    int *bad_w = reinterpret_cast<int *>(smem + a.off_red + 8);           // a copy wait ran out
    const uint32_t bars = ptx::smem_u32(smem + a.off_bar) + 8u * (warp * kMaxSlots);
    const uint32_t rbar = ptx::smem_u32(smem + a.off_bar) + 8u * (kWarps * kMaxSlots);
    const unsigned char *src = a.tiles + (size_t)(r0 * a.nb + i0) * kTile;
    const uint32_t limit = *a.wait_limit;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- before the wait: nothing here depends on the previous kernel.
    const uint64_t pol = ptx::policy_evict_first();
    auto issue = [&](int k) {  // lane 0: chunk k of this warp's tiles into its slot
        const int s = k & (nslots - 1);
        const uint32_t bytes = (uint32_t)min(kChunk, nit - k * kChunk) * kTile;
        ptx::mbar_arrive_expect_tx(bars + 8u * s, bytes);
        ptx::bulk_g2s(ptx::smem_u32(wsm + s * kChunk * kTile), src + (size_t)k * kChunk * kTile, bytes,
                      bars + 8u * s, pol);
    };
    const int npre = nchunks < nslots ? nchunks : nslots;
    if (lane == 0) {
        for (int s = 0; s < nslots; s++) ptx::mbar_init(bars + 8u * s, 1);
        if (warp == 0) ptx::mbar_init(rbar, 1);
        ptx::fence_mbar_init();
        for (int k = 0; k < npre; k++) issue(k);
        if (warp == 0) {
            const uint32_t bytes = (uint32_t)nr * kTileRows * sizeof(float);
            ptx::mbar_arrive_expect_tx(rbar, bytes);
            ptx::bulk_g2s(ptx::smem_u32(rsc), a.rowscale + r0 * kTileRows, bytes, rbar, pol);
        }
    }
    for (int i = tid; i < nr * kTileRows; i += kThreads) acc[i] = 0;
    if (tid == 0) {
        *amax_w = 0u;
        *qsum_w = 0;
        *bad_w = 0;
    }
    // Index state of the product loop, set up here, off the critical path.
    const int r = i0 / a.nb;
    int j = i0 - r * a.nb;
    int *accp = acc + r * kTileRows + g;  // rows g and g + 8 of the current tile
    const uint4 *qrow = reinterpret_cast<const uint4 *>(qw + t * 8);  // block 0, this lane's part
    const uint4 *qp = qrow + j * 8;
    const uint4 *wl = reinterpret_cast<const uint4 *>(wsm) + lane;
    // Wait for the copies issued above while the previous kernel still runs
    // (a wait is cheap here and costly after griddepcontrol.wait).  Lanes 0..15
    // of warp 0 poll warp lane's copies, lane 16 the row scales, sleeping
    // between tries; the other warps block in the barrier and take no issue
    // slots from the kernel that shares the SM.  The barrier first: every
    // warp's lane 0 has initialised its slot barriers (and issued its copies)
    // before warp 0 polls them -- shared memory left by an earlier CTA could
    // otherwise look like a completed phase -- and bad_w is zero.
    __syncthreads();
    if (warp == 0 && lane <= kWarps) {
        bool good = true;
        if (lane < kWarps) {
            const int wn = (int)(((int64_t)(lane + 1) * n) / kWarps) - (int)(((int64_t)lane * n) / kWarps);
            const int wc = (wn + kChunk - 1) / kChunk;
            const int wpre = wc < nslots ? wc : nslots;
            const uint32_t wb = ptx::smem_u32(smem + a.off_bar) + 8u * (lane * kMaxSlots);
            for (int k = 0; k < wpre && good; k++) good = ptx::mbar_wait_sleep(wb + 8u * k, 0u, limit, nullptr, 128);
        } else {
            good = ptx::mbar_wait_sleep(rbar, 0u, limit, nullptr, 128);
        }
        if (!good) *bad_w = 1;
    }
    __syncthreads();  // copies landed (or bad_w set); acc and the reduction words are zero
    bool ok = *bad_w == 0;

    asm volatile("griddepcontrol.wait;" ::: "memory");  // x (or q, s) ready; y free

    // ---- activations: s, q (permuted) in shared memory, sum(q).
    const int K4 = a.K >> 2;
    float s, inv_s;
    int qsum = 0;
    if constexpr (FUSED) {
        const float4 *x4 = reinterpret_cast<const float4 *>(a.x);
        float4 xv[NX];
        float m = 0.0f;
#pragma unroll
        for (int u = 0; u < NX; u++) {
            const int i = tid + u * kThreads;
            xv[u] = i < K4 ? x4[i] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            m = fmaxf(m, fmaxf(fmaxf(fabsf(xv[u].x), fabsf(xv[u].y)), fmaxf(fabsf(xv[u].z), fabsf(xv[u].w))));
        }
        // m >= 0 and not NaN (fmaxf drops NaN): its bit pattern orders like its value.
        const unsigned mu = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
        if (lane == 0) atomicMax(amax_w, mu);
        __syncthreads();
        const float amax = __uint_as_float(*amax_w);
        s = __fdiv_rn(127.0f, amax > kEps ? amax : kEps);
        inv_s = __frcp_rn(s);
        if (c == 0 && tid == 0 && a.s_out) a.s_out[0] = s;
        uint32_t *qo = (c == 0 && a.q_out) ? reinterpret_cast<uint32_t *>(a.q_out) : nullptr;
#pragma unroll
        for (int u = 0; u < NX; u++) {
            const int i = tid + u * kThreads;
            if (i < K4) {
                const uint32_t w = quant4_fast(xv[u], s);
                qw[perm_word(i)] = w;
                qsum = dp4a_ss((int)w, 0x01010101, qsum);
                if (qo) qo[i] = w;
            }
        }
    } else {
        s = *a.s;
        inv_s = __frcp_rn(s);
        const uint32_t *q4 = reinterpret_cast<const uint32_t *>(a.q);
        for (int i = tid; i < K4; i += kThreads) {
            const uint32_t w = q4[i];
            qw[perm_word(i)] = w;
            qsum = dp4a_ss((int)w, 0x01010101, qsum);
        }
    }
    qsum = __reduce_add_sync(0xffffffffu, qsum);
    if (lane == 0) atomicAdd(qsum_w, qsum);
    __syncthreads();

    // ---- products.  Items of this warp: i0 .. i0 + nit - 1 (tile r = i / nb,
    // block j = i % nb), item `it` in shared-memory slot it % wcap; the four
    // group sums of rows g and g + 8 are held until the tile changes.
    int aA[4] = {0, 0, 0, 0}, aB[4] = {0, 0, 0, 0};
    auto flush = [&]() {
        const int pA = tig_reduce(combine4(aA));
        const int pB = tig_reduce(combine4(aB));
        if (t == 0) {
            atomicAdd(accp, pA);
            atomicAdd(accp + 8, pB);
        }
#pragma unroll
        for (int k = 0; k < 4; k++) aA[k] = aB[k] = 0;
    };
    // The products of one item: tile word w (lane's 16 bytes), activation
    // words at qv (qa0 qb0 qa1 qb1 | qa2 qb2 qa3 qb3).
    auto item = [&](const uint4 w, const uint4 *qv) {
        const uint4 q0 = qv[0], q1 = qv[1];
        const int qa[4] = {(int)q0.x, (int)q0.z, (int)q1.x, (int)q1.z};
        const int qb[4] = {(int)q0.y, (int)q0.w, (int)q1.y, (int)q1.w};
#pragma unroll
        for (int gg = 0; gg < 4; gg++) {
            const uint32_t mk = 0xC0C0C0C0u >> (2 * gg);
            aA[gg] = dp4a_us(w.x & mk, qa[gg], aA[gg]);
            aA[gg] = dp4a_us(w.z & mk, qb[gg], aA[gg]);
            aB[gg] = dp4a_us(w.y & mk, qa[gg], aB[gg]);
            aB[gg] = dp4a_us(w.w & mk, qb[gg], aB[gg]);
        }
    };
    int it = 0;
    if (nit <= wcap) {
        // Every tile of the warp is already in shared memory: runs of items
        // within one row tile, one flush per run.
        while (it < nit && ok) {
            const int run = min(nit - it, a.nb - j);
            const uint4 *wv = wl + it * 32;
#pragma unroll 2
            for (int e = 0; e < run; e++) item(wv[e * 32], qp + e * 8);
            it += run;
            j += run;
            qp += run * 8;
            if (j == a.nb) {
                flush();
                accp += kTileRows;
                j = 0;
                qp = qrow;
            }
        }
    } else {
        // Streaming: item `it` sits in slot it % wcap; chunks from nslots on
        // are waited for here and refilled as their slots free up.
        for (; it < nit && ok; it++) {
            if (it >= wcap && (it & (kChunk - 1)) == 0) {
                const int k = it / kChunk;
                int got = 0;
                if (lane == 0)
                    got = ptx::mbar_wait(bars + 8u * (k & (nslots - 1)), (uint32_t)(k / nslots) & 1u, limit,
                                         nullptr) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
            }
            item(wl[(it & (wcap - 1)) * 32], qp);
            qp += 8;
            if (++j == a.nb) {
                flush();
                accp += kTileRows;
                j = 0;
                qp = qrow;
            }
            if ((it & (kChunk - 1)) == kChunk - 1 && it / kChunk + nslots < nchunks) {
                __syncwarp();  // every lane has read the chunk's slot
                if (lane == 0) {
                    ptx::fence_proxy_async_smem();
                    issue(it / kChunk + nslots);
                }
            }
        }
    }
    if (!ok) {
        // Timed out: record it, then wait out this warp's copies still in flight
        // (chunks it / kChunk .. the last one issued).
        if (lane == 0) {
            atomicOr(a.err, kErrTimeout);
            const int k0 = it / kChunk;
            for (int k = k0; k < nchunks && k < k0 + nslots; k++)
                ptx::mbar_wait(bars + 8u * (k & (nslots - 1)), (uint32_t)(k / nslots) & 1u, kDrainLimit, nullptr);
            if (warp == 0) ptx::mbar_wait(rbar, 0u, kDrainLimit, nullptr);
        }
        __syncwarp();
    }
    if (j != 0) flush();  // items since the last tile change (none if j == 0)
    __syncthreads();

    const int tot = *qsum_w;  // sum(q) over the row
    // ---- epilogue: y = rowscale * (sum c*q - sum q) * (1/s) in fp32: three
    // roundings, relative error below 2e-7 (the int sum is exact in fp32,
    // |sum| <= 127 * K < 2^22).  The general kernel keeps the fp64 epilogue.
    for (int i = tid; i < nr * kTileRows; i += kThreads) {
        const int64_t o = r0 * kTileRows + i;
        if (o < a.rows) a.y[o] = __fmul_rn(__fmul_rn(rsc[i], int_to_float(acc[i] - tot)), inv_s);
    }
}

// Batches of 2..16 tokens (q and s given, uniform rows): the same weight
// ring and launch shape; the codes of an item are shifted down once
// (unscaled c = t + 1 per byte) and reused for every token, each token's
// eight activation words of the block come from its own row of the permuted
// shared-memory copy of q, and the row sums of rows g and g + 8 are held per
// token until the row tile changes.
template <int BT>
__global__ void __launch_bounds__(kThreads, BT >= 8 ? 1 : 2) decode_bn_kernel(const DecArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    uint32_t *qw = reinterpret_cast<uint32_t *>(smem + a.off_q);             // [BT][K/4] permuted
    int *acc = reinterpret_cast<int *>(smem + a.off_acc);                     // [nr*16][BT]
    float *rsc = reinterpret_cast<float *>(smem + a.off_rsc);
    int *qsum_w = reinterpret_cast<int *>(smem + a.off_red);                  // [BT] sum(q) per token
    float *inv_w = reinterpret_cast<float *>(smem + a.off_red + 4 * BT);      // [BT] 1/s per token
    int *bad_w = reinterpret_cast<int *>(smem + a.off_red + 8 * BT);          // a copy wait ran out
    const uint32_t limit = *a.wait_limit;
    const int B = a.B;
    WeightRing ring;
    ring.init(a, smem, warp);

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (lane == 0) ring.start(a, rsc, warp);
    for (int i = tid; i < ring.nr * kTileRows * BT; i += kThreads) acc[i] = 0;
    if (tid < BT) qsum_w[tid] = 0;
    if (tid == 0) *bad_w = 0;
    __syncthreads();  // every warp's slot barriers are initialised before warp 0 polls them
    ring.wait_started(a, smem, bad_w, limit, warp, lane);
    __syncthreads();
    bool ok = *bad_w == 0;

    asm volatile("griddepcontrol.wait;" ::: "memory");  // q, s ready; y free

    // ---- q rows (zero rows past B), permuted, and sum(q) per token.
    const int K4 = a.K >> 2;
    const uint32_t *q4 = reinterpret_cast<const uint32_t *>(a.q);
    int qs[BT];
#pragma unroll
    for (int b = 0; b < BT; b++) qs[b] = 0;
    for (int m = tid; m < K4; m += kThreads) {  // all tokens' loads of a word index in flight together
        uint32_t w[BT];
#pragma unroll
        for (int b = 0; b < BT; b++) w[b] = b < B ? q4[(size_t)b * K4 + m] : 0u;
        const int pm = perm_word(m);
#pragma unroll
        for (int b = 0; b < BT; b++) {
            qw[b * K4 + pm] = w[b];
            qs[b] = dp4a_ss((int)w[b], 0x01010101, qs[b]);
        }
    }
#pragma unroll
    for (int b = 0; b < BT; b++) {
        const int v = __reduce_add_sync(0xffffffffu, qs[b]);
        if (lane == 0 && b < B) atomicAdd(qsum_w + b, v);
    }
    if (tid < B) inv_w[tid] = __frcp_rn(a.s[tid]);
    __syncthreads();

    // ---- products.
    int aA[BT], aB[BT];
#pragma unroll
    for (int b = 0; b < BT; b++) aA[b] = aB[b] = 0;
    const uint4 *qrow = reinterpret_cast<const uint4 *>(qw + t * 8);  // token 0, block 0, this lane's part
    const int qstride = K4 / 4;                                        // uint4 per token row
    auto item = [&](const uint4 w, int j) {
        uint32_t dA[8], dB[8];  // codes c of rows g, g + 8: [2 * group + half]
#pragma unroll
        for (int gg = 0; gg < 4; gg++) {
            const int sh = 6 - 2 * gg;
            dA[2 * gg] = (w.x >> sh) & 0x03030303u;
            dA[2 * gg + 1] = (w.z >> sh) & 0x03030303u;
            dB[2 * gg] = (w.y >> sh) & 0x03030303u;
            dB[2 * gg + 1] = (w.w >> sh) & 0x03030303u;
        }
#pragma unroll
        for (int b = 0; b < BT; b++) {
            const uint4 *qv = qrow + b * qstride + j * 8;  // qa0 qb0 qa1 qb1 | qa2 qb2 qa3 qb3
            const uint4 q0 = qv[0], q1 = qv[1];
            const int qv8[8] = {(int)q0.x, (int)q0.y, (int)q0.z, (int)q0.w,
                                (int)q1.x, (int)q1.y, (int)q1.z, (int)q1.w};
#pragma unroll
            for (int k = 0; k < 8; k++) {
                aA[b] = dp4a_us(dA[k], qv8[k], aA[b]);
                aB[b] = dp4a_us(dB[k], qv8[k], aB[b]);
            }
        }
    };
    auto flush = [&](int r) {
        int *rowA = acc + (r * kTileRows + g) * BT;
#pragma unroll
        for (int b = 0; b < BT; b++) {
            const int pA = tig_reduce(aA[b]);
            const int pB = tig_reduce(aB[b]);
            if (t == 0) {
                atomicAdd(rowA + b, pA);
                atomicAdd(rowA + 8 * BT + b, pB);
            }
            aA[b] = aB[b] = 0;
        }
    };
    ring.run(a, ok, limit, warp, lane, item, flush);
    __syncthreads();

    // ---- epilogue: y[b][o] = rowscale * (sum c*q - sum q) * (1/s_b), fp32.
    for (int i = tid; i < ring.nr * kTileRows * B; i += kThreads) {
        const int row = i / B, b = i - row * B;
        const int64_t o = ring.r0 * kTileRows + row;
        if (o < a.rows)
            a.y[(int64_t)b * a.rows + o] =
                __fmul_rn(__fmul_rn(rsc[row], int_to_float(acc[row * BT + b] - qsum_w[b])), inv_w[b]);
    }
}

// Table-lookup variant (batch 1, uniform rows), built for comparison with the
// dp4a products: the pages' CPU kernels replace multiplications by lookups of
// precomputed activation sub-sums indexed by weight codes ("浏览器里跑 1-bit
// 大模型 BitNet WebAssembly 的 50 倍提速实操", section "查表（LUT）内核").
// Here a nibble of an i2_s byte holds the codes of two weights (columns b and
// b + 32, or b + 64 and b + 96, of a 128-weight block), so each CTA builds,
// for every block j and byte position b, two 16-entry tables
//   T[j][b][h][4 * c1 + c2] = (c1 - 1) * q[128 j + b + 64 h] + (c2 - 1) * q[128 j + b + 32 + 64 h]
// (code 3 does not occur in repacked weights; its entries are 0) and a lane
// sums two lookups per weight byte.  The ring, the row-tile ownership and the
// epilogue are the decode kernel's.
__global__ void __launch_bounds__(kThreads, 1) decode_lut_kernel(const DecArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    int8_t *qn = reinterpret_cast<int8_t *>(smem + a.off_q);                   // [K] natural order
    int16_t *lut = reinterpret_cast<int16_t *>(smem + a.off_q + a.K);          // [nb][32][2][16]
    int *acc = reinterpret_cast<int *>(smem + a.off_acc);
    float *rsc = reinterpret_cast<float *>(smem + a.off_rsc);
    int *bad_w = reinterpret_cast<int *>(smem + a.off_red);
    const uint32_t limit = *a.wait_limit;
    WeightRing ring;
    ring.init(a, smem, warp);

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (lane == 0) ring.start(a, rsc, warp);
    for (int i = tid; i < ring.nr * kTileRows; i += kThreads) acc[i] = 0;
    if (tid == 0) *bad_w = 0;
    __syncthreads();  // every warp's slot barriers are initialised before warp 0 polls them
    ring.wait_started(a, smem, bad_w, limit, warp, lane);
    __syncthreads();
    bool ok = *bad_w == 0;

    asm volatile("griddepcontrol.wait;" ::: "memory");  // q, s ready; y free

    const int K4 = a.K >> 2;
    const uint32_t *q4 = reinterpret_cast<const uint32_t *>(a.q);
    for (int i = tid; i < K4; i += kThreads) reinterpret_cast<uint32_t *>(qn)[i] = q4[i];
    const float inv_s = __frcp_rn(*a.s);
    __syncthreads();
    for (int e = tid; e < a.nb * 32 * 2 * 16; e += kThreads) {
        const int idx = e & 15, h = (e >> 4) & 1, b = (e >> 5) & 31, j = e >> 10;
        const int c1 = idx >> 2, c2 = idx & 3;
        const int qa = qn[128 * j + b + 64 * h], qb = qn[128 * j + b + 32 + 64 * h];
        lut[e] = (int16_t)((c1 == 3 || c2 == 3) ? 0 : (c1 - 1) * qa + (c2 - 1) * qb);
    }
    __syncthreads();

    int sA = 0, sB = 0;
    // Bytes 4t..4t+3 (words x, y) and 16+4t.. (words z, w) of the block.
    auto item = [&](const uint4 w, int j) {
        const int16_t *tj = lut + j * 1024;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const int b0 = 4 * t + k, b1 = b0 + 16;
            const int16_t *t0 = tj + b0 * 32, *t1 = tj + b1 * 32;
            sA += t0[(w.x >> (8 * k + 4)) & 15] + t0[16 + ((w.x >> (8 * k)) & 15)];
            sB += t0[(w.y >> (8 * k + 4)) & 15] + t0[16 + ((w.y >> (8 * k)) & 15)];
            sA += t1[(w.z >> (8 * k + 4)) & 15] + t1[16 + ((w.z >> (8 * k)) & 15)];
            sB += t1[(w.w >> (8 * k + 4)) & 15] + t1[16 + ((w.w >> (8 * k)) & 15)];
        }
    };
    auto flush = [&](int r) {
        const int pA = tig_reduce(sA), pB = tig_reduce(sB);
        if (t == 0) {
            atomicAdd(acc + r * kTileRows + g, pA);
            atomicAdd(acc + r * kTileRows + g + 8, pB);
        }
        sA = sB = 0;
    };
    ring.run(a, ok, limit, warp, lane, item, flush);
    __syncthreads();

    for (int i = tid; i < ring.nr * kTileRows; i += kThreads) {
        const int64_t o = ring.r0 * kTileRows + i;
        if (o < a.rows) a.y[o] = __fmul_rn(__fmul_rn(rsc[i], int_to_float(acc[i])), inv_s);
    }
}

struct Plan {
    int grid, nx, wcap;
    size_t smem;
    DecArgs a;
};

// Shapes, grid and shared-memory layout for BT tokens per launch (1 = the
// batch-1 kernel); false if the kernel does not take the shape (the general
// kernel does).
bool plan(const Layout &L, bool fused, int BT, Plan *p) {
    const int sms = num_sms();
    const int grid = (int)(L.ntr < sms ? L.ntr : sms);
    const int K = (int)L.cols;
    int nx = 1;
    while (nx * 4 * kThreads < K) nx *= 2;
    if (K > 16384) return false;  // x in registers (fused); int sums below 2^22 for the fp32 epilogue
    if (fused && BT != 1) return false;
    const int64_t lo = L.ntr / grid, hi = lo + (L.ntr % grid ? 1 : 0);
    const int64_t per_warp = (hi * L.nb + kWarps - 1) / kWarps;
    int wcap = kChunk;  // power of two >= the tiles of a warp, at most kChunk * kMaxSlots
    while (wcap < per_warp && wcap < kChunk * kMaxSlots) wcap *= 2;
    // Two CTAs per SM (one from 8 tokens up): fewer weight slots if q needs room.
    const size_t limit = BT >= 8 ? 200 * 1024 : 100 * 1024;
    DecArgs &a = p->a;
    size_t smem = 0;
    for (;; wcap /= 2) {
        a.off_q = (uint32_t)(kWarps * wcap * kTile);
        a.off_acc = (uint32_t)align_up(a.off_q + (size_t)BT * K, 16);
        a.off_rsc = a.off_acc + (uint32_t)(hi * kTileRows * BT * sizeof(int));
        a.off_red = a.off_rsc + (uint32_t)(hi * kTileRows * sizeof(float));
        a.off_bar = a.off_red + (uint32_t)align_up(8 * BT + 4, 128);
        smem = a.off_bar + 8 * (kWarps * kMaxSlots + 1);
        if (smem <= limit) break;
        if (wcap == kChunk) return false;
    }
    a.rows = L.rows;
    a.K = K;
    a.nb = (int)L.nb;
    a.B = BT;
    a.tiles_lo = (int)lo;
    a.extra = (int)(L.ntr % grid);
    a.wcap = wcap;
    p->grid = grid;
    p->nx = nx;
    p->wcap = wcap;
    p->smem = smem;
    return true;
}

// Layout for the table-lookup kernel: q in natural order, then the tables
// (2 KB per 128-weight block); one CTA per SM.
bool plan_lut(const Layout &L, Plan *p) {
    const int sms = num_sms();
    const int grid = (int)(L.ntr < sms ? L.ntr : sms);
    const int K = (int)L.cols;
    if (K > 8192) return false;
    const int64_t lo = L.ntr / grid, hi = lo + (L.ntr % grid ? 1 : 0);
    const int64_t per_warp = (hi * L.nb + kWarps - 1) / kWarps;
    int wcap = kChunk;
    while (wcap < per_warp && wcap < kChunk * kMaxSlots) wcap *= 2;
    DecArgs &a = p->a;
    for (;; wcap /= 2) {  // fewer weight slots if the tables need the room
        a.off_q = (uint32_t)(kWarps * wcap * kTile);
        a.off_acc = (uint32_t)align_up(a.off_q + (size_t)K + (size_t)L.nb * 2048, 16);
        a.off_rsc = a.off_acc + (uint32_t)(hi * kTileRows * sizeof(int));
        a.off_red = a.off_rsc + (uint32_t)(hi * kTileRows * sizeof(float));
        a.off_bar = a.off_red + 128;
        p->smem = a.off_bar + 8 * (kWarps * kMaxSlots + 1);
        if (p->smem <= 200 * 1024) break;
        if (wcap == kChunk) return false;
    }
    a.rows = L.rows;
    a.K = K;
    a.nb = (int)L.nb;
    a.B = 1;
    a.tiles_lo = (int)lo;
    a.extra = (int)(L.ntr % grid);
    a.wcap = wcap;
    p->grid = grid;
    p->nx = 1;
    p->wcap = wcap;
    return true;
}

int batch_tile(int64_t B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16; }

// smem_cap: the kernel's dynamic shared-memory opt-in (the most any of its
// plans asks for: 100 KB for two CTAs per SM, 200 KB for one).
template <class Kernel>
cudaError_t launch(Kernel k, std::atomic<bool> *configured, int smem_cap, const Plan &p, cudaStream_t st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    // Two host threads may both configure a kernel the first time; setting the
    // same attributes twice is harmless, and the flag itself is atomic.
    if (!configured[dev].load(std::memory_order_acquire)) {
        // Every launch asks for the same shared-memory carveout, so CTAs of
        // consecutive linears can share an SM without it being reconfigured.
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_cap);
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, p.a);
}

template <bool FUSED, int NX>
cudaError_t run_b1(const Plan &p, cudaStream_t st) {
    static std::atomic<bool> configured[64];
    return launch(decode_b1_kernel<FUSED, NX>, configured, 100 * 1024, p, st);
}

template <int BT>
cudaError_t run_bn(const Plan &p, cudaStream_t st) {
    static std::atomic<bool> configured[64];
    return launch(decode_bn_kernel<BT>, configured, BT >= 8 ? 200 * 1024 : 100 * 1024, p, st);
}

}  // namespace

cudaError_t launch_decode_lut(const void *data, int64_t rows, int64_t cols, const int8_t *q, const float *s, float *y,
                              const DeviceGlobals &g, cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    Plan p;
    if (!plan_lut(L, &p)) return cudaErrorNotSupported;
    const unsigned char *base = static_cast<const unsigned char *>(data);
    DecArgs &a = p.a;
    a.tiles = base + L.off_tiles;
    a.rowscale = reinterpret_cast<const float *>(base + L.off_rowscale);
    a.q = q;
    a.s = s;
    a.x = nullptr;
    a.q_out = nullptr;
    a.s_out = nullptr;
    a.y = y;
    a.err = g.err;
    a.wait_limit = g.wait_limit;
    static std::atomic<bool> configured[64];
    return launch(decode_lut_kernel, configured, 200 * 1024, p, st);
}

bool decode_supported(int64_t rows, int64_t cols, int64_t B, bool fused) {
    Plan p;
    return B >= 1 && B <= 16 && plan(layout_of(rows, cols), fused, batch_tile(B), &p);
}

cudaError_t launch_decode(const void *data, int64_t rows, int64_t cols, int64_t B, const int8_t *q, const float *s,
                          float *y, const float *x, int8_t *q_out, float *s_out, const DeviceGlobals &g,
                          cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    const int bt = batch_tile(B);
    Plan p;
    if (B < 1 || B > 16 || !plan(L, x != nullptr, bt, &p)) return cudaErrorNotSupported;
    const unsigned char *base = static_cast<const unsigned char *>(data);
    DecArgs &a = p.a;
    a.tiles = base + L.off_tiles;
    a.rowscale = reinterpret_cast<const float *>(base + L.off_rowscale);
    a.q = q;
    a.s = s;
    a.x = x;
    a.q_out = q_out;
    a.s_out = s_out;
    a.y = y;
    a.err = g.err;
    a.wait_limit = g.wait_limit;
    a.B = (int)B;
    switch (bt) {
        case 2: return run_bn<2>(p, st);
        case 4: return run_bn<4>(p, st);
        case 8: return run_bn<8>(p, st);
        case 16: return run_bn<16>(p, st);
        default: break;
    }
    if (!x) return run_b1<false, 1>(p, st);
    switch (p.nx) {
        case 1: return run_b1<true, 1>(p, st);
        case 2: return run_b1<true, 2>(p, st);
        case 4: return run_b1<true, 4>(p, st);
        default: return run_b1<true, 8>(p, st);
    }
}

}  // namespace bitnet
