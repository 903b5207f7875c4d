// decode_seq.cu -- a whole sequence of batch-1 W2A8 linears (uniform rows) in
// one persistent kernel: the weights of every linear in the list stream from
// HBM without a gap between linears.
//
// Each linear computes what the batch-1 decode kernel computes: per-token
// absmax int8 quantisation of its fp32 input x (s = 127 / max(absmax, 1e-5),
// q = rint(x * s)), the integer product of the ternary weights with q (+1
// adds, -1 subtracts, 0 skips: "BitRun v0.2 实测：1-bit LLM 终端驾驶舱与毫瓦级
// 功耗遥测", section "三值权重与 1.58-bit 的由来"; 2-bit weights x 8-bit
// activations with dp4a: "5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构对
// 决", section "GPU内核突破") and y = rowscale * (sum - sum(q)) * (1/s) in fp32,
// bit for bit the decode kernel's result.
//
// Why one kernel: batch-1 decode reads every weight once and is bound by HBM
// bandwidth ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操",
// section "为什么是 WASM"), but one kernel per linear pays, per linear, a
// launch, the activation phase and a tail in which HBM idles.  Here the weights
// do not depend on the activations, so each warp streams its share of every
// linear's tiles into its own shared-memory ring from the start of the kernel
// to its end, and only the products wait for activations.
//
// Schedule.  A linear's wave is 0 if its x is ready at launch, else one more
// than the wave of the linear whose y it reads (`dep`).  Within a wave, the
// row tiles of all its linears, in list order, are split over the CTAs by
// weight bytes: a tile belongs to the CTA whose share of the wave's items
// (512-byte tiles of 16 rows x 128 weights) holds the tile's first item.  A
// CTA walks its (linear, tile range) segments in wave order; per segment:
//   A  wait for the producer linear (if any), read x, absmax across the CTA,
//      quantise into shared memory in the lanes' read order, sum(q);
//   B  each warp takes an even, contiguous share of the segment's items from
//      its ring (bulk copies of up to eight tiles, refilled as soon as a slot
//      is read, so the next segments' tiles are already in flight);  a tile a
//      warp holds whole is reduced in registers and written to y at once,
//      tiles split between warps are summed in shared memory;
//   C  the split tiles' rows are written; if a later linear reads this
//      linear's y, the CTA adds its tile count to the linear's counter in the
//      caller's workspace (a release add), which the consumers poll (acquire)
//      until it reaches the linear's tile count.
// Linears without a producer thus overlap freely (a CTA holds a contiguous
// slice of the wave, usually one to three linears); a chain of dependent
// linears pays one grid-wide hand-off per linear but never waits for weights.
// Dependent waits need every CTA resident: such calls are cooperative
// launches (one CTA per SM).  Every wait is bounded; on a timeout the kernel
// latches the error word, raises an abort word that ends the other CTAs'
// waits, stops, waits (bounded) for its copies in flight and returns.  The
// last CTA to finish zeroes the counters and the abort word for the next call.
#include <atomic>

#include "common.cuh"
#include "dp4a.cuh"
#include "tcgen05.cuh"

namespace bitnet {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = kTileBytes;
constexpr int kChunk = 8;        // tiles per bulk copy (4 KB; measured faster than 1 and 2 KB copies)
constexpr int kSlots = 3;        // copies in flight per warp: a 12 KB ring per warp
constexpr int kSmallTiles = 32;  // segments of at most this many tiles sum every row in shared memory
constexpr int kRsDepth = 4;      // row-scale loads issued this many tiles ahead
constexpr uint32_t kDrainLimit = 1u << 26;

constexpr int kOffRing = 0;
constexpr int kRingBytes = kWarps * kSlots * kChunk * kTile;  // 192 KB
constexpr int kOffQ = kOffRing + kRingBytes;                  // q, K bytes (permuted words)
constexpr int kOffAcc = kOffQ + kSeqMaxK;                     // [kSmallTiles * 16] int32
constexpr int kOffSeg = kOffAcc + kSmallTiles * kTileRows * 4;
constexpr int kOffRed = kOffSeg + 3 * kSeqMaxLinears * 4 + 64;  // absmax bits, sum(q), abort flag
constexpr int kOffBar = kOffRed + 64;
constexpr int kSmem = kOffBar + kWarps * kSlots * 8;
static_assert(kSmem <= 227 * 1024, "shared memory");

struct SeqLin {
    const unsigned char *tiles;
    const float *rowscale;
    const float *x;
    float *y;
    int64_t item_base;  // items of the earlier linears of the same wave
    int64_t wave_items; // items of every linear of the same wave
    int ntr, nb, rows;
    int dep;            // index of the linear whose y this x reads, or -1
    int signal;         // 1: a later linear waits for this one
};

struct SeqArgs {
    unsigned *done;        // [n] tiles finished per linear (workspace), or null
    unsigned *exit_count;  // CTAs finished (workspace), or null
    unsigned *abort;       // set by a CTA that gave up, so the others stop waiting (workspace), or null
    unsigned *err;
    const unsigned *wait_limit;
    int n;
    SeqLin lin[kSeqMaxLinears];
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Wall-clock bound of the wait for a producer linear (polls of a global
// counter, one L2 round trip each): 4e9 SM cycles, about 2 s, read every
// 1024 polls.
struct PollClock {
    long long t0 = 0;
    __device__ __forceinline__ bool expired(uint32_t i) {
        if ((i & 1023u) != 1023u) return false;
        const long long t = clock64();
        if (t0 == 0) {
            t0 = t;
            return false;
        }
        return t - t0 > 4000000000ll;
    }
};
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

__global__ void __launch_bounds__(kThreads, 1) decode_seq_kernel(const __grid_constant__ SeqArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int c = blockIdx.x, G = gridDim.x;
    int *seg_lo = reinterpret_cast<int *>(smem + kOffSeg);
    int *seg_cnt = seg_lo + kSeqMaxLinears;
    int *seg_list = seg_cnt + kSeqMaxLinears;  // linears with tiles in this CTA, in list order
    int *seg_wcnt = seg_list + kSeqMaxLinears; // [8] + count
    uint32_t *qw = reinterpret_cast<uint32_t *>(smem + kOffQ);
    int *acc = reinterpret_cast<int *>(smem + kOffAcc);
    unsigned *amax_w = reinterpret_cast<unsigned *>(smem + kOffRed);
    int *qsum_w = reinterpret_cast<int *>(smem + kOffRed + 4);
    volatile int *bad_w = reinterpret_cast<volatile int *>(smem + kOffRed + 8);
    unsigned char *ring = smem + kOffRing + (size_t)warp * (kSlots * kChunk * kTile);
    const uint32_t bar0 = ptx::smem_u32(smem + kOffBar) + 8u * (warp * kSlots);
    const uint32_t limit = *a.wait_limit;
    const int n = a.n;
    // The next kernel in the stream may start on the SMs this grid leaves;
    // it reads nothing of ours before its own griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- this CTA's row tiles of every linear: [seg_lo, seg_lo + seg_cnt).
    // The list sits in the kernel parameters, behind the constant cache, which
    // serves the lanes of a warp that read different addresses one after
    // another: with one linear per lane this loop took 8-16 us.  Here every
    // lane of a warp reads the same linear, kPro linears per warp at a time
    // (their loads independent, so in flight together), and lane u keeps
    // linear u of the batch.
    constexpr int kPro = 8;
    for (int L0 = warp * kPro; L0 < n; L0 += kWarps * kPro) {
        int64_t base = 0, W = 0;
        int ntr = 0, nb = 1;
#pragma unroll
        for (int u = 0; u < kPro; u++) {
            if (L0 + u < n) {
                const SeqLin &l = a.lin[L0 + u];
                const int64_t base_u = l.item_base, W_u = l.wave_items;
                const int ntr_u = l.ntr, nb_u = l.nb;
                if (lane == u) {
                    base = base_u;
                    W = W_u;
                    ntr = ntr_u;
                    nb = nb_u;
                }
            }
        }
        if (lane < kPro && L0 + lane < n) {
            const int64_t lo = (int64_t)c * W / G - base;
            const int64_t hi = (int64_t)(c + 1) * W / G - base;
            const int64_t rlo = min((int64_t)ntr, lo <= 0 ? 0 : (lo + nb - 1) / nb);
            const int64_t rhi = min((int64_t)ntr, hi <= 0 ? 0 : (hi + nb - 1) / nb);
            seg_lo[L0 + lane] = (int)rlo;
            seg_cnt[L0 + lane] = (int)(rhi - rlo);
        }
    }
    for (int i = tid; i < kSmallTiles * kTileRows; i += kThreads) acc[i] = 0;
    if (tid == 0) {
        *amax_w = 0u;
        *qsum_w = 0;
        *bad_w = 0;
    }
    if (lane == 0) {
        for (int s = 0; s < kSlots; s++) ptx::mbar_init(bar0 + 8u * s, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    // Compact list of this CTA's segments (warp ballots; n <= 256 = 8 warps).
    const int cL = warp * 32 + lane;
    const bool has = warp < kSeqMaxLinears / 32 && cL < n && seg_cnt[cL] > 0;
    const unsigned hmask = __ballot_sync(0xffffffffu, has);
    if (warp < kSeqMaxLinears / 32 && lane == 0) seg_wcnt[warp] = __popc(hmask);
    __syncthreads();
    if (warp < kSeqMaxLinears / 32) {
        int before = 0;
        for (int w = 0; w < warp; w++) before += seg_wcnt[w];
        if (has) seg_list[before + __popc(hmask & ((1u << lane) - 1u))] = cL;
        if (warp == kSeqMaxLinears / 32 - 1 && lane == 0) seg_wcnt[kSeqMaxLinears / 32] = before + __popc(hmask);
    }
    __syncthreads();
    const int nseg = seg_wcnt[kSeqMaxLinears / 32];

    // This warp's items of segment L: [i0, i1) of the segment's cnt * nb.
    // Warp b's share of a segment's items starts at share_of(b): an even
    // split rounded down to a multiple of four, so that with tiles of a
    // multiple of four items the four-item step of the product loop never
    // straddles a tile.
    auto share_of = [](int b, int64_t items) -> int64_t {
        return b >= kWarps ? items : (((int64_t)b * items / kWarps) & ~(int64_t)3);
    };
    auto run_of = [&](int L, int &i0, int &i1) {
        const int64_t items = (int64_t)seg_cnt[L] * a.lin[L].nb;
        i0 = (int)share_of(warp, items);
        i1 = (int)share_of(warp + 1, items);
    };

    // ---- issue cursor (lane 0): the next chunk of this warp's item stream.
    const uint64_t pol = ptx::policy_evict_first();
    int ik = -1, iL = -1, ii = 0, iend = 0;  // segment, its linear, next item, end of its run
    uint32_t iq = 0;                         // chunks issued
    const unsigned char *isrc = nullptr;     // the next chunk's first tile
    auto next_run = [&]() {
        while (++ik < nseg) {
            iL = seg_list[ik];
            run_of(iL, ii, iend);
            if (iend > ii) {
                const SeqLin &l = a.lin[iL];
                isrc = l.tiles + ((size_t)seg_lo[iL] * l.nb + ii) * kTile;
                return;
            }
        }
        iL = n;
    };
    uint32_t islot = 0;  // slot of the next chunk issued (iq mod kSlots)
    auto issue = [&]() {
        if (iL >= n) return;
        const int nt = min(kChunk, iend - ii);
        const uint32_t slot = islot;
        islot = islot + 1 == kSlots ? 0u : islot + 1;
        const uint32_t bar = bar0 + 8u * slot;
        ptx::mbar_arrive_expect_tx(bar, (uint32_t)(nt * kTile));
        ptx::bulk_g2s(ptx::smem_u32(ring + slot * (kChunk * kTile)), isrc, (uint32_t)(nt * kTile), bar, pol);
        iq++;
        ii += nt;
        isrc += (size_t)nt * kTile;
        if (ii >= iend) next_run();
    };
    // The first segment's x into L2 ahead of the weight copies (a prefetch
    // reads nothing into this SM, so it may precede griddepcontrol.wait).
    if (nseg > 0 && a.lin[seg_list[0]].dep < 0) {
        const SeqLin &l0 = a.lin[seg_list[0]];
        for (int i = tid; i < l0.nb * 4; i += kThreads) prefetch_l2(l0.x + i * 32);
    }
    if (lane == 0) {
        next_run();
        for (int k = 0; k < kSlots; k++) issue();
    }
    // Weights are never written by a kernel, so their copies start before the
    // wait for the previous kernel in the stream (programmatic dependent
    // launch); x, y and the workspace counters are touched only after it.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    uint32_t cq = 0;                      // chunks consumed (every lane keeps the same count)
    uint32_t cslot = 0, cphase = 0;       // its slot and the parity of that slot's phase
    bool ok = true;
    const uint4 *qrow = reinterpret_cast<const uint4 *>(qw + t * 8);  // block 0, this lane's part

    for (int k = 0; k < nseg; k++) {
        const int L = seg_list[k];
        const int cnt = seg_cnt[L];
        const SeqLin &l = a.lin[L];
        const int nb = l.nb, rlo = seg_lo[L];
        const int64_t items = (int64_t)cnt * nb;
        const bool small = cnt <= kSmallTiles;

        // Rows this thread writes in phase C, and their scales (loaded now).
        int erow = -1, eidx = -1;
        if (small) {
            if (tid < cnt * kTileRows) {
                eidx = tid;
                erow = rlo * kTileRows + tid;
            }
        } else if (tid < kWarps * kTileRows) {
            const int b = tid / kTileRows;
            const int64_t pos = share_of(b, items);
            if (b >= 1 && pos % nb != 0) {
                eidx = tid;
                erow = (int)((rlo + pos / nb) * kTileRows + tid % kTileRows);
            }
        }
        const float ers = erow >= 0 ? __ldg(l.rowscale + erow) : 0.0f;
        // This warp's items and the row scales of its first tiles: they do not
        // depend on a producer linear, so their loads overlap phase A (in a
        // chain of dependent linears, each CTA's share of a linear is one or
        // two tiles, and these loads were otherwise the first thing phase B
        // waited for).
        int i0, i1;
        run_of(L, i0, i1);
        float rsq[kRsDepth];
        {
            const int r = i0 / nb, rlast = (i1 - 1) / nb;
#pragma unroll
            for (int k = 0; k < kRsDepth; k++)
                rsq[k] = i1 > i0 && r + k <= rlast
                             ? __ldg(l.rowscale + (int64_t)(rlo + r + k) * kTileRows + (lane & 15))
                             : 0.0f;
        }

        // ---- A: producer, x, absmax, q, sum(q)
        if (l.dep >= 0 && tid == 1) {
            // Each poll is an L2 round trip: a sixteenth of the copy-wait
            // iteration cap and a wall-clock cap bound the wait; another CTA's
            // abort ends it at once.
            const uint32_t dlim = limit >> 4 ? limit >> 4 : 1u;
            uint32_t it = 0;
            PollClock clk;
            const unsigned need = (unsigned)a.lin[l.dep].ntr;
            while (ld_acquire_gpu(a.done + l.dep) < need) {
                if (++it >= dlim || clk.expired(it) || *reinterpret_cast<volatile unsigned *>(a.abort)) {
                    *bad_w = 1;
                    atomicOr(a.err, kErrTimeout);
                    atomicExch(a.abort, 1u);
                    break;
                }
            }
        }
        __syncthreads();  // (1)
        if (*bad_w) break;
        const int K4 = nb * 32;
        const float4 *x4 = reinterpret_cast<const float4 *>(l.x);
        float4 xv[kSeqMaxK / 4 / kThreads];
        float m = 0.0f;
#pragma unroll
        for (int u = 0; u < kSeqMaxK / 4 / kThreads; u++) {
            const int i = tid + u * kThreads;
            if (i < K4) {
                xv[u] = l.dep >= 0 ? __ldcg(x4 + i) : __ldg(x4 + i);
                m = fmaxf(m, fmaxf(fmaxf(fabsf(xv[u].x), fabsf(xv[u].y)), fmaxf(fabsf(xv[u].z), fabsf(xv[u].w))));
            }
        }
        // The next segment's x, if it is ready at launch, into L2 meanwhile.
        if (k + 1 < nseg && a.lin[seg_list[k + 1]].dep < 0) {
            const SeqLin &l2 = a.lin[seg_list[k + 1]];
            for (int i = tid; i < l2.nb * 4; i += kThreads) prefetch_l2(l2.x + i * 32);
        }
        // m >= 0 and not NaN (fmaxf drops NaN): its bit pattern orders like its value.
        const unsigned mu = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
        if (lane == 0) atomicMax(amax_w, mu);
        __syncthreads();  // (2)
        const float amax = __uint_as_float(*amax_w);
        const float s = __fdiv_rn(127.0f, amax > kEps ? amax : kEps);
        const float inv_s = __frcp_rn(s);
        int qs = 0;
#pragma unroll
        for (int u = 0; u < kSeqMaxK / 4 / kThreads; u++) {
            const int i = tid + u * kThreads;
            if (i < K4) {
                const uint32_t w = quant4_fast(xv[u], s);
                qw[perm_word(i)] = w;
                qs = dp4a_ss((int)w, 0x01010101, qs);
            }
        }
        qs = __reduce_add_sync(0xffffffffu, qs);
        if (lane == 0) atomicAdd(qsum_w, qs);
        __syncthreads();  // (3)
        const int tot = *qsum_w;
        if (tid == 0) *amax_w = 0u;  // every thread read it before (3)

        // ---- B: products over this warp's items [i0, i1)
        if (ok && i1 > i0) {
            int r = i0 / nb, j = i0 - r * nb;
            const int rlast = (i1 - 1) / nb;
            const uint4 *qp = qrow + j * 8;
            int aA[4] = {0, 0, 0, 0}, aB[4] = {0, 0, 0, 0};
            // rsq: row scales of tiles r .. r + kRsDepth - 1 (lane l: row l & 15).
            auto flush = [&]() {
                const int pA = tig_reduce(combine4(aA));
                const int pB = tig_reduce(combine4(aB));
                const bool whole = !small && r * nb >= i0 && (r + 1) * nb <= i1;
                const float sA = __shfl_sync(0xffffffffu, rsq[0], g);
                const float sB = __shfl_sync(0xffffffffu, rsq[0], g + 8);
                if (t == 0) {
                    if (whole) {
                        const int64_t o = (int64_t)(rlo + r) * kTileRows + g;
                        if (o < l.rows) l.y[o] = __fmul_rn(__fmul_rn(sA, int_to_float(pA - tot)), inv_s);
                        if (o + 8 < l.rows) l.y[o + 8] = __fmul_rn(__fmul_rn(sB, int_to_float(pB - tot)), inv_s);
                    } else {
                        const int slot = small ? r : (r * nb < i0 ? warp : warp + 1);
                        atomicAdd(acc + slot * kTileRows + g, pA);
                        atomicAdd(acc + slot * kTileRows + g + 8, pB);
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; k++) aA[k] = aB[k] = 0;
#pragma unroll
                for (int k = 0; k + 1 < kRsDepth; k++) rsq[k] = rsq[k + 1];
                rsq[kRsDepth - 1] =
                    r + kRsDepth <= rlast
                        ? __ldg(l.rowscale + (int64_t)(rlo + r + kRsDepth) * kTileRows + (lane & 15))
                        : 0.0f;
            };
            // The products of one item: tile word w (this lane's 16 bytes),
            // activation words at q (qa0 qb0 qa1 qb1 | qa2 qb2 qa3 qb3).
            auto item = [&](const uint4 w, const uint4 *q) {
                const uint4 q0 = q[0], q1 = q[1];
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
            int i = i0;
            while (i < i1) {
                const uint32_t slot = cslot;
                int got = 1;
                if (lane == 0) got = ptx::mbar_wait(bar0 + 8u * slot, cphase, limit, bad_w) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    if (lane == 0 && !*bad_w) {
                        *bad_w = 1;
                        atomicOr(a.err, kErrTimeout);
                        if (a.abort) atomicExch(a.abort, 1u);
                    }
                    ok = false;
                    break;
                }
                const int nt = min(kChunk, i1 - i);
                const uint4 *wv = reinterpret_cast<const uint4 *>(ring + slot * (kChunk * kTile)) + lane;
                for (int e = 0; e < nt;) {
                    if (e + 4 <= nt && j + 4 <= nb) {
                        // Four items of the current row tile.
#pragma unroll
                        for (int u = 0; u < 4; u++) item(wv[(e + u) * 32], qp + u * 8);
                        qp += 32;
                        j += 4;
                        e += 4;
                        if (j == nb) {
                            flush();
                            r++;
                            j = 0;
                            qp = qrow;
                        }
                    } else {
                        item(wv[e * 32], qp);
                        qp += 8;
                        e++;
                        if (++j == nb) {
                            flush();
                            r++;
                            j = 0;
                            qp = qrow;
                        }
                    }
                }
                i += nt;
                cq++;
                if (++cslot == kSlots) {
                    cslot = 0;
                    cphase ^= 1u;
                }
                __syncwarp();  // every lane has read the slot
                if (lane == 0) {
                    ptx::fence_proxy_async_smem();
                    issue();
                }
            }
            if (ok && j != 0) flush();  // the run ends inside tile r
        }
        __syncthreads();  // (4) partial sums complete; direct rows written
        if (tid == 0) *qsum_w = 0;  // every thread read it before (4)

        // ---- C: rows of split tiles; hand-off to consumers
        if (eidx >= 0) {
            const int v = acc[eidx];
            acc[eidx] = 0;
            if (erow < l.rows && !*bad_w) l.y[erow] = __fmul_rn(__fmul_rn(ers, int_to_float(v - tot)), inv_s);
        }
        if (l.signal) {
            // Every thread's y stores precede the barrier; one release add
            // (cumulative over them) publishes the CTA's tiles.  Thread 1 does
            // it: it issues no bulk copies, so nothing of its own is in flight.
            __syncthreads();
            if (tid == 1 && !*bad_w)
                asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(a.done + L), "r"((unsigned)cnt)
                             : "memory");
        }
    }

    // ---- copies still in flight (only after a timeout) are waited out
    if (!ok || *bad_w) {
        if (lane == 0)
            for (uint32_t k = cq; k < iq; k++) ptx::mbar_wait(bar0 + 8u * (k % kSlots), (k / kSlots) & 1u, kDrainLimit, nullptr);
        __syncwarp();
    }
    __syncthreads();
    if (a.done && tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(a.exit_count, 1u);
        if (prev == (unsigned)G - 1) {  // every other CTA is past its last wait
            __threadfence();
            for (int L = 0; L < n; L++) a.done[L] = 0u;
            *a.exit_count = 0u;
            *a.abort = 0u;
            __threadfence();
        }
    }
}

}  // namespace

size_t seq_workspace_bytes(int n) { return align_up((size_t)(n + 2) * sizeof(unsigned), 256); }

cudaError_t launch_decode_seq(const SeqLinear *list, int n, void *workspace, const DeviceGlobals &g,
                              cudaStream_t st) {
    static std::atomic<bool> configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(decode_seq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    static thread_local SeqArgs a;  // ~18 KB: kept off the stack
    a.err = g.err;
    a.wait_limit = g.wait_limit;
    a.n = n;
    // Waves: 0 without a producer, else one more than the producer's.
    int wave[kSeqMaxLinears];
    int64_t wave_items[kSeqMaxLinears];
    int nwaves = 0;
    bool any_dep = false;
    for (int i = 0; i < n; i++) {
        wave[i] = list[i].dep < 0 ? 0 : wave[list[i].dep] + 1;
        nwaves = wave[i] + 1 > nwaves ? wave[i] + 1 : nwaves;
        any_dep = any_dep || list[i].dep >= 0;
    }
    for (int w = 0; w < nwaves; w++) wave_items[w] = 0;
    for (int i = 0; i < n; i++) {
        const Layout Lo = layout_of(list[i].rows, list[i].cols);
        const unsigned char *base = static_cast<const unsigned char *>(list[i].data);
        SeqLin &l = a.lin[i];
        l.tiles = base + Lo.off_tiles;
        l.rowscale = reinterpret_cast<const float *>(base + Lo.off_rowscale);
        l.x = list[i].x;
        l.y = list[i].y;
        l.ntr = (int)Lo.ntr;
        l.nb = (int)Lo.nb;
        l.rows = (int)list[i].rows;
        l.dep = list[i].dep;
        l.signal = 0;
        l.item_base = wave_items[wave[i]];
        wave_items[wave[i]] += (int64_t)Lo.ntr * Lo.nb;
    }
    for (int i = 0; i < n; i++) a.lin[i].wave_items = wave_items[wave[i]];
    for (int i = 0; i < n; i++)
        if (list[i].dep >= 0) a.lin[list[i].dep].signal = 1;
    unsigned *ws = static_cast<unsigned *>(workspace);
    a.done = any_dep ? ws : nullptr;
    a.exit_count = any_dep ? ws + n : nullptr;
    a.abort = any_dep ? ws + n + 1 : nullptr;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // producer waits need every CTA resident
    attr[0].val.cooperative = 1;
    if (!any_dep) {
        // Without producer waits: programmatic dependent launch, so the
        // prologue and the first weight copies overlap the previous kernel.
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_seq_kernel, a);
}

}  // namespace bitnet
