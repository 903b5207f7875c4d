// gemv.cu -- decode / small-batch W2A8 GEMV (1 <= B <= 16) with dp4a.
//
// y[b][o] = (sum_j scale[o][j] * acc[b][o][j]) / s[b],
// acc[b][o][j] = sum_{k in block j} t[o][k] * q[b][k]   (int32, exact).
//
// The pages describe the decode-time W2A8 linear as a 2-bit-weight x 8-bit-
// activation GEMV built on dp4a ("5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理
// 架构对决", section "GPU内核突破") and the workload as memory-bandwidth bound
// ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操", section
// "为什么是 WASM").  The kernel below is this library's own design for sm_100a:
//
//  * Weights are read once, 16 bytes per lane per 16x128 tile (a warp reads a
//    whole 512-byte tile with one coalesced instruction), streamed past L1.
//  * The 2-bit codes are never expanded to bytes.  A 32-bit word of i2_s bytes
//    masked with 0x03030303 << (6 - 2*group) holds four codes of four
//    consecutive columns, scaled by 4^(3-group).  dp4a (unsigned codes x
//    signed q) accumulates each group separately and the four sums are
//    recombined with exact shifts.  Using the code c = t + 1 instead of t
//    costs one subtraction of sum(q) per row instead of one per weight:
//    sum t*q = sum c*q - sum q.   (Batch 1; for B >= 2 the codes are shifted
//    down once per tile and reused for every batch row.)
//  * A CTA (8 warps) owns RT row tiles; its warps split the K blocks of those
//    tiles (block j goes to warp j % 8), so even 2560-row layers fill all 148
//    SMs.  The activations of the CTA are staged once in shared memory.
//  * Uniform rows (all block scales equal, the per-tensor absmean case):
//    int32 accumulation over the whole row, one exact fp64 product with the
//    row scale and one fp64 divide by s.  General rows: every block's int32
//    partial is multiplied by its fp32 scale in fp64 (exact) and summed in
//    fp64; one rounding to fp32 at the end.
//  * Cross-lane and cross-warp reductions run in a fixed order, so results
//    are deterministic.
#include "common.cuh"

namespace bitnet {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kQSmemBudget = 32 * 1024;  // bytes of activations staged per K tile

__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ int dp4a_ss(int a, int b, int c) { return __dp4a(a, b, c); }

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Four masked-and-scaled group sums -> sum of code*q.
__device__ __forceinline__ int combine4(const int a[4]) {
    return a[3] + (a[2] >> 2) + (a[1] >> 4) + (a[0] >> 6);
}

template <typename T>
__device__ __forceinline__ T tig_reduce(T v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

struct Args {
    const uint4 *tiles;
    const float *tscales;
    const float *rowscale;
    const int8_t *q;
    const float *s;
    float *y;
    int32_t *acc;
    int B;
    int64_t rows;
    int K;
    int nb;
    int64_t ntr;
    int KT;
};

// Loads the activation words one lane needs for block j of the staged tile:
// qa[g] = q[32g + 4t .. +3], qb[g] = q[32g + 16 + 4t .. +3] (block-relative).
__device__ __forceinline__ void load_qwords(const int8_t *qs, int t, int qa[4], int qb[4]) {
#pragma unroll
    for (int g = 0; g < 4; g++) {
        qa[g] = *reinterpret_cast<const int *>(qs + 32 * g + 4 * t);
        qb[g] = *reinterpret_cast<const int *>(qs + 32 * g + 16 + 4 * t);
    }
}

__device__ __forceinline__ int qword_sum(const int qa[4], const int qb[4]) {
    int s = 0;
#pragma unroll
    for (int g = 0; g < 4; g++) {
        s = dp4a_ss(qa[g], 0x01010101, s);
        s = dp4a_ss(qb[g], 0x01010101, s);
    }
    return s;
}

// Stages q[b][kt, kt+n) for b < BT (zero rows for b >= B) in shared memory,
// row stride a.KT bytes.
template <int BT>
__device__ __forceinline__ void stage_q(const Args &a, int8_t *qs, int kt, int n) {
    const int per_row = n / 16;
    for (int idx = threadIdx.x; idx < BT * per_row; idx += kThreads) {
        const int b = idx / per_row, c = idx - b * per_row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (b < a.B) v = __ldg(reinterpret_cast<const uint4 *>(a.q + (int64_t)b * a.K + kt) + c);
        reinterpret_cast<uint4 *>(qs + b * a.KT)[c] = v;
    }
}

// ---------------------------------------------------------------------------
// Batch 1: masked dp4a, RT row tiles per CTA.
// ---------------------------------------------------------------------------
template <int RT, bool GENERAL, bool ACC>
__global__ void __launch_bounds__(kThreads)
gemv_b1_kernel(const Args a) {
    extern __shared__ __align__(16) unsigned char smem[];
    int8_t *qs = reinterpret_cast<int8_t *>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t rt0 = (int64_t)blockIdx.x * RT;

    constexpr bool kBlockwise = GENERAL || ACC;
    int accA[RT][4], accB[RT][4];
    double sumA[RT], sumB[RT];
    int totA[RT], totB[RT];
#pragma unroll
    for (int r = 0; r < RT; r++) {
#pragma unroll
        for (int k = 0; k < 4; k++) accA[r][k] = accB[r][k] = 0;
        sumA[r] = sumB[r] = 0.0;
        totA[r] = totB[r] = 0;
    }
    int qtot = 0;

    for (int kt = 0; kt < a.K; kt += a.KT) {
        const int ktn = min(a.KT, a.K - kt);
        __syncthreads();
        stage_q<1>(a, qs, kt, ktn);
        __syncthreads();
        const int j0 = kt / 128, j1 = (kt + ktn) / 128;
        int j = j0 + warp;
        uint4 cur[RT];
        if (j < j1) {
#pragma unroll
            for (int r = 0; r < RT; r++)
                if (rt0 + r < a.ntr) cur[r] = ld_stream(a.tiles + ((rt0 + r) * a.nb + j) * 32 + lane);
        }
        for (; j < j1; j += kWarps) {
            uint4 nxt[RT];
            const int jn = j + kWarps;
            if (jn < j1) {
#pragma unroll
                for (int r = 0; r < RT; r++)
                    if (rt0 + r < a.ntr)
                        nxt[r] = ld_stream(a.tiles + ((rt0 + r) * a.nb + jn) * 32 + lane);
            }
            int qa[4], qb[4];
            load_qwords(qs + (j * 128 - kt), t, qa, qb);
            const int qpart = qword_sum(qa, qb);
            if (!kBlockwise) qtot += qpart;
#pragma unroll
            for (int r = 0; r < RT; r++) {
                if (rt0 + r >= a.ntr) continue;
                const uint4 c = cur[r];
                int bA[4], bB[4];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    bA[k] = kBlockwise ? 0 : accA[r][k];
                    bB[k] = kBlockwise ? 0 : accB[r][k];
                }
#pragma unroll
                for (int gg = 0; gg < 4; gg++) {
                    const uint32_t m = 0xC0C0C0C0u >> (2 * gg);
                    bA[gg] = dp4a_us(c.x & m, qa[gg], bA[gg]);
                    bA[gg] = dp4a_us(c.z & m, qb[gg], bA[gg]);
                    bB[gg] = dp4a_us(c.y & m, qa[gg], bB[gg]);
                    bB[gg] = dp4a_us(c.w & m, qb[gg], bB[gg]);
                }
                if (kBlockwise) {
                    const int pA = combine4(bA) - qpart;
                    const int pB = combine4(bB) - qpart;
                    if (GENERAL) {
                        const float *sc = a.tscales + ((rt0 + r) * a.nb + j) * 16;
                        sumA[r] += (double)__ldg(sc + g) * (double)pA;
                        sumB[r] += (double)__ldg(sc + g + 8) * (double)pB;
                    } else {
                        totA[r] += pA;
                        totB[r] += pB;
                    }
                    if (ACC) {
                        const int fA = tig_reduce(pA), fB = tig_reduce(pB);
                        const int64_t oA = (rt0 + r) * 16 + g, oB = oA + 8;
                        if (t == 0) {
                            if (oA < a.rows) a.acc[oA * a.nb + j] = fA;
                            if (oB < a.rows) a.acc[oB * a.nb + j] = fB;
                        }
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        accA[r][k] = bA[k];
                        accB[r][k] = bB[k];
                    }
                }
            }
            if (jn < j1) {
#pragma unroll
                for (int r = 0; r < RT; r++) cur[r] = nxt[r];
            }
        }
    }

    // Cross-lane then cross-warp reduction, fixed order.
    __syncthreads();
    if (GENERAL) {
        double *red = reinterpret_cast<double *>(smem);  // [warp][RT*16]
#pragma unroll
        for (int r = 0; r < RT; r++) {
            const double vA = tig_reduce(sumA[r]), vB = tig_reduce(sumB[r]);
            if (t == 0) {
                red[(warp * RT + r) * 16 + g] = vA;
                red[(warp * RT + r) * 16 + g + 8] = vB;
            }
        }
        __syncthreads();
        if (threadIdx.x < RT * 16) {
            const int r = threadIdx.x / 16, row = threadIdx.x % 16;
            const int64_t o = (rt0 + r) * 16 + row;
            double v = 0.0;
            for (int w = 0; w < kWarps; w++) v += red[(w * RT + r) * 16 + row];
            if (rt0 + r < a.ntr && o < a.rows) a.y[o] = (float)(v / (double)a.s[0]);
        }
    } else {
        int *red = reinterpret_cast<int *>(smem);
#pragma unroll
        for (int r = 0; r < RT; r++) {
            int pA, pB;
            if (kBlockwise) {
                pA = totA[r];
                pB = totB[r];
            } else {
                pA = combine4(accA[r]) - qtot;
                pB = combine4(accB[r]) - qtot;
            }
            pA = tig_reduce(pA);
            pB = tig_reduce(pB);
            if (t == 0) {
                red[(warp * RT + r) * 16 + g] = pA;
                red[(warp * RT + r) * 16 + g + 8] = pB;
            }
        }
        __syncthreads();
        if (threadIdx.x < RT * 16) {
            const int r = threadIdx.x / 16, row = threadIdx.x % 16;
            const int64_t o = (rt0 + r) * 16 + row;
            int v = 0;
            for (int w = 0; w < kWarps; w++) v += red[(w * RT + r) * 16 + row];
            if (rt0 + r < a.ntr && o < a.rows)
                a.y[o] = (float)((double)__ldg(a.rowscale + o) * (double)v / (double)a.s[0]);
        }
    }
}

// ---------------------------------------------------------------------------
// Batch 2..16: codes shifted down once per tile and reused across the batch.
// ---------------------------------------------------------------------------
template <int BT, int RT, bool GENERAL, bool ACC>
__global__ void __launch_bounds__(kThreads)
gemv_bn_kernel(const Args a) {
    extern __shared__ __align__(16) unsigned char smem[];
    int8_t *qs = reinterpret_cast<int8_t *>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t rt0 = (int64_t)blockIdx.x * RT;
    constexpr bool kBlockwise = GENERAL || ACC;

    int accA[RT][BT], accB[RT][BT];
    double sumA[GENERAL ? RT : 1][GENERAL ? BT : 1], sumB[GENERAL ? RT : 1][GENERAL ? BT : 1];
    int qtot[BT];
#pragma unroll
    for (int b = 0; b < BT; b++) {
        qtot[b] = 0;
#pragma unroll
        for (int r = 0; r < RT; r++) {
            accA[r][b] = accB[r][b] = 0;
            if (GENERAL) sumA[r][b] = sumB[r][b] = 0.0;
        }
    }

    for (int kt = 0; kt < a.K; kt += a.KT) {
        const int ktn = min(a.KT, a.K - kt);
        __syncthreads();
        stage_q<BT>(a, qs, kt, ktn);
        __syncthreads();
        const int j0 = kt / 128, j1 = (kt + ktn) / 128;
        int j = j0 + warp;
        uint4 cur[RT];
        if (j < j1) {
#pragma unroll
            for (int r = 0; r < RT; r++)
                if (rt0 + r < a.ntr) cur[r] = ld_stream(a.tiles + ((rt0 + r) * a.nb + j) * 32 + lane);
        }
        for (; j < j1; j += kWarps) {
            uint4 nxt[RT];
            const int jn = j + kWarps;
            if (jn < j1) {
#pragma unroll
                for (int r = 0; r < RT; r++)
                    if (rt0 + r < a.ntr)
                        nxt[r] = ld_stream(a.tiles + ((rt0 + r) * a.nb + jn) * 32 + lane);
            }
            // Decode: d[r][gg][0..3] = codes of group gg in words x, y, z, w.
            uint32_t d[RT][4][4];
#pragma unroll
            for (int r = 0; r < RT; r++) {
#pragma unroll
                for (int gg = 0; gg < 4; gg++) {
                    const int sh = 6 - 2 * gg;
                    d[r][gg][0] = (cur[r].x >> sh) & 0x03030303u;
                    d[r][gg][1] = (cur[r].y >> sh) & 0x03030303u;
                    d[r][gg][2] = (cur[r].z >> sh) & 0x03030303u;
                    d[r][gg][3] = (cur[r].w >> sh) & 0x03030303u;
                }
            }
            float scA[RT], scB[RT];
            if (GENERAL) {
#pragma unroll
                for (int r = 0; r < RT; r++) {
                    const float *sc = a.tscales + ((rt0 + r < a.ntr ? rt0 + r : 0) * a.nb + j) * 16;
                    scA[r] = __ldg(sc + g);
                    scB[r] = __ldg(sc + g + 8);
                }
            }
#pragma unroll
            for (int b = 0; b < BT; b++) {
                int qa[4], qb[4];
                load_qwords(qs + b * a.KT + (j * 128 - kt), t, qa, qb);
                const int qpart = qword_sum(qa, qb);
                if (!kBlockwise) qtot[b] += qpart;
#pragma unroll
                for (int r = 0; r < RT; r++) {
                    int pA = kBlockwise ? 0 : accA[r][b];
                    int pB = kBlockwise ? 0 : accB[r][b];
#pragma unroll
                    for (int gg = 0; gg < 4; gg++) {
                        pA = dp4a_ss((int)d[r][gg][0], qa[gg], pA);
                        pA = dp4a_ss((int)d[r][gg][2], qb[gg], pA);
                        pB = dp4a_ss((int)d[r][gg][1], qa[gg], pB);
                        pB = dp4a_ss((int)d[r][gg][3], qb[gg], pB);
                    }
                    if (kBlockwise) {
                        pA -= qpart;
                        pB -= qpart;
                        if (GENERAL) {
                            sumA[GENERAL ? r : 0][GENERAL ? b : 0] += (double)scA[r] * (double)pA;
                            sumB[GENERAL ? r : 0][GENERAL ? b : 0] += (double)scB[r] * (double)pB;
                        } else {
                            accA[r][b] += pA;
                            accB[r][b] += pB;
                        }
                        if (ACC) {
                            const int fA = tig_reduce(pA), fB = tig_reduce(pB);
                            const int64_t oA = (rt0 + r) * 16 + g, oB = oA + 8;
                            if (t == 0 && b < a.B && rt0 + r < a.ntr) {
                                if (oA < a.rows) a.acc[((int64_t)b * a.rows + oA) * a.nb + j] = fA;
                                if (oB < a.rows) a.acc[((int64_t)b * a.rows + oB) * a.nb + j] = fB;
                            }
                        }
                    } else {
                        accA[r][b] = pA;
                        accB[r][b] = pB;
                    }
                }
            }
            if (jn < j1) {
#pragma unroll
                for (int r = 0; r < RT; r++) cur[r] = nxt[r];
            }
        }
    }

    __syncthreads();
    const int nred = RT * 16 * BT;
    if (GENERAL) {
        double *red = reinterpret_cast<double *>(smem);  // [warp][RT][16][BT]
#pragma unroll
        for (int r = 0; r < RT; r++) {
#pragma unroll
            for (int b = 0; b < BT; b++) {
                const double vA = tig_reduce(sumA[GENERAL ? r : 0][GENERAL ? b : 0]);
                const double vB = tig_reduce(sumB[GENERAL ? r : 0][GENERAL ? b : 0]);
                if (t == 0) {
                    red[warp * nred + (r * 16 + g) * BT + b] = vA;
                    red[warp * nred + (r * 16 + g + 8) * BT + b] = vB;
                }
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nred; i += kThreads) {
            const int b = i % BT, rr = i / BT, r = rr / 16, row = rr % 16;
            const int64_t o = (rt0 + r) * 16 + row;
            double v = 0.0;
            for (int w = 0; w < kWarps; w++) v += red[w * nred + i];
            if (b < a.B && rt0 + r < a.ntr && o < a.rows)
                a.y[(int64_t)b * a.rows + o] = (float)(v / (double)a.s[b]);
        }
    } else {
        int *red = reinterpret_cast<int *>(smem);
#pragma unroll
        for (int r = 0; r < RT; r++) {
#pragma unroll
            for (int b = 0; b < BT; b++) {
                int pA = accA[r][b], pB = accB[r][b];
                if (!kBlockwise) {
                    pA -= qtot[b];
                    pB -= qtot[b];
                }
                pA = tig_reduce(pA);
                pB = tig_reduce(pB);
                if (t == 0) {
                    red[warp * nred + (r * 16 + g) * BT + b] = pA;
                    red[warp * nred + (r * 16 + g + 8) * BT + b] = pB;
                }
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nred; i += kThreads) {
            const int b = i % BT, rr = i / BT, r = rr / 16, row = rr % 16;
            const int64_t o = (rt0 + r) * 16 + row;
            int v = 0;
            for (int w = 0; w < kWarps; w++) v += red[w * nred + i];
            if (b < a.B && rt0 + r < a.ntr && o < a.rows)
                a.y[(int64_t)b * a.rows + o] =
                    (float)((double)__ldg(a.rowscale + o) * (double)v / (double)a.s[b]);
        }
    }
}

template <int RT, bool GENERAL, bool ACC>
cudaError_t run_b1(const Args &a, cudaStream_t st) {
    const size_t red = (size_t)kWarps * RT * 16 * sizeof(double);
    const size_t smem = a.KT > (int)red ? (size_t)a.KT : red;
    auto k = gemv_b1_kernel<RT, GENERAL, ACC>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const unsigned grid = (unsigned)((a.ntr + RT - 1) / RT);
    k<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int BT, int RT, bool GENERAL, bool ACC>
cudaError_t run_bn(const Args &a, cudaStream_t st) {
    const size_t red = (size_t)kWarps * RT * 16 * BT * (GENERAL ? sizeof(double) : sizeof(int));
    const size_t q = (size_t)BT * a.KT;
    const size_t smem = q > red ? q : red;
    auto k = gemv_bn_kernel<BT, RT, GENERAL, ACC>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const unsigned grid = (unsigned)((a.ntr + RT - 1) / RT);
    k<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <bool GENERAL, bool ACC>
cudaError_t dispatch_b1(const Args &a, cudaStream_t st) {
    if constexpr (ACC) {
        return run_b1<1, GENERAL, ACC>(a, st);
    } else {
        // Largest row-tile count per CTA that still leaves >= 2 CTAs per SM.
        if (a.ntr >= 4 * 296) return run_b1<4, GENERAL, ACC>(a, st);
        if (a.ntr >= 2 * 296) return run_b1<2, GENERAL, ACC>(a, st);
        return run_b1<1, GENERAL, ACC>(a, st);
    }
}

template <int BT, bool GENERAL, bool ACC>
cudaError_t dispatch_bn(const Args &a, cudaStream_t st) {
    if constexpr (!GENERAL && !ACC && BT <= 4) {
        if (a.ntr >= 2 * 296) return run_bn<BT, 2, GENERAL, ACC>(a, st);
    }
    return run_bn<BT, 1, GENERAL, ACC>(a, st);
}

template <bool GENERAL, bool ACC>
cudaError_t dispatch(Args &a, cudaStream_t st) {
    int bt = a.B <= 1 ? 1 : a.B <= 2 ? 2 : a.B <= 4 ? 4 : a.B <= 8 ? 8 : 16;
    int kt = kQSmemBudget / bt;
    kt = kt / 128 * 128;
    a.KT = a.K < kt ? a.K : kt;
    switch (bt) {
        case 1: return dispatch_b1<GENERAL, ACC>(a, st);
        case 2: return dispatch_bn<2, GENERAL, ACC>(a, st);
        case 4: return dispatch_bn<4, GENERAL, ACC>(a, st);
        case 8: return dispatch_bn<8, GENERAL, ACC>(a, st);
        default: return dispatch_bn<16, GENERAL, ACC>(a, st);
    }
}

}  // namespace

cudaError_t launch_gemv(const void *data, int64_t rows, int64_t cols, bool uniform,
                        const int8_t *q, const float *s, int64_t B, float *y, int32_t *acc,
                        cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    const char *base = static_cast<const char *>(data);
    Args a;
    a.tiles = reinterpret_cast<const uint4 *>(base + L.off_tiles);
    a.tscales = reinterpret_cast<const float *>(base + L.off_tscales);
    a.rowscale = reinterpret_cast<const float *>(base + L.off_rowscale);
    a.q = q;
    a.s = s;
    a.y = y;
    a.acc = acc;
    a.B = (int)B;
    a.rows = rows;
    a.K = (int)cols;
    a.nb = (int)L.nb;
    a.ntr = L.ntr;
    a.KT = 0;
    if (acc) return uniform ? dispatch<false, true>(a, st) : dispatch<true, true>(a, st);
    return uniform ? dispatch<false, false>(a, st) : dispatch<true, false>(a, st);
}

}  // namespace bitnet
