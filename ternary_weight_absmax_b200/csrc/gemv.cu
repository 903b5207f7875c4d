// gemv.cu -- small-batch W2A8 GEMV (1 <= B <= 16) with dp4a: the general
// kernel (per-block scales, accumulator export, fused linear at B >= 2,
// K > 16384).  Calls on uniform rows otherwise go to the decode kernels
// (decode.cu); launch_gemv at the end of this file chooses.
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
//    Each warp puts up to 8 such loads in flight before it touches the
//    activations, so a launch costs about one DRAM latency plus its bytes.
//  * Programmatic dependent launch: the weight loads are issued before
//    griddepcontrol.wait, so they overlap the kernel that produces q (the
//    activation quantiser); q and s are read and y is written only after it.
//    Weights must therefore not be written by the kernel just before.
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
#include "dp4a.cuh"

namespace bitnet {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kQSmemBudget = 32 * 1024;  // bytes of activations staged per K tile
constexpr int kDepth = 8;                // weight loads in flight per lane

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
    // fused activation quantisation (bitnet_w2a8_linear)
    const float *x;   // [B][K] fp32
    int8_t *q_out;    // nullable: q written by CTA 0
    float *s_out;     // nullable: s written by CTA 0
    size_t smem_main; // bytes of the shared q tile / reduction area
};

// The activation words one lane needs for one block of the staged tile:
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
        if (b < a.B) v = reinterpret_cast<const uint4 *>(a.q + (int64_t)b * a.K + kt)[c];
        reinterpret_cast<uint4 *>(qs + b * a.KT)[c] = v;
    }
}

// Fused activation quantisation, pass 1: per batch row, s = 127 / max(absmax,
// 1e-5) with exactly the arithmetic of the standalone quantiser; s_sh[b] gets
// it (1 for padding rows), CTA 0 also writes it to s_out.
template <int BT>
__device__ __forceinline__ void fused_scales(const Args &a, float *s_sh, float *scratch) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n4 = a.K / 4;
#pragma unroll 1
    for (int b = 0; b < BT; b++) {
        float m = 0.0f;
        if (b < a.B) {
            const float4 *xr = reinterpret_cast<const float4 *>(a.x + (int64_t)b * a.K);
            for (int i = threadIdx.x; i < n4; i += kThreads) {
                const float4 v = xr[i];
                m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) scratch[warp * BT + b] = m;
    }
    __syncthreads();
    if (threadIdx.x < BT) {
        const int b = threadIdx.x;
        float mm = scratch[b];
        for (int w = 1; w < kWarps; w++) mm = fmaxf(mm, scratch[w * BT + b]);
        const float sc = __fdiv_rn(127.0f, mm > kEps ? mm : kEps);
        s_sh[b] = b < a.B ? sc : 1.0f;
        if (b < a.B && a.s_out && blockIdx.x == 0) a.s_out[b] = sc;
    }
    __syncthreads();
}

// Fused activation quantisation, pass 2: q[b][kt, kt+n) into the staged tile
// (zero rows for b >= B); CTA 0 also writes q to q_out.
template <int BT>
__device__ __forceinline__ void fused_stage_q(const Args &a, int8_t *qs, const float *s_sh, int kt, int n) {
    const int n4 = n / 4;
#pragma unroll 1
    for (int b = 0; b < BT; b++) {
        uint32_t *dst = reinterpret_cast<uint32_t *>(qs + b * a.KT);
        if (b < a.B) {
            const float4 *xr = reinterpret_cast<const float4 *>(a.x + (int64_t)b * a.K + kt);
            const float sc = s_sh[b];
            uint32_t *qo = (a.q_out && blockIdx.x == 0)
                               ? reinterpret_cast<uint32_t *>(a.q_out + (int64_t)b * a.K + kt)
                               : nullptr;
            for (int i = threadIdx.x; i < n4; i += kThreads) {
                const uint32_t w = quant4(xr[i], sc);
                dst[i] = w;
                if (qo) qo[i] = w;
            }
        } else {
            for (int i = threadIdx.x; i < n4; i += kThreads) dst[i] = 0u;
        }
    }
}

// ---------------------------------------------------------------------------
// One kernel for every batch size: BT = 1 uses the masked scheme (four scaled
// group accumulators per row), BT >= 2 shifts the codes down once per tile.
// Work items of a warp: (row tile r, block j) for j = warp, warp+8, ... in the
// current K tile, r fastest; item i lives in ring slot i % kDepth.
// ---------------------------------------------------------------------------
template <int BT, int RT, bool GENERAL, bool ACC, bool FUSED>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(const Args a) {
    static_assert(kDepth % RT == 0, "ring depth must be a multiple of RT");
    constexpr bool kMasked = (BT == 1);
    constexpr bool kBlockwise = GENERAL || ACC;
    constexpr int NG = kMasked ? 4 : 1;
    constexpr int GR = GENERAL ? RT : 1, GB = GENERAL ? BT : 1;
    extern __shared__ __align__(16) unsigned char smem[];
    int8_t *qs = reinterpret_cast<int8_t *>(smem);
    float *s_sh = reinterpret_cast<float *>(smem + a.smem_main);          // [16]
    float *scratch = reinterpret_cast<float *>(smem + a.smem_main + 64);  // [kWarps][BT]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t rt0 = (int64_t)blockIdx.x * RT;
    const int nrt = (int)min((int64_t)RT, a.ntr - rt0);
    auto s_of = [&](int b) { return FUSED ? s_sh[b] : a.s[b]; };

    int accA[RT][BT][NG], accB[RT][BT][NG];
    double sumA[GR][GB], sumB[GR][GB];
    int qtot[BT];
#pragma unroll
    for (int b = 0; b < BT; b++) {
        qtot[b] = 0;
#pragma unroll
        for (int r = 0; r < RT; r++) {
#pragma unroll
            for (int k = 0; k < NG; k++) accA[r][b][k] = accB[r][b][k] = 0;
        }
    }
#pragma unroll
    for (int r = 0; r < GR; r++)
#pragma unroll
        for (int b = 0; b < GB; b++) sumA[r][b] = sumB[r][b] = 0.0;

    // Let the next kernel on the stream launch; it waits for our completion
    // before it reads anything we write.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    for (int kt = 0; kt < a.K; kt += a.KT) {
        const int ktn = min(a.KT, a.K - kt);
        const int j0 = kt / 128, j1 = (kt + ktn) / 128;
        const int nblk = (j0 + warp < j1) ? (j1 - j0 - warp + kWarps - 1) / kWarps : 0;
        const int nit = nblk * RT;
        auto item_ptr = [&](int it) {
            const int r = it % RT, jj = it / RT;
            return a.tiles + ((rt0 + r) * a.nb + (j0 + warp + kWarps * jj)) * 32 + lane;
        };
        uint4 ring[kDepth];
#pragma unroll
        for (int p = 0; p < kDepth; p++)
            if (p < nit && (p % RT) < nrt) ring[p] = ld_stream(item_ptr(p));

        if (kt == 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");  // q, s (or x) ready; y free
            if (FUSED) fused_scales<BT>(a, s_sh, scratch);
        }
        __syncthreads();
        if (FUSED)
            fused_stage_q<BT>(a, qs, s_sh, kt, ktn);
        else
            stage_q<BT>(a, qs, kt, ktn);
        __syncthreads();

        for (int base = 0; base < nit; base += kDepth) {
#pragma unroll
            for (int p = 0; p < kDepth; p++) {
                const int it = base + p;
                if (it >= nit) break;
                const int r = p % RT;  // = it % RT: base is a multiple of kDepth
                if (r >= nrt) continue;
                const int j = j0 + warp + kWarps * (it / RT);
                const uint4 c = ring[p];
                if (it + kDepth < nit && ((it + kDepth) % RT) < nrt) ring[p] = ld_stream(item_ptr(it + kDepth));
                const int8_t *qblk = qs + (j * 128 - kt);

                if constexpr (kMasked) {
                    int qa[4], qb[4];
                    load_qwords(qblk, t, qa, qb);
                    const int qpart = qword_sum(qa, qb);
                    if (!kBlockwise && r == 0) qtot[0] += qpart;
                    int bA[4], bB[4];
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        bA[k] = kBlockwise ? 0 : accA[r][0][k];
                        bB[k] = kBlockwise ? 0 : accB[r][0][k];
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
                            sumA[GENERAL ? r : 0][0] += (double)__ldg(sc + g) * (double)pA;
                            sumB[GENERAL ? r : 0][0] += (double)__ldg(sc + g + 8) * (double)pB;
                        } else {
                            accA[r][0][0] += pA;
                            accB[r][0][0] += pB;
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
                            accA[r][0][k] = bA[k];
                            accB[r][0][k] = bB[k];
                        }
                    }
                } else {
                    uint32_t d[4][4];
#pragma unroll
                    for (int gg = 0; gg < 4; gg++) {
                        const int sh = 6 - 2 * gg;
                        d[gg][0] = (c.x >> sh) & 0x03030303u;
                        d[gg][1] = (c.y >> sh) & 0x03030303u;
                        d[gg][2] = (c.z >> sh) & 0x03030303u;
                        d[gg][3] = (c.w >> sh) & 0x03030303u;
                    }
                    float scA = 0.0f, scB = 0.0f;
                    if (GENERAL) {
                        const float *sc = a.tscales + ((rt0 + r) * a.nb + j) * 16;
                        scA = __ldg(sc + g);
                        scB = __ldg(sc + g + 8);
                    }
#pragma unroll
                    for (int b = 0; b < BT; b++) {
                        int qa[4], qb[4];
                        load_qwords(qblk + b * a.KT, t, qa, qb);
                        const int qpart = qword_sum(qa, qb);
                        if (!kBlockwise && r == 0) qtot[b] += qpart;
                        int pA = kBlockwise ? 0 : accA[r][b][0];
                        int pB = kBlockwise ? 0 : accB[r][b][0];
#pragma unroll
                        for (int gg = 0; gg < 4; gg++) {
                            pA = dp4a_ss((int)d[gg][0], qa[gg], pA);
                            pA = dp4a_ss((int)d[gg][2], qb[gg], pA);
                            pB = dp4a_ss((int)d[gg][1], qa[gg], pB);
                            pB = dp4a_ss((int)d[gg][3], qb[gg], pB);
                        }
                        if (kBlockwise) {
                            pA -= qpart;
                            pB -= qpart;
                            if (GENERAL) {
                                sumA[GENERAL ? r : 0][GENERAL ? b : 0] += (double)scA * (double)pA;
                                sumB[GENERAL ? r : 0][GENERAL ? b : 0] += (double)scB * (double)pB;
                            } else {
                                accA[r][b][0] += pA;
                                accB[r][b][0] += pB;
                            }
                            if (ACC) {
                                const int fA = tig_reduce(pA), fB = tig_reduce(pB);
                                const int64_t oA = (rt0 + r) * 16 + g, oB = oA + 8;
                                if (t == 0 && b < a.B) {
                                    if (oA < a.rows) a.acc[((int64_t)b * a.rows + oA) * a.nb + j] = fA;
                                    if (oB < a.rows) a.acc[((int64_t)b * a.rows + oB) * a.nb + j] = fB;
                                }
                            }
                        } else {
                            accA[r][b][0] = pA;
                            accB[r][b][0] = pB;
                        }
                    }
                }
            }
        }
    }

    // Cross-lane then cross-warp reduction, fixed order.
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
            if (b < a.B && r < nrt && o < a.rows) a.y[(int64_t)b * a.rows + o] = (float)(v / (double)s_of(b));
        }
    } else {
        int *red = reinterpret_cast<int *>(smem);
#pragma unroll
        for (int r = 0; r < RT; r++) {
#pragma unroll
            for (int b = 0; b < BT; b++) {
                int pA, pB;
                if (kBlockwise) {
                    pA = accA[r][b][0];
                    pB = accB[r][b][0];
                } else if (kMasked) {
                    pA = combine4(accA[r][b]) - qtot[b];
                    pB = combine4(accB[r][b]) - qtot[b];
                } else {
                    pA = accA[r][b][0] - qtot[b];
                    pB = accB[r][b][0] - qtot[b];
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
            if (b < a.B && r < nrt && o < a.rows)
                a.y[(int64_t)b * a.rows + o] =
                    (float)((double)__ldg(a.rowscale + o) * (double)v / (double)s_of(b));
        }
    }
}

template <int BT, int RT, bool GENERAL, bool ACC, bool FUSED>
cudaError_t run(Args a, cudaStream_t st) {
    const size_t red = (size_t)kWarps * RT * 16 * BT * (GENERAL ? sizeof(double) : sizeof(int));
    const size_t q = (size_t)BT * a.KT;
    a.smem_main = align_up(q > red ? q : red, 16);
    const size_t smem = a.smem_main + 64 + (size_t)kWarps * BT * sizeof(float);
    auto k = gemv_kernel<BT, RT, GENERAL, ACC, FUSED>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((a.ntr + RT - 1) / RT));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, a);
}

template <int BT, bool GENERAL, bool ACC, bool FUSED>
cudaError_t dispatch_bt(const Args &a, cudaStream_t st) {
    // Largest row-tile count per CTA that still leaves >= 2 CTAs per SM.
    if constexpr (ACC || (GENERAL && BT >= 8)) {
        return run<BT, 1, GENERAL, ACC, FUSED>(a, st);
    } else if constexpr (BT == 1) {
        if (a.ntr >= 4 * 296) return run<1, 4, GENERAL, ACC, FUSED>(a, st);
        if (a.ntr >= 2 * 296) return run<1, 2, GENERAL, ACC, FUSED>(a, st);
        return run<1, 1, GENERAL, ACC, FUSED>(a, st);
    } else {
        if (a.ntr >= 2 * 296) return run<BT, 2, GENERAL, ACC, FUSED>(a, st);
        return run<BT, 1, GENERAL, ACC, FUSED>(a, st);
    }
}

template <bool GENERAL, bool ACC, bool FUSED>
cudaError_t dispatch(Args &a, cudaStream_t st) {
    const int bt = a.B <= 1 ? 1 : a.B <= 2 ? 2 : a.B <= 4 ? 4 : a.B <= 8 ? 8 : 16;
    int kt = kQSmemBudget / bt;
    kt = kt / 128 * 128;
    a.KT = a.K < kt ? a.K : kt;
    switch (bt) {
        case 1: return dispatch_bt<1, GENERAL, ACC, FUSED>(a, st);
        case 2: return dispatch_bt<2, GENERAL, ACC, FUSED>(a, st);
        case 4: return dispatch_bt<4, GENERAL, ACC, FUSED>(a, st);
        case 8: return dispatch_bt<8, GENERAL, ACC, FUSED>(a, st);
        default: return dispatch_bt<16, GENERAL, ACC, FUSED>(a, st);
    }
}

}  // namespace

cudaError_t launch_gemv(const void *data, int64_t rows, int64_t cols, bool uniform,
                        const int8_t *q, const float *s, int64_t B, float *y, int32_t *acc,
                        const float *x, int8_t *q_out, float *s_out, const DeviceGlobals &g,
                        cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    const char *base = static_cast<const char *>(data);
    if (uniform && !acc && decode_supported(rows, cols, B, x != nullptr))
        return launch_decode(data, rows, cols, B, q, s, y, x, q_out, s_out, g, st);
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
    a.x = x;
    a.q_out = q_out;
    a.s_out = s_out;
    a.smem_main = 0;
    if (x) {
        if (acc) return uniform ? dispatch<false, true, true>(a, st) : dispatch<true, true, true>(a, st);
        return uniform ? dispatch<false, false, true>(a, st) : dispatch<true, false, true>(a, st);
    }
    if (acc) return uniform ? dispatch<false, true, false>(a, st) : dispatch<true, true, false>(a, st);
    return uniform ? dispatch<false, false, false>(a, st) : dispatch<true, false, false>(a, st);
}

}  // namespace bitnet
