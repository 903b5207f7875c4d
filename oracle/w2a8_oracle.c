/*
 * w2a8_oracle.c -- plain, slow, single-threaded CPU reference for the
 * ternary-weight x int8-activation (W2A8) linear layer.
 *
 * TEST INFRASTRUCTURE.  This file is the oracle that the CUDA library is
 * checked against.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header, table or helper
 * with the library under ternary_weight_absmax_b200/ and includes nothing
 * from it.  It is written for a reader checking it against the pages by eye:
 * no blocking, no fusion, no reordering, integers where the method is integer
 * and fp64 where it is floating point (except where the pages' own format
 * fixes fp32: the activation scale and the packed block scale).
 *
 * Sources (web pages on BitNet b1.58; section headings as printed there):
 *   [WASM]   "浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操"
 *            sections "i2_s 到底是什么" (what i2_s is), "查表（LUT）内核"
 *            (the LUT kernels) and "为什么是 WASM" (ternary weights, absmean).
 *   [CSDN]   "5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构对决",
 *            section "GPU内核突破" (W2A8 = 2-bit weights x 8-bit activations).
 *   [BitRun] "BitRun v0.2 实测：1-bit LLM 终端驾驶舱与毫瓦级功耗遥测",
 *            sections "三值权重与 1.58-bit 的由来" (+1 add, -1 subtract,
 *            0 skip) and "矩阵内存边界与步幅安全" (row stride = cols/4 bytes).
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes with its reason):
 *   R1  group_idx inside a 128-weight block is (i / 32): byte i % 32 of the
 *       block holds weights i, i+32, i+64, i+96 at shifts 6, 4, 2, 0.
 *   R2  block scales live in a separate [rows][cols/128] fp32 array.
 *   R3  absmean gamma: mean |W| summed in fp64, rounded once to fp32, floored
 *       at 1e-5f; t = clamp(rint(W / gamma), -1, 1) with an fp32 divide.
 *   R4  activation scale s = 127 / max(absmax, 1e-5f) (fp32 divide),
 *       q = clamp(rint(x * s), -127, 127) (one fp32 multiply, ties to even).
 *   R5  dequantisation divides by s: y = (sum_j scale_j * acc_j) / s, done in
 *       fp64 with j ascending, rounded once to fp32.
 *
 * Status codes returned here are the oracle's own (0 ok, 1 bad value,
 * 2 corrupt code, 3 bad shape).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_VALUE 1
#define ORC_CORRUPT 2
#define ORC_BAD_SHAPE 3

/* [WASM] "i2_s 到底是什么": x86 blocks hold 128 weights, one float scale each. */
#define ORC_QK 128
/* Floor on absmax / absmean so an all-zero row or tensor is well defined
 * (reading R3/R4; the pages do not give one). */
#define ORC_EPS 1e-5f

static int shape_ok(int64_t rows, int64_t cols) {
    return rows >= 0 && cols >= 0 && cols % ORC_QK == 0;
}

/* ---------------------------------------------------------------------------
 * i2_s pack.  [WASM] "i2_s 到底是什么": a float weight becomes a q8 code,
 * negative -> 0, near zero -> 1, positive -> 2 ("0,1,2 <-> -1,0,1"); four
 * codes share one byte, code i shifted left by (6 - 2*group_idx); 128 weights
 * per block.  [BitRun] "矩阵内存边界与步幅安全": a packed row is cols/4 bytes.
 * Input t is already ternary; anything else is rejected.
 * ------------------------------------------------------------------------- */
int orc_pack_i2s(const int8_t *t, int64_t rows, int64_t cols, uint8_t *codes) {
    if (!shape_ok(rows, cols)) return ORC_BAD_SHAPE;
    int64_t row_bytes = cols / 4;
    for (int64_t o = 0; o < rows; o++) {
        uint8_t *row = codes + o * row_bytes;
        memset(row, 0, (size_t)row_bytes);
        for (int64_t k = 0; k < cols; k++) {
            int v = t[o * cols + k];
            if (v < -1 || v > 1) return ORC_BAD_VALUE;
            unsigned code = (unsigned)(v + 1);          /* -1,0,+1 -> 0,1,2 */
            int64_t block = k / ORC_QK;
            int64_t i = k % ORC_QK;                      /* index in block   */
            int64_t group_idx = i / 32;                  /* reading R1       */
            int64_t byte = block * 32 + (i % 32);
            row[byte] |= (uint8_t)(code << (6 - 2 * group_idx));
        }
    }
    return ORC_OK;
}

/* Inverse of orc_pack_i2s.  Code 3 has no meaning in the format: corrupt. */
int orc_unpack_i2s(const uint8_t *codes, int64_t rows, int64_t cols, int8_t *t) {
    if (!shape_ok(rows, cols)) return ORC_BAD_SHAPE;
    int64_t row_bytes = cols / 4;
    for (int64_t o = 0; o < rows; o++) {
        for (int64_t k = 0; k < cols; k++) {
            int64_t block = k / ORC_QK;
            int64_t i = k % ORC_QK;
            int64_t group_idx = i / 32;
            uint8_t byte = codes[o * row_bytes + block * 32 + (i % 32)];
            unsigned code = (byte >> (6 - 2 * group_idx)) & 3u;
            if (code == 3u) return ORC_CORRUPT;
            t[o * cols + k] = (int8_t)((int)code - 1);
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * absmean ternarisation.  [WASM] "为什么是 WASM": weights constrained to
 * {-1,0,1} with absmean quantisation; [BitRun] "三值权重与 1.58-bit 的由来".
 * Per-tensor variant (one gamma for the whole tensor), reading R3.
 * ------------------------------------------------------------------------- */
static int8_t ternary_of(float w, float gamma) {
    float r = w / gamma;                   /* fp32 divide */
    float n = nearbyintf(r);               /* ties to even */
    if (n > 1.0f) return 1;
    if (n < -1.0f) return -1;
    return (int8_t)n;
}

void orc_absmean_tensor(const float *w, int64_t n, int8_t *t, float *gamma_out) {
    double sum = 0.0;
    for (int64_t i = 0; i < n; i++) sum += fabs((double)w[i]);
    float gamma = n > 0 ? (float)(sum / (double)n) : 0.0f;
    if (!(gamma >= ORC_EPS)) gamma = ORC_EPS;
    for (int64_t i = 0; i < n; i++) t[i] = ternary_of(w[i], gamma);
    *gamma_out = gamma;
}

/* Per-block variant: each 128-weight block gets the absmean of its own
 * weights as its scale (exercises arbitrary per-block scales). */
int orc_absmean_blocks(const float *w, int64_t rows, int64_t cols, int8_t *t,
                       float *scales) {
    if (!shape_ok(rows, cols)) return ORC_BAD_SHAPE;
    int64_t nb = cols / ORC_QK;
    for (int64_t o = 0; o < rows; o++) {
        for (int64_t j = 0; j < nb; j++) {
            const float *blk = w + o * cols + j * ORC_QK;
            double sum = 0.0;
            for (int64_t i = 0; i < ORC_QK; i++) sum += fabs((double)blk[i]);
            float gamma = (float)(sum / (double)ORC_QK);
            if (!(gamma >= ORC_EPS)) gamma = ORC_EPS;
            for (int64_t i = 0; i < ORC_QK; i++)
                t[o * cols + j * ORC_QK + i] = ternary_of(blk[i], gamma);
            scales[o * nb + j] = gamma;
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * Per-token absmax int8 activation quantisation, reading R4.  [CSDN] "GPU内核
 * 突破": the activations of W2A8 are 8-bit; [WASM] "查表（LUT）内核": the
 * activations are quantised and a scale is derived from them.
 * blocksum (nullable): sum of q over each 128-element block.
 * ------------------------------------------------------------------------- */
int orc_quant_act(const float *x, int64_t T, int64_t K, int8_t *q, float *s,
                  int32_t *blocksum) {
    if (T < 0 || K < 0 || (blocksum && K % ORC_QK != 0)) return ORC_BAD_SHAPE;
    for (int64_t b = 0; b < T; b++) {
        const float *row = x + b * K;
        float m = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float a = fabsf(row[k]);
            if (a > m) m = a;
        }
        float scale = 127.0f / (m > ORC_EPS ? m : ORC_EPS);   /* fp32 divide */
        s[b] = scale;
        for (int64_t k = 0; k < K; k++) {
            float p = row[k] * scale;                          /* fp32 multiply */
            float r = nearbyintf(p);                           /* ties to even */
            int v = (int)r;
            if (v > 127) v = 127;
            if (v < -127) v = -127;
            q[b * K + k] = (int8_t)v;
        }
        if (blocksum) {
            for (int64_t j = 0; j < K / ORC_QK; j++) {
                int32_t acc = 0;
                for (int64_t i = 0; i < ORC_QK; i++) acc += q[b * K + j * ORC_QK + i];
                blocksum[b * (K / ORC_QK) + j] = acc;
            }
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * Integer block dot products.  [BitRun] "三值权重与 1.58-bit 的由来": a
 * ternary weight turns the multiply into add (+1), subtract (-1) or skip (0);
 * [WASM] "i2_s 到底是什么": no floating-point matmul anywhere.
 * acc[b][o][j] = sum over the 128 weights of block j of t[o][k] * q[b][k].
 * Done the slow way: unpack a row, then add / subtract / skip.
 * ------------------------------------------------------------------------- */
int orc_block_acc(const uint8_t *codes, int64_t rows, int64_t cols,
                  const int8_t *q, int64_t T, int32_t *acc) {
    if (!shape_ok(rows, cols) || T < 0) return ORC_BAD_SHAPE;
    int64_t nb = cols / ORC_QK;
    int8_t *t = (int8_t *)malloc((size_t)(cols > 0 ? cols : 1));
    if (!t) return ORC_BAD_SHAPE;
    for (int64_t o = 0; o < rows; o++) {
        int rc = orc_unpack_i2s(codes + o * (cols / 4), 1, cols, t);
        if (rc != ORC_OK) { free(t); return rc; }
        for (int64_t b = 0; b < T; b++) {
            const int8_t *qb = q + b * cols;
            for (int64_t j = 0; j < nb; j++) {
                int32_t a = 0;
                for (int64_t i = 0; i < ORC_QK; i++) {
                    int64_t k = j * ORC_QK + i;
                    if (t[k] == 1) a += qb[k];
                    else if (t[k] == -1) a -= qb[k];
                    /* t == 0: skip */
                }
                acc[(b * rows + o) * nb + j] = a;
            }
        }
    }
    free(t);
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * The linear layer, reading R5.  [WASM] "i2_s 到底是什么": dequantisation is
 * a lookup plus scaling.  y[b][o] = (sum_j scale[o][j] * acc[b][o][j]) / s[b],
 * every product exact in fp64, j ascending, one rounding to fp32 at the end.
 * y64 (nullable) receives the fp64 value before that rounding.
 * ------------------------------------------------------------------------- */
int orc_linear(const uint8_t *codes, const float *scales, int64_t rows, int64_t cols,
               const int8_t *q, const float *s, int64_t T, float *y, double *y64) {
    if (!shape_ok(rows, cols) || T < 0) return ORC_BAD_SHAPE;
    int64_t nb = cols / ORC_QK;
    int32_t *acc = (int32_t *)malloc((size_t)((nb > 0 ? nb : 1) * sizeof(int32_t)));
    if (!acc) return ORC_BAD_SHAPE;
    for (int64_t o = 0; o < rows; o++) {
        for (int64_t b = 0; b < T; b++) {
            int rc = orc_block_acc(codes + o * (cols / 4), 1, cols, q + b * cols, 1, acc);
            if (rc != ORC_OK) { free(acc); return rc; }
            double sum = 0.0;
            for (int64_t j = 0; j < nb; j++)
                sum += (double)scales[o * nb + j] * (double)acc[j];
            double v = sum / (double)s[b];
            if (y64) y64[b * rows + o] = v;
            y[b * rows + o] = (float)v;
        }
    }
    free(acc);
    return ORC_OK;
}
