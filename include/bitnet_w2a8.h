/*
 * bitnet_w2a8.h -- C ABI of libbitnet_w2a8.so, a B200 (sm_100a) library for
 * the BitNet b1.58 ternary-weight x int8-activation ("W2A8") linear layer.
 *
 * What the layer computes, and where the pages say so:
 *   - Weights are ternary {-1, 0, +1}, stored as "i2_s": 2-bit codes
 *     0, 1, 2 for -1, 0, +1, four codes per byte, code shifted left by
 *     (6 - 2*group_idx), 128-weight blocks with one float scale per block.
 *     ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操",
 *     section "i2_s 到底是什么".)  group_idx is the index inside the block
 *     divided by 32, so byte b of a block holds weights b, b+32, b+64, b+96.
 *   - A packed row of `cols` weights takes cols/4 bytes ("BitRun v0.2
 *     实测：1-bit LLM 终端驾驶舱与毫瓦级功耗遥测", section
 *     "矩阵内存边界与步幅安全").
 *   - Activations are 8-bit ("5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理
 *     架构对决", section "GPU内核突破"): per token, s = 127 / max(absmax,
 *     1e-5) in fp32 and q = round-half-to-even(x * s), clamped to [-127, 127].
 *   - The product is integer: +1 adds, -1 subtracts, 0 skips ("BitRun v0.2
 *     实测", section "三值权重与 1.58-bit 的由来").  acc[b][o][j] is the int32
 *     sum over block j, and y[b][o] = (sum_j scale[o][j] * acc[b][o][j]) / s[b]
 *     ("i2_s 到底是什么": dequantisation is a lookup plus scaling).
 *
 * Conventions for every call:
 *   - Row-major everywhere.  Weights are [rows = out][cols = K]; activations
 *     are [T][K]; outputs are [T][out].  cols (K) must be a multiple of 128.
 *   - The library never allocates and never frees caller memory.  Every
 *     buffer is owned by the caller; device buffers may come from any CUDA
 *     allocator (for example PyTorch).
 *   - Device pointers named *_dev must be device memory on the current
 *     device, 16-byte aligned unless a call says otherwise.
 *   - Calls marked "async" validate their arguments on the host, enqueue
 *     kernels on `stream` and return; errors found later on the device (a
 *     bounded wait that ran out, a corrupt code) are latched in a per-device
 *     error word read by bitnet_get_device_error().  Kernels never trap.
 *   - A call that fails validation enqueues nothing and returns the status.
 *     A launch failure returns BITNET_ERR_CUDA.
 *   - bitnet_last_error_detail() gives a human-readable reason for the last
 *     non-OK status returned on the calling host thread.
 *   - NaN or Inf in activations or scales give unspecified (but memory-safe)
 *     results.
 */
#ifndef BITNET_W2A8_H
#define BITNET_W2A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st *bitnet_stream_t;

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_NULL = 1,        /* a required pointer is NULL               */
    BITNET_ERR_SHAPE = 2,       /* a size is negative, too large, or K%128  */
    BITNET_ERR_ALIGN = 3,       /* a pointer is not aligned as required     */
    BITNET_ERR_VALUE = 4,       /* an input value is outside its domain     */
    BITNET_ERR_CORRUPT = 5,     /* packed data holds the unused code 3      */
    BITNET_ERR_BUFSIZE = 6,     /* a caller buffer is smaller than needed   */
    BITNET_ERR_CUDA = 7,        /* a CUDA runtime call or launch failed     */
    BITNET_ERR_TIMEOUT = 8,     /* a bounded device wait ran out            */
    BITNET_ERR_UNSUPPORTED = 9  /* no kernel for this case / this device    */
} bitnet_status;

/* Static string naming a status.  Never NULL. */
const char *bitnet_status_string(bitnet_status status);

/* Reason for the last non-OK status on this host thread ("" if none). */
const char *bitnet_last_error_detail(void);

/* Library version, (major << 16) | minor. */
uint32_t bitnet_version(void);

/* ------------------------------------------------------------------------
 * Sizes.  Return 0 for an invalid shape (negative, or cols % 128 != 0).
 * ---------------------------------------------------------------------- */

/* Bytes of i2_s codes for a rows x cols ternary matrix: rows * cols / 4. */
size_t bitnet_i2s_code_bytes(int64_t rows, int64_t cols);

/* Number of fp32 block scales: rows * cols / 128. */
size_t bitnet_i2s_num_scales(int64_t rows, int64_t cols);

/* Bytes of the device weight buffer that bitnet_repack_device fills. */
size_t bitnet_repacked_bytes(int64_t rows, int64_t cols);

/* ------------------------------------------------------------------------
 * Host-side i2_s packing (plain, synchronous, no GPU needed).
 * ---------------------------------------------------------------------- */

/* Packs a row-major int8 matrix of {-1, 0, +1} into i2_s codes
 * ("i2_s 到底是什么": -1 -> 0, 0 -> 1, +1 -> 2, code << (6 - 2*group_idx)).
 * codes_out receives rows * cols / 4 bytes, row stride cols / 4.
 * Errors: NULL, SHAPE, BUFSIZE (codes_bytes too small), VALUE (an entry is
 * not in {-1, 0, +1}; codes_out is then unspecified). */
bitnet_status bitnet_pack_i2s(const int8_t *ternary, int64_t rows, int64_t cols,
                              uint8_t *codes_out, size_t codes_bytes);

/* Inverse of bitnet_pack_i2s.  ternary_out receives rows * cols int8.
 * Errors: NULL, SHAPE, BUFSIZE, CORRUPT (a 2-bit field holds code 3). */
bitnet_status bitnet_unpack_i2s(const uint8_t *codes, int64_t rows, int64_t cols,
                                int8_t *ternary_out, size_t ternary_bytes);

/* ------------------------------------------------------------------------
 * Device-side absmean ternarisation + i2_s packing (async).
 * ---------------------------------------------------------------------- */

#define BITNET_ABSMEAN_PER_TENSOR 0 /* one gamma for the whole matrix       */
#define BITNET_ABSMEAN_PER_BLOCK 1  /* one gamma per 128-weight block       */

/* Bytes of device scratch bitnet_ternarize_absmean_device needs (any mode). */
size_t bitnet_ternarize_workspace_bytes(int64_t rows, int64_t cols);

/* Ternarises fp32 weights w_dev [rows][cols] with absmean scaling and packs
 * them as i2_s ("浏览器里跑 1-bit 大模型 ..." sections "为什么是 WASM" and
 * "i2_s 到底是什么"; "BitRun v0.2 实测" section "三值权重与 1.58-bit 的由来"):
 *   gamma = max(mean |W| (fp64 sum, rounded once to fp32), 1e-5)
 *   t = clamp(rint(W / gamma), -1, 1)  (fp32 divide, ties to even)
 * over the whole matrix (PER_TENSOR) or over each 128-weight block
 * (PER_BLOCK).  Writes codes_out_dev [rows][cols/4] (4-byte aligned) and the
 * block scales scales_out_dev [rows][cols/128] (every one equal to gamma in
 * PER_TENSOR mode).  workspace_dev (>= bitnet_ternarize_workspace_bytes,
 * 16-byte aligned, contents ignored) is caller-owned scratch; the per-tensor
 * reduction runs in a fixed order, so results are reproducible bit for bit.
 * Errors: NULL, SHAPE, ALIGN, BUFSIZE, VALUE (unknown mode), CUDA. */
bitnet_status bitnet_ternarize_absmean_device(const float *w_dev, int64_t rows, int64_t cols, int mode,
                                              uint8_t *codes_out_dev, float *scales_out_dev,
                                              void *workspace_dev, size_t workspace_bytes,
                                              bitnet_stream_t stream);

/* Same as bitnet_ternarize_absmean_device, for callers that cannot allocate
 * device memory: no workspace argument.  The pages have no counterpart; this
 * entry point exists because some callers cannot hand the library scratch
 * memory -- a host whose own fixed pool already owns all device memory, a
 * binding with no device allocator, or a serving loop that must not call
 * cudaMalloc (it may synchronise the device).  The scratch instead lives in a
 * static device array inside the library, 2048 * 8 + 256 = 16640 bytes, which
 * every GPU that loads the library keeps until the process exits; a request
 * needing more (none with today's fixed reduction grid) is refused with
 * BITNET_ERR_BUFSIZE.  The array is shared by all calls on a device and keeps
 * the last call's contents (nothing in it has to start at zero): calls that
 * overlap on the GPU -- on different streams, or from different host
 * threads -- race on it and must be serialised by the caller.  The first call
 * on each device looks the array's address up (cudaGetSymbolAddress, with
 * that device current) and caches it; make that first call before any stream
 * capture.  Calls no cudaMalloc, cudaFree or allocating library routine.
 * Errors: as bitnet_ternarize_absmean_device, plus BUFSIZE as above and CUDA
 * if the address lookup fails. */
bitnet_status bitnet_ternarize_absmean_device_noalloc(const float *w_dev, int64_t rows, int64_t cols, int mode,
                                                      uint8_t *codes_out_dev, float *scales_out_dev,
                                                      bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Device weights.
 * ---------------------------------------------------------------------- */

#define BITNET_LAYOUT_VERSION 1u
/* flags filled in by bitnet_repack_device */
#define BITNET_WEIGHT_UNIFORM_ROWS 1u /* every row's block scales are equal */

typedef struct {
    int64_t rows;            /* out */
    int64_t cols;            /* K, multiple of 128 */
    void *data;              /* device, caller-owned, 256-byte aligned     */
    size_t bytes;            /* >= bitnet_repacked_bytes(rows, cols)       */
    uint32_t layout_version; /* BITNET_LAYOUT_VERSION after a repack       */
    uint32_t flags;          /* BITNET_WEIGHT_* after a repack             */
} bitnet_weight;

/* Converts i2_s codes [rows][cols/4] and block scales [rows][cols/128]
 * (both device memory, left unchanged) into the kernels' device layout in
 * w_out->data: 16-row x 128-column tiles of codes in the order the GEMV and
 * GEMM kernels read them, the block scales per tile, and one scale per row
 * when all of that row's block scales are equal.  The caller sets
 * w_out->data and w_out->bytes; rows, cols, layout_version and flags are
 * written here.  This call is once per weight and is SYNCHRONOUS: it waits
 * for `stream` to read back the uniformity flag and the corruption check.
 * codes_dev must be 4-byte aligned, scales_dev 4-byte aligned.
 * Errors: NULL, SHAPE, ALIGN, BUFSIZE, CORRUPT (code 3 found; w_out is then
 * unusable), CUDA. */
bitnet_status bitnet_repack_device(const uint8_t *codes_dev, const float *scales_dev,
                                   int64_t rows, int64_t cols, bitnet_weight *w_out,
                                   bitnet_stream_t stream);

/* Inverse of bitnet_repack_device (async): rewrites the i2_s codes
 * [rows][cols/4] and block scales [rows][cols/128] from a repacked weight.
 * Lets a caller check the device layout byte for byte. */
bitnet_status bitnet_unrepack_device(const bitnet_weight *w, uint8_t *codes_out_dev,
                                     float *scales_out_dev, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Activation quantisation (async).
 * ---------------------------------------------------------------------- */

/* Per-row absmax int8 quantisation of fp32 x [T][K]:
 *   s[t] = 127 / max(max_k |x[t][k]|, 1e-5)      (fp32, IEEE divide)
 *   q[t][k] = clamp(rint(x[t][k] * s[t]), -127, 127)   (ties to even)
 * q_dev receives T*K int8 (16-byte aligned), s_dev T fp32 (4-byte aligned).
 * blocksum_dev (nullable, 4-byte aligned) receives T*(K/128) int32 sums of q
 * over each 128-element block.  T may be 0 (nothing is launched).
 * Errors: NULL, SHAPE, ALIGN, CUDA. */
bitnet_status bitnet_quant_act(const float *x_dev, int64_t T, int64_t K, int8_t *q_dev,
                               float *s_dev, int32_t *blocksum_dev, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * The linear layer (async).
 * ---------------------------------------------------------------------- */

/* Decode / small-batch GEMV, 1 <= B <= 64:
 *   y[b][o] = (sum_j scale[o][j] * acc[b][o][j]) / s[b]
 * with acc the int32 block dot products of the ternary weights and q.
 * q_dev: B*K int8 (16-byte aligned); s_dev: B fp32; y_dev: B*rows fp32
 * (4-byte aligned).  The int32 sums are exact.  Kernels and epilogues:
 *   - weights with uniform rows (BITNET_WEIGHT_UNIFORM_ROWS, the per-tensor
 *     absmean case): y = scale * acc * (1/s) in fp32 (three roundings, within
 *     2.4e-7 relative of the fp64 value), bit for bit the same for every B:
 *     B = 1 and K <= 16384 the batch-1 decode kernel (dp4a); B = 2..4 and
 *     K <= 16384 the batched decode kernel (dp4a); B >= 5 the tensor-core
 *     kernel (warp-level int8 MMA, mma.sync m16n8k32, with the repacked code
 *     tiles as its A fragments; K split over a thread block cluster);
 *     otherwise the general kernel;
 *   - other weights: the sum over blocks runs in fp64 and is rounded once
 *     (the general kernel, exact for B <= 16; the GEMM's block-scale path,
 *     y = fp32(sum * (1/s)), for B > 16).
 * Errors: NULL, SHAPE (B outside 1..64, K mismatch), ALIGN, VALUE (w not
 * repacked), CUDA.  Bounded device waits that run out latch
 * BITNET_ERR_TIMEOUT.
 * The GEMV, the fused linear and the quantiser use programmatic dependent
 * launch: a GEMV may start reading its (constant) weights while the kernel
 * before it on the stream is still running, and reads q, s (or x) and writes
 * y only after that kernel has finished.  Weights are never written by the
 * library's own kernels after bitnet_repack_device returns. */
bitnet_status bitnet_w2a8_gemv(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev,
                               int64_t B, float *y_dev, bitnet_stream_t stream);

/* Decode linear layer, 1 <= B <= 64: quantises fp32 x [B][K] exactly as
 * bitnet_quant_act does, then computes what bitnet_w2a8_gemv computes.
 * x_dev: B*K fp32 (16-byte aligned); y_dev: B*rows fp32.  q_out_dev (B*K
 * int8) and s_out_dev (B fp32) are optional at B <= 16 (NULL = not written)
 * and receive the quantised activations.
 *   - Without q_out_dev / s_out_dev (B <= 16): ONE kernel; every CTA
 *     re-quantises x into shared memory, no global round trip of q.  B = 1 on
 *     uniform rows with K <= 16384 is the batch-1 decode kernel (fp32
 *     epilogue); otherwise the general kernel (fp64 epilogue).
 *   - With both (required for B > 16; q_out_dev then 16-byte aligned): the
 *     quantiser writes them, and the GEMV of bitnet_w2a8_gemv reads them (two
 *     kernels, the second overlapping its weight fetch with the first): the
 *     tensor-core kernel for uniform rows from B = 5 on.
 * Errors: NULL (B > 16 without q_out_dev / s_out_dev), SHAPE, ALIGN, VALUE,
 * BUFSIZE, CUDA; BITNET_ERR_TIMEOUT is latched as for the GEMV. */
bitnet_status bitnet_w2a8_linear(const bitnet_weight *w, const float *x_dev, int64_t B, float *y_dev,
                                 int8_t *q_out_dev, float *s_out_dev, bitnet_stream_t stream);

/* Linear layer for any token count T >= 1 (prefill): quantises fp32 x
 * [T][K] exactly as bitnet_quant_act does into q_out_dev / s_out_dev
 * (required), then computes y [T][rows] as bitnet_w2a8_gemm (T > 64) or
 * bitnet_w2a8_linear (T <= 64) does, bit for bit.  With a workspace of
 * bitnet_w2a8_gemm_workspace_bytes(rows, cols) (or NULL), on uniform rows
 * from 256 tokens and K <= 32768, ONE kernel quantises x and expands the
 * weights into the workspace side by side, then the GEMM of
 * bitnet_w2a8_gemm_ws runs; otherwise the quantiser, then the GEMM.
 * x_dev, y_dev, q_out_dev: 16-byte aligned; s_out_dev 4; workspace_dev 256
 * (caller owned, stream ordered as for bitnet_w2a8_gemm_ws).
 * Errors: NULL, SHAPE, ALIGN, VALUE, BUFSIZE (workspace), UNSUPPORTED (T > 64
 * on a device that is not sm_100), CUDA; bounded device waits latch
 * BITNET_ERR_TIMEOUT. */
bitnet_status bitnet_w2a8_linear_ws(const bitnet_weight *w, const float *x_dev, int64_t T, float *y_dev,
                                    int8_t *q_out_dev, float *s_out_dev, void *workspace_dev, size_t workspace_bytes,
                                    bitnet_stream_t stream);

/* A sequence of batch-1 decode linears in ONE persistent kernel.  Each entry
 * computes exactly what bitnet_w2a8_linear computes with B = 1 on uniform rows
 * (same q, s, int32 sums and fp32 epilogue, bit for bit): per-token absmax
 * int8 quantisation of x ("5倍性能跃升：BitNet与llama.cpp的1-bit LLM推理架构
 * 对决", section "GPU内核突破": 8-bit activations, 2-bit weights), the
 * integer add / subtract / skip product ("BitRun v0.2 实测", section
 * "三值权重与 1.58-bit 的由来") and y = rowscale * sum * (1/s).  Batch-1
 * decode reads every weight once and is bound by memory bandwidth ("浏览器里跑
 * 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操", section "为什么是 WASM");
 * one kernel for the whole list keeps the weights streaming from HBM with no
 * gap between linears, where one launch per linear pays a launch, an
 * activation phase and a tail each.
 *
 * wait_for = -1: x is ready when the call is enqueued (it may be written by
 * earlier work on `stream`).  wait_for = j (0 <= j < this entry's index): x is
 * (part of) the y of entry j, and this linear's products wait, on the device,
 * until every output of entry j is written.  Linears that wait for nothing
 * run concurrently; a chain of waits runs one linear after another.
 * Performance note: each wait is a grid-wide hand-off through global memory
 * (about 4.5 us per dependent linear on a B200, measured); for a pure chain
 * (every entry waits for the one before it) one bitnet_w2a8_linear call per
 * entry on one stream, whose kernels overlap their starts under programmatic
 * dependent launch, is faster today (about 2.9 us per linear).  Lists whose
 * entries are mostly independent of each other run fastest here.
 * Memory rules (checked on the host; BITNET_ERR_VALUE otherwise): no two y
 * ranges overlap, and an x range may overlap a y range only of an entry it
 * waits for directly or through a chain of waits, or of an entry that waits
 * (directly or through a chain) for it (in-place reuse of a buffer once read).
 * w: repacked, BITNET_WEIGHT_UNIFORM_ROWS, cols <= BITNET_SEQ_MAX_COLS; x_dev
 * [cols] fp32, 16-byte aligned; y_dev [rows] fp32, 4-byte aligned.
 * workspace_dev: device memory of at least
 * bitnet_w2a8_linear_seq_workspace_bytes(n) bytes, 4-byte aligned, caller
 * owned, ZERO-FILLED before its first use; every call leaves it zeroed.  It
 * may be NULL (and workspace_bytes 0) when no entry waits.  Calls that share
 * a workspace must not overlap on the GPU.  A call with waits is a
 * cooperative launch (one CTA per SM, all resident); it fails with
 * BITNET_ERR_CUDA if the device cannot co-schedule them.  A call without
 * waits is a programmatic dependent launch: its set-up and first weight
 * copies may start while the previous kernel on `stream` finishes, and it
 * reads x, writes y and touches the workspace only after that kernel is
 * complete, so stream order holds as for any launch.
 * Errors: NULL, SHAPE (n outside 1..BITNET_SEQ_MAX_LINEARS), ALIGN, VALUE
 * (bad wait_for, not repacked, overlapping buffers), UNSUPPORTED (rows not
 * uniform, or cols > BITNET_SEQ_MAX_COLS), BUFSIZE (workspace), CUDA.  Bounded
 * device waits (copies, producers) that run out latch BITNET_ERR_TIMEOUT. */
#define BITNET_SEQ_MAX_LINEARS 256
#define BITNET_SEQ_MAX_COLS 16384

typedef struct {
    const bitnet_weight *w;
    const float *x_dev;
    float *y_dev;
    int32_t wait_for;
} bitnet_linear_desc;

size_t bitnet_w2a8_linear_seq_workspace_bytes(int32_t n);

bitnet_status bitnet_w2a8_linear_seq(const bitnet_linear_desc *list, int32_t n, void *workspace_dev,
                                     size_t workspace_bytes, bitnet_stream_t stream);

/* Prefill GEMM, T >= 1 tokens, same result as the GEMV (tcgen05 int8
 * tensor cores, int32 accumulators in tensor memory).
 * q_dev: T*K int8 (16-byte aligned); s_dev: T fp32; y_dev: T*rows fp32
 * (16-byte aligned).  T = 0 launches nothing.
 * Errors: NULL, SHAPE, ALIGN, VALUE, UNSUPPORTED (not an sm_100 device),
 * CUDA.  Device-side bounded waits that run out latch BITNET_ERR_TIMEOUT. */
bitnet_status bitnet_w2a8_gemm(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev,
                               int64_t T, float *y_dev, bitnet_stream_t stream);

/* The same GEMM with a caller-owned workspace for the weights expanded to
 * int8.  On uniform rows from 256 tokens the call first expands the packed
 * codes to t = c - 1 bytes, [rows rounded up to 16][cols] row-major, in the
 * workspace (one pass, 4 bytes written per packed byte read), then runs the
 * tcgen05 GEMM with both operands loaded by TMA: each weight is decoded once
 * per call instead of once per 128-token tile.  Same y, bit for bit, as
 * bitnet_w2a8_gemm.  Below 256 tokens, on block-scale weights, or with
 * workspace_dev NULL it is bitnet_w2a8_gemm.
 * workspace_dev: device memory of at least
 * bitnet_w2a8_gemm_workspace_bytes(rows, cols) bytes, 256-byte aligned,
 * caller owned, contents undefined between calls; calls that share it must
 * be stream ordered (the expansion waits for the previous kernel on `stream`
 * before it writes).  Errors: those of bitnet_w2a8_gemm, ALIGN (workspace),
 * BUFSIZE (workspace too small). */
size_t bitnet_w2a8_gemm_workspace_bytes(int64_t rows, int64_t cols);
bitnet_status bitnet_w2a8_gemm_ws(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev, int64_t T,
                                  float *y_dev, void *workspace_dev, size_t workspace_bytes,
                                  bitnet_stream_t stream);

/* Table-lookup variant of bitnet_w2a8_gemv at B = 1, kept for comparison with
 * the dp4a kernels: the CPU kernels of "浏览器里跑 1-bit 大模型 BitNet
 * WebAssembly 的 50 倍提速实操" (section "查表（LUT）内核") replace products by
 * lookups of precomputed activation sub-sums indexed by weight codes; here
 * each CTA builds, per 128-weight block and byte position, two 16-entry int16
 * tables over the two weights of a nibble and sums two lookups per byte.
 * Same arguments and y as bitnet_w2a8_gemv with B = 1 (fp32 epilogue of the
 * decode kernel).  Errors: NULL, ALIGN, VALUE, UNSUPPORTED (weights without
 * uniform rows, or K > 8192), CUDA; copy-wait timeouts latch
 * BITNET_ERR_TIMEOUT. */
bitnet_status bitnet_w2a8_gemv_lut(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev,
                                   float *y_dev, bitnet_stream_t stream);

/* Test variants of the two calls above that also write the int32 block
 * accumulators acc_dev[b][o][j], b < B (or T), o < rows, j < cols/128
 * (4-byte aligned), so they can be compared bit for bit. */
bitnet_status bitnet_w2a8_gemv_acc(const bitnet_weight *w, const int8_t *q_dev,
                                   const float *s_dev, int64_t B, float *y_dev,
                                   int32_t *acc_dev, bitnet_stream_t stream);
bitnet_status bitnet_w2a8_linear_acc(const bitnet_weight *w, const float *x_dev, int64_t B, float *y_dev,
                                     int8_t *q_out_dev, float *s_out_dev, int32_t *acc_dev,
                                     bitnet_stream_t stream);
bitnet_status bitnet_w2a8_gemm_acc(const bitnet_weight *w, const int8_t *q_dev,
                                   const float *s_dev, int64_t T, float *y_dev,
                                   int32_t *acc_dev, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Device-side error reporting.
 * ---------------------------------------------------------------------- */

/* Waits for `stream`, then reads and clears the current device's error word:
 * BITNET_OK, BITNET_ERR_TIMEOUT (a bounded wait ran out), BITNET_ERR_CORRUPT
 * (a kernel met code 3) or BITNET_ERR_CUDA (the stream itself failed). */
bitnet_status bitnet_get_device_error(bitnet_stream_t stream);

/* Test hook: sets the iteration cap of the device-side bounded waits on the
 * current device (0 restores the default).  A tiny cap makes a wait run out
 * without hanging anything, so the timeout path can be exercised. */
bitnet_status bitnet_set_wait_limit(uint32_t max_iterations);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_W2A8_H */
