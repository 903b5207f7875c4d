// abi.cu -- the extern "C" entry points of libbitnet_w2a8.so: host-side
// validation, dispatch to the kernels, status reporting, and the host i2_s
// packer.  Declarations and their documentation: include/bitnet_w2a8.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace bitnet {

__device__ unsigned g_error_word = 0u;
__device__ unsigned g_wait_limit = kDefaultWaitLimit;

namespace {

thread_local char t_detail[256] = "";

bitnet_status fail(bitnet_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
bitnet_status fail(bitnet_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_detail, sizeof(t_detail), fmt, ap);
    va_end(ap);
    return st;
}

bitnet_status cuda_fail(cudaError_t e, const char *what) {
    return fail(BITNET_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

constexpr int64_t kMaxCols = int64_t(1) << 20;
constexpr int64_t kMaxRows = int64_t(1) << 31;
constexpr int64_t kMaxT = int64_t(1) << 31;

bool shape_ok(int64_t rows, int64_t cols) {
    return rows >= 0 && cols >= 0 && cols % kQK == 0 && rows < kMaxRows && cols <= kMaxCols;
}

std::mutex g_mu;
DeviceGlobals g_dev[64];
bool g_dev_ok[64];

bitnet_status check_weight(const bitnet_weight *w) {
    if (!w) return fail(BITNET_ERR_NULL, "weight handle is NULL");
    if (!w->data) return fail(BITNET_ERR_NULL, "weight data is NULL");
    if (!shape_ok(w->rows, w->cols) || w->rows == 0 || w->cols == 0)
        return fail(BITNET_ERR_SHAPE, "weight shape %lld x %lld invalid", (long long)w->rows,
                    (long long)w->cols);
    if (w->layout_version != BITNET_LAYOUT_VERSION)
        return fail(BITNET_ERR_VALUE, "weight not repacked (layout_version %u)", w->layout_version);
    if (!aligned(w->data, 256)) return fail(BITNET_ERR_ALIGN, "weight data not 256-byte aligned");
    if (w->bytes < layout_of(w->rows, w->cols).total)
        return fail(BITNET_ERR_BUFSIZE, "weight buffer %zu bytes, need %zu", w->bytes,
                    layout_of(w->rows, w->cols).total);
    return BITNET_OK;
}

}  // namespace

bitnet_status set_error_detail(bitnet_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_detail, sizeof(t_detail), fmt, ap);
    va_end(ap);
    return st;
}

cudaError_t device_globals(DeviceGlobals *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev_ok[dev]) {
        DeviceGlobals g;
        e = cudaGetSymbolAddress((void **)&g.err, g_error_word);
        if (e != cudaSuccess) return e;
        e = cudaGetSymbolAddress((void **)&g.wait_limit, g_wait_limit);
        if (e != cudaSuccess) return e;
        g_dev[dev] = g;
        g_dev_ok[dev] = true;
    }
    *out = g_dev[dev];
    return cudaSuccess;
}

int num_sms() {
    static std::atomic<int> n[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int v = n[dev].load(std::memory_order_relaxed);
    if (!v) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        n[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

}  // namespace bitnet

using namespace bitnet;

extern "C" {

const char *bitnet_status_string(bitnet_status s) {
    switch (s) {
        case BITNET_OK: return "BITNET_OK";
        case BITNET_ERR_NULL: return "BITNET_ERR_NULL";
        case BITNET_ERR_SHAPE: return "BITNET_ERR_SHAPE";
        case BITNET_ERR_ALIGN: return "BITNET_ERR_ALIGN";
        case BITNET_ERR_VALUE: return "BITNET_ERR_VALUE";
        case BITNET_ERR_CORRUPT: return "BITNET_ERR_CORRUPT";
        case BITNET_ERR_BUFSIZE: return "BITNET_ERR_BUFSIZE";
        case BITNET_ERR_CUDA: return "BITNET_ERR_CUDA";
        case BITNET_ERR_TIMEOUT: return "BITNET_ERR_TIMEOUT";
        case BITNET_ERR_UNSUPPORTED: return "BITNET_ERR_UNSUPPORTED";
    }
    return "BITNET_ERR_UNKNOWN";
}

const char *bitnet_last_error_detail(void) { return t_detail; }

uint32_t bitnet_version(void) { return (1u << 16) | 0u; }

size_t bitnet_i2s_code_bytes(int64_t rows, int64_t cols) {
    return shape_ok(rows, cols) ? (size_t)rows * (size_t)cols / 4 : 0;
}

size_t bitnet_i2s_num_scales(int64_t rows, int64_t cols) {
    return shape_ok(rows, cols) ? (size_t)rows * (size_t)(cols / kQK) : 0;
}

size_t bitnet_repacked_bytes(int64_t rows, int64_t cols) {
    return shape_ok(rows, cols) ? layout_of(rows, cols).total : 0;
}

// Host packer.  Byte (block*32 + i%32) of a row gets the code of weight i of
// the block at shift 6 - 2*(i/32); the codes of a byte are gathered first so
// every byte is written once.
bitnet_status bitnet_pack_i2s(const int8_t *ternary, int64_t rows, int64_t cols,
                              uint8_t *codes_out, size_t codes_bytes) {
    t_detail[0] = 0;
    if (!ternary || !codes_out) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!shape_ok(rows, cols)) return fail(BITNET_ERR_SHAPE, "bad shape");
    const size_t need = (size_t)rows * (size_t)cols / 4;
    if (codes_bytes < need) return fail(BITNET_ERR_BUFSIZE, "codes buffer %zu < %zu", codes_bytes, need);
    for (int64_t r = 0; r < rows; r++) {
        const int8_t *src = ternary + r * cols;
        uint8_t *dst = codes_out + r * (cols / 4);
        for (int64_t blk = 0; blk < cols / kQK; blk++) {
            const int8_t *w = src + blk * kQK;
            for (int b = 0; b < 32; b++) {
                unsigned byte = 0;
                for (int grp = 0; grp < 4; grp++) {
                    const int v = w[grp * 32 + b];
                    if (v != -1 && v != 0 && v != 1)
                        return fail(BITNET_ERR_VALUE, "value %d at row %lld col %lld is not ternary", v,
                                    (long long)r, (long long)(blk * kQK + grp * 32 + b));
                    byte |= (unsigned)(v + 1) << (6 - 2 * grp);
                }
                dst[blk * 32 + b] = (uint8_t)byte;
            }
        }
    }
    return BITNET_OK;
}

bitnet_status bitnet_unpack_i2s(const uint8_t *codes, int64_t rows, int64_t cols,
                                int8_t *ternary_out, size_t ternary_bytes) {
    t_detail[0] = 0;
    if (!codes || !ternary_out) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!shape_ok(rows, cols)) return fail(BITNET_ERR_SHAPE, "bad shape");
    const size_t need = (size_t)rows * (size_t)cols;
    if (ternary_bytes < need) return fail(BITNET_ERR_BUFSIZE, "output buffer %zu < %zu", ternary_bytes, need);
    for (int64_t r = 0; r < rows; r++) {
        const uint8_t *src = codes + r * (cols / 4);
        int8_t *dst = ternary_out + r * cols;
        for (int64_t blk = 0; blk < cols / kQK; blk++) {
            for (int b = 0; b < 32; b++) {
                const unsigned byte = src[blk * 32 + b];
                for (int grp = 0; grp < 4; grp++) {
                    const unsigned c = (byte >> (6 - 2 * grp)) & 3u;
                    if (c == 3u)
                        return fail(BITNET_ERR_CORRUPT, "code 3 at row %lld byte %lld", (long long)r,
                                    (long long)(blk * 32 + b));
                    dst[blk * kQK + grp * 32 + b] = (int8_t)((int)c - 1);
                }
            }
        }
    }
    return BITNET_OK;
}

size_t bitnet_ternarize_workspace_bytes(int64_t rows, int64_t cols) {
    if (!shape_ok(rows, cols)) return 0;
    return (size_t)absmean_num_partials(rows * cols) * sizeof(double) + 256;
}

bitnet_status bitnet_ternarize_absmean_device(const float *w_dev, int64_t rows, int64_t cols, int mode,
                                              uint8_t *codes_out_dev, float *scales_out_dev,
                                              void *workspace_dev, size_t workspace_bytes,
                                              bitnet_stream_t stream) {
    t_detail[0] = 0;
    if (!shape_ok(rows, cols)) return fail(BITNET_ERR_SHAPE, "shape %lld x %lld invalid", (long long)rows,
                                           (long long)cols);
    if (mode != BITNET_ABSMEAN_PER_TENSOR && mode != BITNET_ABSMEAN_PER_BLOCK)
        return fail(BITNET_ERR_VALUE, "unknown mode %d", mode);
    if (rows == 0 || cols == 0) return BITNET_OK;
    if (!w_dev || !codes_out_dev || !scales_out_dev || !workspace_dev) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!aligned(w_dev, 4) || !aligned(codes_out_dev, 4) || !aligned(scales_out_dev, 4) ||
        !aligned(workspace_dev, 16))
        return fail(BITNET_ERR_ALIGN, "w/codes/scales need 4-byte, workspace 16-byte alignment");
    const size_t need = bitnet_ternarize_workspace_bytes(rows, cols);
    if (workspace_bytes < need) return fail(BITNET_ERR_BUFSIZE, "workspace %zu < %zu bytes", workspace_bytes, need);
    double *partials = static_cast<double *>(workspace_dev);
    float *gamma_slot = reinterpret_cast<float *>(static_cast<char *>(workspace_dev) + need - 256);
    cudaError_t e = launch_ternarize(w_dev, rows, cols, mode == BITNET_ABSMEAN_PER_BLOCK,
                                     reinterpret_cast<uint32_t *>(codes_out_dev), scales_out_dev, partials,
                                     gamma_slot, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "ternarize launch");
}

bitnet_status bitnet_repack_device(const uint8_t *codes_dev, const float *scales_dev, int64_t rows,
                                   int64_t cols, bitnet_weight *w_out, bitnet_stream_t stream) {
    t_detail[0] = 0;
    if (!codes_dev || !scales_dev || !w_out || !w_out->data) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!shape_ok(rows, cols) || rows == 0 || cols == 0)
        return fail(BITNET_ERR_SHAPE, "shape %lld x %lld invalid", (long long)rows, (long long)cols);
    if (!aligned(codes_dev, 4) || !aligned(scales_dev, 4) || !aligned(w_out->data, 256))
        return fail(BITNET_ERR_ALIGN, "codes/scales need 4-byte, data 256-byte alignment");
    const Layout L = layout_of(rows, cols);
    if (w_out->bytes < L.total) return fail(BITNET_ERR_BUFSIZE, "data %zu < %zu bytes", w_out->bytes, L.total);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    w_out->layout_version = 0;
    w_out->flags = 0;
    cudaError_t e = launch_repack(codes_dev, scales_dev, rows, cols, w_out->data, st);
    if (e != cudaSuccess) return cuda_fail(e, "repack launch");
    unsigned hdr[2] = {0u, 0u};
    e = cudaMemcpyAsync(hdr, w_out->data, sizeof(hdr), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "repack readback");
    if (hdr[1]) return fail(BITNET_ERR_CORRUPT, "packed codes hold code 3");
    w_out->rows = rows;
    w_out->cols = cols;
    w_out->flags = hdr[0] == 0u ? BITNET_WEIGHT_UNIFORM_ROWS : 0u;
    w_out->layout_version = BITNET_LAYOUT_VERSION;
    return BITNET_OK;
}

bitnet_status bitnet_unrepack_device(const bitnet_weight *w, uint8_t *codes_out_dev,
                                     float *scales_out_dev, bitnet_stream_t stream) {
    t_detail[0] = 0;
    bitnet_status s = check_weight(w);
    if (s != BITNET_OK) return s;
    if (!codes_out_dev || !scales_out_dev) return fail(BITNET_ERR_NULL, "NULL output");
    if (!aligned(codes_out_dev, 4) || !aligned(scales_out_dev, 4))
        return fail(BITNET_ERR_ALIGN, "outputs need 4-byte alignment");
    cudaError_t e = launch_unrepack(w->data, w->rows, w->cols, codes_out_dev, scales_out_dev,
                                    reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "unrepack launch");
}

bitnet_status bitnet_quant_act(const float *x_dev, int64_t T, int64_t K, int8_t *q_dev, float *s_dev,
                               int32_t *blocksum_dev, bitnet_stream_t stream) {
    t_detail[0] = 0;
    if (T < 0 || T >= kMaxT || K <= 0 || K % kQK != 0 || K > kMaxCols)
        return fail(BITNET_ERR_SHAPE, "T=%lld K=%lld invalid", (long long)T, (long long)K);
    if (T == 0) return BITNET_OK;
    if (!x_dev || !q_dev || !s_dev) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!aligned(x_dev, 16) || !aligned(q_dev, 16) || !aligned(s_dev, 4) ||
        (blocksum_dev && !aligned(blocksum_dev, 4)))
        return fail(BITNET_ERR_ALIGN, "x and q need 16-byte, s and blocksum 4-byte alignment");
    cudaError_t e = launch_quant_act(x_dev, T, K, q_dev, s_dev, blocksum_dev,
                                     reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "quant_act launch");
}

// Device work of a GEMV on given q, s: the warp-MMA kernel for uniform rows
// from kMmaMinBatch tokens, the decode / general kernels up to 16 tokens,
// the GEMM's block-scale path (per-block fp64 sums) beyond.
static cudaError_t gemv_dispatch(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev, int64_t B,
                                 float *y_dev, int32_t *acc_dev, const DeviceGlobals &g, cudaStream_t st) {
    const bool uniform = (w->flags & BITNET_WEIGHT_UNIFORM_ROWS) != 0;
    if (uniform && !acc_dev && B >= kMmaMinBatch && gemv_mma_supported(w->rows, w->cols, B))
        return launch_gemv_mma(w->data, w->rows, w->cols, q_dev, s_dev, B, y_dev, st);
    if (B <= 16)
        return launch_gemv(w->data, w->rows, w->cols, uniform, q_dev, s_dev, B, y_dev, acc_dev, nullptr, nullptr,
                           nullptr, g, st);
    return launch_gemm(w->data, w->rows, w->cols, false, q_dev, s_dev, B, y_dev, acc_dev, g, st);
}

static bitnet_status gemv_impl(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev,
                               int64_t B, float *y_dev, int32_t *acc_dev, bitnet_stream_t stream) {
    t_detail[0] = 0;
    bitnet_status s = check_weight(w);
    if (s != BITNET_OK) return s;
    if (B < 1 || B > 64) return fail(BITNET_ERR_SHAPE, "GEMV batch %lld outside 1..64", (long long)B);
    if (!q_dev || !s_dev || !y_dev) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!aligned(q_dev, 16) || !aligned(s_dev, 4) || !aligned(y_dev, 4) || (acc_dev && !aligned(acc_dev, 4)))
        return fail(BITNET_ERR_ALIGN, "q needs 16-byte, s/y/acc 4-byte alignment");
    DeviceGlobals g;
    cudaError_t e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    e = gemv_dispatch(w, q_dev, s_dev, B, y_dev, acc_dev, g, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemv launch");
}

static bitnet_status linear_impl(const bitnet_weight *w, const float *x_dev, int64_t B, float *y_dev,
                                 int8_t *q_out_dev, float *s_out_dev, int32_t *acc_dev, bitnet_stream_t stream) {
    t_detail[0] = 0;
    bitnet_status s = check_weight(w);
    if (s != BITNET_OK) return s;
    if (B < 1 || B > 64) return fail(BITNET_ERR_SHAPE, "linear batch %lld outside 1..64", (long long)B);
    if (!x_dev || !y_dev) return fail(BITNET_ERR_NULL, "NULL pointer");
    const bool staged = B >= 2 && q_out_dev && s_out_dev;
    if (B > 16 && !staged)
        return fail(BITNET_ERR_NULL, "linear batch %lld > 16 needs q_out and s_out", (long long)B);
    if (!aligned(x_dev, 16) || !aligned(y_dev, 4) || (q_out_dev && !aligned(q_out_dev, staged ? 16 : 4)) ||
        (s_out_dev && !aligned(s_out_dev, 4)) || (acc_dev && !aligned(acc_dev, 4)))
        return fail(BITNET_ERR_ALIGN, "x needs 16-byte, y/s_out/acc 4-byte, q_out 4-byte (16 from B = 2 "
                                      "with s_out) alignment");
    DeviceGlobals g;
    cudaError_t e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (staged) {
        // Two kernels: the quantiser into the caller's q_out / s_out, then the
        // GEMV on them (programmatic dependent launch overlaps the GEMV's
        // weight fetch with the quantiser).
        e = launch_quant_act(x_dev, B, w->cols, q_out_dev, s_out_dev, nullptr, st);
        if (e == cudaSuccess) e = gemv_dispatch(w, q_out_dev, s_out_dev, B, y_dev, acc_dev, g, st);
        return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "linear launch");
    }
    e = launch_gemv(w->data, w->rows, w->cols, (w->flags & BITNET_WEIGHT_UNIFORM_ROWS) != 0, nullptr, nullptr, B,
                    y_dev, acc_dev, x_dev, q_out_dev, s_out_dev, g, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "linear launch");
}

bitnet_status bitnet_w2a8_linear(const bitnet_weight *w, const float *x_dev, int64_t B, float *y_dev,
                                 int8_t *q_out_dev, float *s_out_dev, bitnet_stream_t stream) {
    return linear_impl(w, x_dev, B, y_dev, q_out_dev, s_out_dev, nullptr, stream);
}

bitnet_status bitnet_w2a8_linear_acc(const bitnet_weight *w, const float *x_dev, int64_t B, float *y_dev,
                                     int8_t *q_out_dev, float *s_out_dev, int32_t *acc_dev,
                                     bitnet_stream_t stream) {
    if (!acc_dev) return fail(BITNET_ERR_NULL, "acc is NULL");
    return linear_impl(w, x_dev, B, y_dev, q_out_dev, s_out_dev, acc_dev, stream);
}

bitnet_status bitnet_w2a8_linear_ws(const bitnet_weight *w, const float *x_dev, int64_t T, float *y_dev,
                                    int8_t *q_out_dev, float *s_out_dev, void *workspace_dev, size_t workspace_bytes,
                                    bitnet_stream_t stream) {
    t_detail[0] = 0;
    bitnet_status s = check_weight(w);
    if (s != BITNET_OK) return s;
    if (T < 1 || T >= kMaxT) return fail(BITNET_ERR_SHAPE, "T=%lld invalid", (long long)T);
    if (!x_dev || !y_dev || !q_out_dev || !s_out_dev) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!aligned(x_dev, 16) || !aligned(y_dev, 16) || !aligned(q_out_dev, 16) || !aligned(s_out_dev, 4))
        return fail(BITNET_ERR_ALIGN, "x, y and q_out need 16-byte, s_out 4-byte alignment");
    if (workspace_dev) {
        if (!aligned(workspace_dev, 256)) return fail(BITNET_ERR_ALIGN, "workspace needs 256-byte alignment");
        if (workspace_bytes < gemm_expanded_bytes(w->rows, w->cols))
            return fail(BITNET_ERR_BUFSIZE, "workspace %zu < %zu bytes", workspace_bytes,
                        gemm_expanded_bytes(w->rows, w->cols));
    }
    if (T <= 64) return linear_impl(w, x_dev, T, y_dev, q_out_dev, s_out_dev, nullptr, stream);
    int dev = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    if (major != 10) return fail(BITNET_ERR_UNSUPPORTED, "GEMM needs an sm_100 device (found sm_%d)", major * 10);
    DeviceGlobals g;
    e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool uniform = (w->flags & BITNET_WEIGHT_UNIFORM_ROWS) != 0;
    int8_t *ws = static_cast<int8_t *>(workspace_dev);
    if (uniform && ws && T >= kGemmExpandMinT && prefill_prep_supported(w->cols)) {
        // One kernel quantises x and expands the weights side by side, then
        // the pair-of-SMs GEMM.
        e = launch_prefill_prep(x_dev, T, w->cols, q_out_dev, s_out_dev, w->data, w->rows, ws, st);
        if (e == cudaSuccess)
            e = launch_gemm_pair(w->data, w->rows, w->cols, q_out_dev, s_out_dev, T, y_dev, ws, g, st);
    } else {
        e = launch_quant_act(x_dev, T, w->cols, q_out_dev, s_out_dev, nullptr, st);
        if (e == cudaSuccess)
            e = launch_gemm(w->data, w->rows, w->cols, uniform, q_out_dev, s_out_dev, T, y_dev, nullptr, g, st, ws);
    }
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "linear_ws launch");
}

bitnet_status bitnet_w2a8_gemv(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev, int64_t B,
                               float *y_dev, bitnet_stream_t stream) {
    return gemv_impl(w, q_dev, s_dev, B, y_dev, nullptr, stream);
}

bitnet_status bitnet_w2a8_gemv_acc(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev,
                                   int64_t B, float *y_dev, int32_t *acc_dev, bitnet_stream_t stream) {
    if (!acc_dev) return fail(BITNET_ERR_NULL, "acc is NULL");
    return gemv_impl(w, q_dev, s_dev, B, y_dev, acc_dev, stream);
}

bitnet_status bitnet_w2a8_gemv_lut(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev, float *y_dev,
                                   bitnet_stream_t stream) {
    t_detail[0] = 0;
    bitnet_status s = check_weight(w);
    if (s != BITNET_OK) return s;
    if (!q_dev || !s_dev || !y_dev) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!aligned(q_dev, 16) || !aligned(s_dev, 4) || !aligned(y_dev, 4))
        return fail(BITNET_ERR_ALIGN, "q needs 16-byte, s/y 4-byte alignment");
    if (!(w->flags & BITNET_WEIGHT_UNIFORM_ROWS) || w->cols > 8192)
        return fail(BITNET_ERR_UNSUPPORTED, "the table-lookup GEMV takes uniform rows and K <= 8192");
    DeviceGlobals g;
    cudaError_t e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    e = launch_decode_lut(w->data, w->rows, w->cols, q_dev, s_dev, y_dev, g, reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return fail(BITNET_ERR_UNSUPPORTED, "shape not taken by the table-lookup GEMV");
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemv_lut launch");
}

size_t bitnet_w2a8_linear_seq_workspace_bytes(int32_t n) {
    return n >= 1 && n <= kSeqMaxLinears ? seq_workspace_bytes(n) : 0;
}

bitnet_status bitnet_w2a8_linear_seq(const bitnet_linear_desc *list, int32_t n, void *workspace_dev,
                                     size_t workspace_bytes, bitnet_stream_t stream) {
    t_detail[0] = 0;
    if (!list) return fail(BITNET_ERR_NULL, "list is NULL");
    if (n < 1 || n > kSeqMaxLinears) return fail(BITNET_ERR_SHAPE, "n=%d outside 1..%d", n, kSeqMaxLinears);
    static thread_local SeqLinear sl[kSeqMaxLinears];
    static thread_local uint64_t anc[kSeqMaxLinears][kSeqMaxLinears / 64];  // anc[i] bit m: m precedes i
    bool any_wait = false;
    for (int i = 0; i < n; i++) {
        const bitnet_linear_desc &d = list[i];
        bitnet_status s = check_weight(d.w);
        if (s != BITNET_OK) return s;
        if (!(d.w->flags & BITNET_WEIGHT_UNIFORM_ROWS) || d.w->cols > kSeqMaxK)
            return fail(BITNET_ERR_UNSUPPORTED, "entry %d: the sequence kernel takes uniform rows and cols <= %d", i,
                        kSeqMaxK);
        if (!d.x_dev || !d.y_dev) return fail(BITNET_ERR_NULL, "entry %d: NULL x or y", i);
        if (!aligned(d.x_dev, 16) || !aligned(d.y_dev, 4))
            return fail(BITNET_ERR_ALIGN, "entry %d: x needs 16-byte, y 4-byte alignment", i);
        if (d.wait_for < -1 || d.wait_for >= i)
            return fail(BITNET_ERR_VALUE, "entry %d: wait_for %d must be -1 or a lower index", i, d.wait_for);
        sl[i] = SeqLinear{d.w->data, d.w->rows, d.w->cols, d.x_dev, d.y_dev, d.wait_for};
        for (int k = 0; k < kSeqMaxLinears / 64; k++) anc[i][k] = 0;
        if (d.wait_for >= 0) {
            const int j = d.wait_for;
            for (int k = 0; k < kSeqMaxLinears / 64; k++) anc[i][k] = anc[j][k];
            anc[i][j >> 6] |= 1ull << (j & 63);
            any_wait = true;
        }
    }
    // Hazards: y ranges disjoint; x of m may overlap y of i only if one of the
    // two precedes the other through waits.
    auto precedes = [&](int a, int b) { return (anc[b][a >> 6] >> (a & 63)) & 1ull; };
    auto overlap = [](const void *p, size_t pn, const void *q, size_t qn) {
        const uintptr_t a = (uintptr_t)p, b = (uintptr_t)q;
        return a < b + qn && b < a + pn;
    };
    for (int i = 0; i < n; i++) {
        const size_t yi = (size_t)sl[i].rows * 4;
        for (int m = 0; m < n; m++) {
            if (m != i && m < i && overlap(sl[i].y, yi, sl[m].y, (size_t)sl[m].rows * 4))
                return fail(BITNET_ERR_VALUE, "entries %d and %d: y ranges overlap", m, i);
            if (overlap(sl[m].x, (size_t)sl[m].cols * 4, sl[i].y, yi) && !(m != i && (precedes(i, m) || precedes(m, i))))
                return fail(BITNET_ERR_VALUE, "entry %d reads x where entry %d writes y without a wait between them", m,
                            i);
        }
    }
    if (any_wait) {
        if (!workspace_dev) return fail(BITNET_ERR_NULL, "entries wait for others: workspace is NULL");
        if (!aligned(workspace_dev, 4)) return fail(BITNET_ERR_ALIGN, "workspace needs 4-byte alignment");
        if (workspace_bytes < seq_workspace_bytes(n))
            return fail(BITNET_ERR_BUFSIZE, "workspace %zu < %zu bytes", workspace_bytes, seq_workspace_bytes(n));
    }
    DeviceGlobals g;
    cudaError_t e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    e = launch_decode_seq(sl, n, any_wait ? workspace_dev : nullptr, g, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "linear_seq launch");
}

static bitnet_status gemm_impl(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev,
                               int64_t T, float *y_dev, int32_t *acc_dev, bitnet_stream_t stream,
                               void *workspace_dev = nullptr, size_t workspace_bytes = 0) {
    t_detail[0] = 0;
    bitnet_status s = check_weight(w);
    if (s != BITNET_OK) return s;
    if (T < 0 || T >= kMaxT) return fail(BITNET_ERR_SHAPE, "T=%lld invalid", (long long)T);
    if (T == 0) return BITNET_OK;
    if (!q_dev || !s_dev || !y_dev) return fail(BITNET_ERR_NULL, "NULL pointer");
    if (!aligned(q_dev, 16) || !aligned(s_dev, 4) || !aligned(y_dev, 16) || (acc_dev && !aligned(acc_dev, 4)))
        return fail(BITNET_ERR_ALIGN, "q and y need 16-byte, s/acc 4-byte alignment");
    if (workspace_dev) {
        if (!aligned(workspace_dev, 256)) return fail(BITNET_ERR_ALIGN, "workspace needs 256-byte alignment");
        if (workspace_bytes < gemm_expanded_bytes(w->rows, w->cols))
            return fail(BITNET_ERR_BUFSIZE, "workspace %zu < %zu bytes", workspace_bytes,
                        gemm_expanded_bytes(w->rows, w->cols));
    }
    int dev = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    if (major != 10) return fail(BITNET_ERR_UNSUPPORTED, "GEMM needs an sm_100 device (found sm_%d)", major * 10);
    DeviceGlobals g;
    e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    e = launch_gemm(w->data, w->rows, w->cols, (w->flags & BITNET_WEIGHT_UNIFORM_ROWS) != 0, q_dev, s_dev,
                    T, y_dev, acc_dev, g, reinterpret_cast<cudaStream_t>(stream),
                    static_cast<int8_t *>(workspace_dev));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemm launch");
}

bitnet_status bitnet_w2a8_gemm(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev, int64_t T,
                               float *y_dev, bitnet_stream_t stream) {
    return gemm_impl(w, q_dev, s_dev, T, y_dev, nullptr, stream);
}

size_t bitnet_w2a8_gemm_workspace_bytes(int64_t rows, int64_t cols) {
    if (rows < 1 || cols < kQK || cols % kQK != 0 || rows > kMaxRows || cols > kMaxCols) return 0;
    return gemm_expanded_bytes(rows, cols);
}

bitnet_status bitnet_w2a8_gemm_ws(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev, int64_t T,
                                  float *y_dev, void *workspace_dev, size_t workspace_bytes,
                                  bitnet_stream_t stream) {
    return gemm_impl(w, q_dev, s_dev, T, y_dev, nullptr, stream, workspace_dev, workspace_bytes);
}

bitnet_status bitnet_w2a8_gemm_acc(const bitnet_weight *w, const int8_t *q_dev, const float *s_dev,
                                   int64_t T, float *y_dev, int32_t *acc_dev, bitnet_stream_t stream) {
    if (!acc_dev) return fail(BITNET_ERR_NULL, "acc is NULL");
    return gemm_impl(w, q_dev, s_dev, T, y_dev, acc_dev, stream);
}

bitnet_status bitnet_get_device_error(bitnet_stream_t stream) {
    t_detail[0] = 0;
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream");
    DeviceGlobals g;
    e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    unsigned word = 0;
    e = cudaMemcpy(&word, g.err, sizeof(word), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(g.err, 0, sizeof(unsigned));
    if (e != cudaSuccess) return cuda_fail(e, "error word");
    if (word & kErrTimeout) return fail(BITNET_ERR_TIMEOUT, "a bounded device wait ran out (word 0x%x)", word);
    if (word & kErrCorrupt) return fail(BITNET_ERR_CORRUPT, "a kernel met code 3 (word 0x%x)", word);
    if (word) return fail(BITNET_ERR_VALUE, "device error word 0x%x", word);
    return BITNET_OK;
}

bitnet_status bitnet_set_wait_limit(uint32_t max_iterations) {
    t_detail[0] = 0;
    DeviceGlobals g;
    cudaError_t e = device_globals(&g);
    if (e != cudaSuccess) return cuda_fail(e, "device globals");
    const unsigned v = max_iterations ? max_iterations : kDefaultWaitLimit;
    e = cudaMemcpy(g.wait_limit, &v, sizeof(v), cudaMemcpyHostToDevice);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "wait limit");
}

}  // extern "C"
