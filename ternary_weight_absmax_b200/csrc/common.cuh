// common.cuh -- internal declarations shared by the library's translation units.
// Not part of the ABI (the ABI is include/bitnet_w2a8.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/bitnet_w2a8.h"

namespace bitnet {

constexpr int kQK = 128;          // weights per i2_s block
constexpr int kTileRows = 16;     // rows per device tile
constexpr int kTileBytes = 512;   // 16 rows x 128 weights x 2 bits
constexpr float kEps = 1e-5f;     // floor on absmax

// Bits of the per-device error word.
constexpr unsigned kErrTimeout = 1u;
constexpr unsigned kErrCorrupt = 2u;
constexpr unsigned kErrBounds = 4u;

// Default iteration cap for bounded device waits.
constexpr unsigned kDefaultWaitLimit = 1u << 26;

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Byte layout of a repacked weight buffer (layout version 1).
//   [0, 256)           header: u32 not_uniform_rows, u32 corrupt
//   off_tiles          [ntr][nb][32 lanes][16 B] code tiles
//   off_tscales        [ntr][nb][16] fp32 block scales, tile order
//   off_rowscale       [ntr*16] fp32: the row's scale if all its block scales
//                      are equal, else NaN
struct Layout {
    int64_t rows, cols, ntr, nb;
    size_t off_tiles, off_tscales, off_rowscale, total;
};

static inline Layout layout_of(int64_t rows, int64_t cols) {
    Layout L;
    L.rows = rows;
    L.cols = cols;
    L.ntr = (rows + kTileRows - 1) / kTileRows;
    L.nb = cols / kQK;
    size_t tiles = (size_t)L.ntr * (size_t)L.nb * kTileBytes;
    size_t tsc = (size_t)L.ntr * (size_t)L.nb * kTileRows * sizeof(float);
    size_t rsc = (size_t)L.ntr * kTileRows * sizeof(float);
    L.off_tiles = 256;
    L.off_tscales = L.off_tiles + align_up(tiles, 256);
    L.off_rowscale = L.off_tscales + align_up(tsc, 256);
    L.total = L.off_rowscale + align_up(rsc, 256);
    return L;
}

// Records a human-readable reason for `st` (returned by
// bitnet_last_error_detail on this host thread) and returns `st`.
bitnet_status set_error_detail(bitnet_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));

// Per-device addresses of the library's device globals.
struct DeviceGlobals {
    unsigned *err;         // error word (kErr* bits)
    unsigned *wait_limit;  // iteration cap for bounded waits
};
cudaError_t device_globals(DeviceGlobals *out);

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

// Launchers (return the launch error, if any).
// The prefill linear's pre-pass: quantise x (T rows) and expand the weights
// into `expanded` in one kernel (quant_act.cu); K up to 32768.
bool prefill_prep_supported(int64_t K);
cudaError_t launch_prefill_prep(const float *x, int64_t T, int64_t K, int8_t *q, float *s, const void *data,
                                int64_t rows, int8_t *expanded, cudaStream_t st);
cudaError_t launch_quant_act(const float *x, int64_t T, int64_t K, int8_t *q, float *s,
                             int32_t *blocksum, cudaStream_t st);
cudaError_t launch_repack(const uint8_t *codes, const float *scales, int64_t rows, int64_t cols,
                          void *data, cudaStream_t st);
cudaError_t launch_unrepack(const void *data, int64_t rows, int64_t cols, uint8_t *codes,
                            float *scales, cudaStream_t st);
// x non-null: the fused path (quantise x in the kernel; q, s ignored; q_out and
// s_out, if non-null, receive the quantised activations).
cudaError_t launch_gemv(const void *data, int64_t rows, int64_t cols, bool uniform,
                        const int8_t *q, const float *s, int64_t B, float *y, int32_t *acc,
                        const float *x, int8_t *q_out, float *s_out, const DeviceGlobals &g,
                        cudaStream_t st);
// Decode kernels for uniform rows (decode.cu): batch 1 (fused or not) and
// batches of 2..16 (q and s given); launch_gemv picks them when
// decode_supported says they take the call.
bool decode_supported(int64_t rows, int64_t cols, int64_t B, bool fused);
cudaError_t launch_decode(const void *data, int64_t rows, int64_t cols, int64_t B, const int8_t *q, const float *s,
                          float *y, const float *x, int8_t *q_out, float *s_out, const DeviceGlobals &g,
                          cudaStream_t st);
// Table-lookup batch-1 variant (decode.cu), uniform rows, K <= 8192;
// cudaErrorNotSupported for other shapes.
cudaError_t launch_decode_lut(const void *data, int64_t rows, int64_t cols, const int8_t *q, const float *s, float *y,
                              const DeviceGlobals &g, cudaStream_t st);
int absmean_num_partials(int64_t n);
cudaError_t launch_ternarize(const float *w, int64_t rows, int64_t cols, bool per_block, uint32_t *codes,
                             float *scales, double *partials, float *gamma_slot, cudaStream_t st);
// Small-batch GEMV on the warp-level int8 MMA (gemv_mma.cu): uniform rows, q
// (16-byte aligned) and s given, 1 <= B <= 64.
constexpr int kMmaMinBatch = 5;  // from this batch on the dispatcher prefers it to the dp4a kernels (measured)
bool gemv_mma_supported(int64_t rows, int64_t cols, int64_t B);
cudaError_t launch_gemv_mma(const void *data, int64_t rows, int64_t cols, const int8_t *q, const float *s,
                            int64_t B, float *y, cudaStream_t st);
// One linear of a sequence call (decode_seq.cu): repacked weight data with
// uniform rows, fp32 x [cols], fp32 y [rows], and the index of the linear whose
// y this x reads (-1: x is ready at launch).
constexpr int kSeqMaxLinears = 256;
constexpr int kSeqMaxK = 16384;
struct SeqLinear {
    const void *data;
    int64_t rows, cols;
    const float *x;
    float *y;
    int dep;
};
size_t seq_workspace_bytes(int n);
cudaError_t launch_decode_seq(const SeqLinear *list, int n, void *workspace, const DeviceGlobals &g,
                              cudaStream_t st);
// Prefill GEMM.  `expanded` (or null): a workspace of gemm_expanded_bytes()
// for the weights expanded to int8, used on uniform rows from
// kGemmExpandMinT tokens (the weights are expanded once per call and both
// MMA operands stream in by TMA, instead of every 128-token tile decoding
// them again).
constexpr int64_t kGemmExpandMinT = 256;
// The GEMM over expanded int8 weights on pairs of SMs (gemm_pair.cu).
cudaError_t launch_gemm_pair(const void *data, int64_t rows, int64_t cols, const int8_t *q, const float *s,
                             int64_t T, float *y, const int8_t *expanded, const DeviceGlobals &g,
                             cudaStream_t st);
size_t gemm_expanded_bytes(int64_t rows, int64_t cols);
cudaError_t launch_gemm(const void *data, int64_t rows, int64_t cols, bool uniform,
                        const int8_t *q, const float *s, int64_t T, float *y, int32_t *acc,
                        const DeviceGlobals &g, cudaStream_t st, int8_t *expanded = nullptr);

}  // namespace bitnet
