// repack.cu -- i2_s codes and block scales -> the kernels' device layout.
//
// i2_s ("浏览器里跑 1-bit 大模型 BitNet WebAssembly 的 50 倍提速实操",
// section "i2_s 到底是什么"): row-major, cols/4 bytes per row, byte b of a
// 128-weight block holding weights b, b+32, b+64, b+96 at shifts 6, 4, 2, 0.
//
// Device layout (version 1): the matrix is cut into 16-row x 128-column tiles
// of 512 bytes, row tiles outermost.  Inside a tile, lane L = 4*g + t of a warp
// owns 16 contiguous bytes = four 32-bit words of i2_s bytes:
//   word 0: row g,     block bytes 4t .. 4t+3
//   word 1: row g + 8, block bytes 4t .. 4t+3
//   word 2: row g,     block bytes 16+4t .. 16+4t+3
//   word 3: row g + 8, block bytes 16+4t .. 16+4t+3
// so one 16-byte load per lane brings a warp a whole tile, every lane's
// words pair with the same activation bytes for both of its rows, and the
// words sit where an m16n8k32 A fragment wants them.  Masking a word with
// 0x03030303 << (6 - 2*group) yields four codes of four consecutive columns.
// Block scales are stored per tile ([tile][16] fp32), and each row also gets
// its single scale when all of its block scales are bitwise equal (the
// per-tensor absmean case), which lets the kernels accumulate a whole row in
// int32 and scale once.
// Rows past `rows` in the last tile are padded with code 1 (weight 0).
#include "common.cuh"

namespace bitnet {
namespace {

__device__ __forceinline__ bool has_code3(uint32_t w) {
    return (w & (w >> 1) & 0x55555555u) != 0u;
}

__global__ void repack_tiles_kernel(const uint32_t *__restrict__ codes, int64_t rows,
                                    int64_t nb, int64_t ntr, uint4 *__restrict__ tiles,
                                    unsigned *__restrict__ hdr) {
    const int64_t words_per_row = nb * 8;  // cols/4 bytes = nb*32 bytes
    const int64_t total = ntr * nb * 32;
    bool bad = false;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int lane = (int)(idx & 31);
        const int64_t tb = idx >> 5;  // tile-block index = rt*nb + j
        const int64_t rt = tb / nb, j = tb - rt * nb;
        const int g = lane >> 2, t = lane & 3;
        const int64_t ra = rt * 16 + g, rb = ra + 8;
        const int64_t w0 = j * 8 + t, w2 = j * 8 + 4 + t;
        uint4 v;
        v.x = ra < rows ? __ldg(codes + ra * words_per_row + w0) : 0x55555555u;
        v.y = rb < rows ? __ldg(codes + rb * words_per_row + w0) : 0x55555555u;
        v.z = ra < rows ? __ldg(codes + ra * words_per_row + w2) : 0x55555555u;
        v.w = rb < rows ? __ldg(codes + rb * words_per_row + w2) : 0x55555555u;
        bad |= has_code3(v.x) | has_code3(v.y) | has_code3(v.z) | has_code3(v.w);
        tiles[idx] = v;
    }
    if (bad) atomicOr(hdr + 1, 1u);
}

__global__ void repack_scales_kernel(const float *__restrict__ scales, int64_t rows, int64_t nb,
                                     int64_t ntr, float *__restrict__ tscales,
                                     float *__restrict__ rowscale, unsigned *__restrict__ hdr) {
    const int64_t total = ntr * nb * 16;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int r = (int)(idx & 15);
        const int64_t tb = idx >> 4;
        const int64_t rt = tb / nb, j = tb - rt * nb;
        const int64_t row = rt * 16 + r;
        tscales[idx] = row < rows ? __ldg(scales + row * nb + j) : 0.0f;
    }
    for (int64_t row = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; row < ntr * 16;
         row += (int64_t)gridDim.x * blockDim.x) {
        if (row >= rows) {
            rowscale[row] = 0.0f;
            continue;
        }
        const float *sr = scales + row * nb;
        const uint32_t s0 = __float_as_uint(__ldg(sr));
        bool uniform = true;
        for (int64_t j = 1; j < nb; j++) uniform &= (__float_as_uint(__ldg(sr + j)) == s0);
        rowscale[row] = uniform ? __uint_as_float(s0) : __uint_as_float(0x7fc00000u);
        if (!uniform) atomicAdd(hdr, 1u);
    }
}

__global__ void unrepack_kernel(const uint4 *__restrict__ tiles, const float *__restrict__ tscales,
                                int64_t rows, int64_t nb, int64_t ntr, uint32_t *__restrict__ codes,
                                float *__restrict__ scales) {
    const int64_t words_per_row = nb * 8;
    const int64_t total = ntr * nb * 32;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int lane = (int)(idx & 31);
        const int64_t tb = idx >> 5;
        const int64_t rt = tb / nb, j = tb - rt * nb;
        const int g = lane >> 2, t = lane & 3;
        const int64_t ra = rt * 16 + g, rb = ra + 8;
        const int64_t w0 = j * 8 + t, w2 = j * 8 + 4 + t;
        const uint4 v = tiles[idx];
        if (ra < rows) {
            codes[ra * words_per_row + w0] = v.x;
            codes[ra * words_per_row + w2] = v.z;
        }
        if (rb < rows) {
            codes[rb * words_per_row + w0] = v.y;
            codes[rb * words_per_row + w2] = v.w;
        }
        if (lane < 16) {
            const int64_t row = rt * 16 + lane;
            if (row < rows) scales[row * nb + j] = tscales[tb * 16 + lane];
        }
    }
}

unsigned grid_for(int64_t work, int threads) {
    int64_t g = (work + threads - 1) / threads;
    if (g < 1) g = 1;
    if (g > 148 * 16) g = 148 * 16;
    return (unsigned)g;
}

}  // namespace

cudaError_t launch_repack(const uint8_t *codes, const float *scales, int64_t rows, int64_t cols,
                          void *data, cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    char *base = static_cast<char *>(data);
    unsigned *hdr = reinterpret_cast<unsigned *>(base);
    cudaError_t e = cudaMemsetAsync(hdr, 0, 256, st);
    if (e != cudaSuccess) return e;
    const int threads = 256;
    repack_tiles_kernel<<<grid_for(L.ntr * L.nb * 32, threads), threads, 0, st>>>(
        reinterpret_cast<const uint32_t *>(codes), rows, L.nb, L.ntr,
        reinterpret_cast<uint4 *>(base + L.off_tiles), hdr);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    repack_scales_kernel<<<grid_for(L.ntr * L.nb * 16, threads), threads, 0, st>>>(
        scales, rows, L.nb, L.ntr, reinterpret_cast<float *>(base + L.off_tscales),
        reinterpret_cast<float *>(base + L.off_rowscale), hdr);
    return cudaGetLastError();
}

cudaError_t launch_unrepack(const void *data, int64_t rows, int64_t cols, uint8_t *codes,
                            float *scales, cudaStream_t st) {
    const Layout L = layout_of(rows, cols);
    const char *base = static_cast<const char *>(data);
    const int threads = 256;
    unrepack_kernel<<<grid_for(L.ntr * L.nb * 32, threads), threads, 0, st>>>(
        reinterpret_cast<const uint4 *>(base + L.off_tiles),
        reinterpret_cast<const float *>(base + L.off_tscales), rows, L.nb, L.ntr,
        reinterpret_cast<uint32_t *>(codes), scales);
    return cudaGetLastError();
}

}  // namespace bitnet
