// expand.cuh -- expansion of repacked i2_s code tiles to int8 weights, shared
// by the expansion kernel of the prefill GEMM and the prefill linear's
// pre-pass.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnet {

// Four codes (group grp of a code word) -> four signed bytes t = c - 1:
// byte b of a block holds weights b, b+32, b+64, b+96 at shifts 6, 4, 2, 0;
// (c + 0x7F) ^ 0x80 subtracts 1 per byte without carries (c <= 2).
static __device__ __forceinline__ uint32_t expand_group(uint32_t w, int grp) {
    const uint32_t c = (w >> (6 - 2 * grp)) & 0x03030303u;
    return (c + 0x7F7F7F7Fu) ^ 0x80808080u;
}

// One warp writes tile tj (16 rows x 128 weights, 512 bytes, held as lane
// words v) as int8 rows of `out` ([ntr * 16][cols] row-major).  Lane 4g+t
// holds bytes 4t.. of row g (x) and of row g+8 (y) and bytes 16+4t.. of the
// same rows (z, w).  The warp stages the tile in `stage` (32 x 16 bytes of
// shared memory) and each lane then writes whole 16-byte pieces of output
// rows, eight lanes to a 128-byte row: piece c of row r is group c / 2,
// words (c & 1) * 4 .. + 3 of the row, i.e. the x (or z; y, w for rows
// 8..15) words of lanes 4g .. 4g+3 decoded at that group's shift.
static __device__ __forceinline__ void expand_tile(uint4 v, uint4 *stage, int8_t *out, int64_t tj, int nb,
                                                   int64_t cols) {
    const int lane = threadIdx.x & 31;
    stage[lane] = v;
    __syncwarp();
    const uint32_t *sw = reinterpret_cast<const uint32_t *>(stage);
    const int j = (int)(tj % nb);
    const int64_t tr = tj / nb;
    const int c = lane & 7, grp = c >> 1;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int r = 4 * i + (lane >> 3);     // output row of the tile
        const int g = r & 7;
        const int f = (r >> 3) + 2 * (c & 1);  // word of a lane's 16 bytes: x 0, y 1, z 2, w 3
        uint4 o;
        o.x = expand_group(sw[(4 * g + 0) * 4 + f], grp);
        o.y = expand_group(sw[(4 * g + 1) * 4 + f], grp);
        o.z = expand_group(sw[(4 * g + 2) * 4 + f], grp);
        o.w = expand_group(sw[(4 * g + 3) * 4 + f], grp);
        *reinterpret_cast<uint4 *>(out + (tr * 16 + r) * cols + 128 * j + 16 * c) = o;
    }
    __syncwarp();  // the stage may be reused by this warp's next tile
}

}  // namespace bitnet
