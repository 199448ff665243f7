// pack.cuh -- S1: re-lay GGUF Q8_0 blocks into the packed device layout and
// back.  One thread per (row, block); threads of consecutive rows of a group
// write consecutive 16-byte pieces, so the writes are fully coalesced.  Pure
// byte moves: bit-exact and invertible (the q bytes are XORed with 0x80).
#pragma once

#include "q8_device.cuh"

namespace q8 {

// gguf: [M][B][34] bytes.  packed: ceil(M/8) groups of 272*B bytes.
__global__ void pack_kernel(const uint8_t *__restrict__ gguf, uint8_t *__restrict__ packed,
                            int64_t M, int64_t B) {
    const int64_t groups = (M + kGroupRows - 1) / kGroupRows;
    const int64_t total = groups * B * kGroupRows;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int r = (int)(i % kGroupRows);
        const int64_t b = (i / kGroupRows) % B;
        const int64_t g = i / (kGroupRows * B);
        const int64_t row = g * kGroupRows + r;
        uint8_t *grp = packed + g * kGroupBytesPerBlock * B;
        uint32_t w[8];  // 32 biased q bytes
        uint16_t d = 0;
        if (row < M) {
            const uint8_t *blk = gguf + (row * B + b) * 34;
            d = (uint16_t)(blk[0] | (blk[1] << 8));
#pragma unroll
            for (int k = 0; k < 8; ++k)
                w[k] = ((uint32_t)blk[2 + 4 * k] | ((uint32_t)blk[3 + 4 * k] << 8) |
                        ((uint32_t)blk[4 + 4 * k] << 16) | ((uint32_t)blk[5 + 4 * k] << 24)) ^
                       0x80808080u;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = 0x80808080u;  // q = 0
        }
        uint4 *lo = reinterpret_cast<uint4 *>(grp + (2 * b) * kColBytes + r * 16);
        uint4 *hi = reinterpret_cast<uint4 *>(grp + (2 * b + 1) * kColBytes + r * 16);
        *lo = make_uint4(w[0], w[1], w[2], w[3]);
        *hi = make_uint4(w[4], w[5], w[6], w[7]);
        reinterpret_cast<uint16_t *>(grp + 256 * B + b * 16)[r] = d;
    }
}

__global__ void unpack_kernel(const uint8_t *__restrict__ packed, uint8_t *__restrict__ gguf,
                              int64_t M, int64_t B) {
    const int64_t total = M * B;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / B;
        const int64_t b = i % B;
        const int64_t g = row / kGroupRows;
        const int r = (int)(row % kGroupRows);
        const uint8_t *grp = packed + g * kGroupBytesPerBlock * B;
        const uint16_t d = reinterpret_cast<const uint16_t *>(grp + 256 * B + b * 16)[r];
        const uint4 lo = *reinterpret_cast<const uint4 *>(grp + (2 * b) * kColBytes + r * 16);
        const uint4 hi = *reinterpret_cast<const uint4 *>(grp + (2 * b + 1) * kColBytes + r * 16);
        const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        uint8_t *blk = gguf + i * 34;
        blk[0] = (uint8_t)(d & 0xff);
        blk[1] = (uint8_t)(d >> 8);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t v = w[k] ^ 0x80808080u;
            blk[2 + 4 * k] = (uint8_t)(v & 0xff);
            blk[3 + 4 * k] = (uint8_t)((v >> 8) & 0xff);
            blk[4 + 4 * k] = (uint8_t)((v >> 16) & 0xff);
            blk[5 + 4 * k] = (uint8_t)(v >> 24);
        }
    }
}

}  // namespace q8
