// tile_gemm.cuh -- S2/S3/S4: Q8_0 x fp32 products for N = 1..16 activation
// columns, optionally with the fused SiLU(gate) * up epilogue.
//
// Structure (one CTA per SM, persistent over tiles):
//   * a tile is TG packed groups (8*TG output rows) over the whole of K;
//   * K is walked in stages of CS 16-byte columns; one stage = a TMA box of
//     the q bytes [TG][CS][8 rows x 16 B], a box of the scales [TG][CS/2][8],
//     and a box of the activations [N][CS][16 fp32] (for SwiGLU also the
//     matching up-projection groups);
//   * warp 8 is the producer: one elected thread issues the TMA loads into a
//     ring of `stages` buffers (full/empty mbarriers).  The weight loads of
//     the first stages are issued before griddepcontrol.wait, so they overlap
//     the previous kernel on the stream; activation loads come after it;
//   * warps 0..7 consume: lane (r = lane & 7, j = lane >> 3) takes row r of
//     column 4*cq + j, dequantises its 16 bytes once (byte permute + add) and
//     reuses them for all N activation columns; the per-column partial is
//     scaled by the block's d.  The 8 lanes of one column read 128 contiguous
//     bytes, so shared-memory reads are conflict-free;
//   * at the end of a tile the four lanes holding the same row are summed by
//     shuffles (and, when TG < 8, the warps sharing a group through shared
//     memory, in a fixed order), so every result is reproducible bit for bit.
// MODE selects the activation type and epilogue: kModeF32 (fp32 x),
// kModeSwiGLU (fp32 x, gate and up tiles, h = silu(g) * u) and kModeQ8Q8
// (Q8_0 activations: int8 xq with binary16 scales; exact int32 block dots on
// the dp4a units, then y += d_w * d_x * dot in fp32).
// Every wait is bounded (see q8_device.cuh); a stalled pipeline records an
// error, drains its in-flight copies and exits.
#pragma once

#include "q8_device.cuh"

namespace q8 {

constexpr int kConsumerWarps = 8;
constexpr int kModeF32 = 0, kModeSwiGLU = 1, kModeQ8Q8 = 2;
constexpr int kTileThreads = (kConsumerWarps + 1) * 32;

struct TileArgs {
    float *y;            // [N][M_out]
    int M_out;           // output rows
    int N;               // activation columns
    int C;               // 16-byte columns per row (K / 16)
    int TG;              // groups per tile (1, 2, 4, 8, 16)
    int CS;              // columns per stage (multiple of 8)
    int ksteps;          // stages per tile = ceil(C / CS)
    int n_tiles;         // tiles in the matrix
    int up_group0;       // SwiGLU: group index of the first up row (I / 8)
    int stages;          // ring depth
    uint32_t q_half;     // bytes of one q box (TG * CS * 128)
    uint32_t d_off;      // offset of the scale region in a stage
    uint32_t d_half;     // bytes reserved per scale box
    uint32_t x_off;      // offset of the activation region in a stage
    const uint16_t *xd;  // Q8Q8: activation scales [N][B] (read through L1)
    int B;               // blocks per row (K / 32)
    uint32_t stage_bytes;
    uint32_t tx_bytes;   // TMA transaction bytes per stage
};

__host__ __device__ constexpr int tile_red_floats(int nmax) { return kConsumerWarps * 2 * nmax * 8; }

// One 16-byte column of one row for up to two groups; accumulates into acc.
template <int NMAX, bool SWIGLU>
__device__ __forceinline__ void tile_process_column(const uint8_t *st, const TileArgs &a,
                                                    int col, int r, int gA, int gB,
                                                    float (&acc)[2][NMAX]) {
    // first operand: group gA of the (gate or plain) half
    float w0[16], w1[16];
    const uint4 q0 = *reinterpret_cast<const uint4 *>(st + (gA * a.CS + col) * kColBytes + r * 16);
    const float d0 = __half2float(*reinterpret_cast<const __half *>(
        st + a.d_off + (gA * (a.CS >> 1) + (col >> 1)) * 16 + r * 2));
    dequant16(q0, w0);
    // second operand: the up half of gA (SwiGLU) or group gB
    const bool two = SWIGLU || gB >= 0;
    float d1 = 0.f;
    if (two) {
        const int g1 = SWIGLU ? gA : gB;
        const uint32_t qoff = SWIGLU ? a.q_half : 0u;
        const uint32_t doff = a.d_off + (SWIGLU ? a.d_half : 0u);
        const uint4 q1 =
            *reinterpret_cast<const uint4 *>(st + qoff + (g1 * a.CS + col) * kColBytes + r * 16);
        d1 = __half2float(*reinterpret_cast<const __half *>(
            st + doff + (g1 * (a.CS >> 1) + (col >> 1)) * 16 + r * 2));
        dequant16(q1, w1);
    }
    const float *xcol = reinterpret_cast<const float *>(st + a.x_off) + col * 16;
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        if (n < a.N) {
            const float4 *xv = reinterpret_cast<const float4 *>(xcol + n * a.CS * 16);
            const float4 x0 = xv[0], x1 = xv[1], x2 = xv[2], x3 = xv[3];
            const float xs[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                  x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
            float p0 = w0[0] * xs[0], p0b = w0[1] * xs[1];
#pragma unroll
            for (int i = 2; i < 16; i += 2) {
                p0 = fmaf(w0[i], xs[i], p0);
                p0b = fmaf(w0[i + 1], xs[i + 1], p0b);
            }
            acc[0][n] = fmaf(p0 + p0b, d0, acc[0][n]);
            if (two) {
                float p1 = w1[0] * xs[0], p1b = w1[1] * xs[1];
#pragma unroll
                for (int i = 2; i < 16; i += 2) {
                    p1 = fmaf(w1[i], xs[i], p1);
                    p1b = fmaf(w1[i + 1], xs[i + 1], p1b);
                }
                acc[1][n] = fmaf(p1 + p1b, d1, acc[1][n]);
            }
        }
    }
}

__device__ __forceinline__ int dp4a_s8(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Q8 x Q8: one 16-byte column (half a block) of row r; lanes j and j^1 hold
// the two halves of one block, so their int32 partials are joined by a
// shuffle before the block's scales are applied (by the even lane only).
// Called by every lane of the warp (the shuffle needs them all); columns past
// the end of K lie inside the zero-filled TMA box and contribute nothing.
template <int NMAX>
__device__ __forceinline__ void tile_process_column_q8(const uint8_t *st, const TileArgs &a,
                                                       int col, int blk, int r, int j, int g,
                                                       float (&acc)[2][NMAX]) {
    const uint4 qb = *reinterpret_cast<const uint4 *>(st + (g * a.CS + col) * kColBytes + r * 16);
    // stored bytes are q + 128; flip the top bit back to signed int8
    const uint32_t w0 = qb.x ^ 0x80808080u, w1 = qb.y ^ 0x80808080u, w2 = qb.z ^ 0x80808080u,
                   w3 = qb.w ^ 0x80808080u;
    const float dw = __half2float(*reinterpret_cast<const __half *>(
        st + a.d_off + (g * (a.CS >> 1) + (col >> 1)) * 16 + r * 2));
    const uint8_t *xq = st + a.x_off + col * 16;
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        if (n < a.N) {
            const uint4 xv = *reinterpret_cast<const uint4 *>(xq + n * a.CS * 16);
            int dot = dp4a_s8(w0, xv.x, 0);
            dot = dp4a_s8(w1, xv.y, dot);
            dot = dp4a_s8(w2, xv.z, dot);
            dot = dp4a_s8(w3, xv.w, dot);
            dot += __shfl_xor_sync(0xffffffffu, dot, 8);
            if ((j & 1) == 0) {
                const float dx = __half2float(__ushort_as_half(__ldg(a.xd + (size_t)n * a.B + blk)));
                acc[0][n] = fmaf((float)dot, dw * dx, acc[0][n]);
            }
        }
    }
}

template <int NMAX, bool SWIGLU>
__device__ __forceinline__ void tile_store(const TileArgs &a, int tile, int g, int r,
                                           const float (&v0)[NMAX], const float (&v1)[NMAX]) {
    const int row = (tile * a.TG + g) * kGroupRows + r;
    if (row >= a.M_out) return;
#pragma unroll
    for (int n = 0; n < NMAX; ++n)
        if (n < a.N) a.y[(size_t)n * a.M_out + row] = SWIGLU ? silu_mul(v0[n], v1[n]) : v0[n];
}

template <int NMAX, int MODE>
__global__ void __launch_bounds__(kTileThreads, 1)
    tile_gemm_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap td,
                     const __grid_constant__ CUtensorMap tx, const TileArgs a) {
    constexpr bool SWIGLU = MODE == kModeSwiGLU;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)a.stages * a.stage_bytes);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);
    float *red = reinterpret_cast<float *>(bars + 2 * a.stages);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(red + tile_red_floats(NMAX));
    volatile int *issued = abort_flag + 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kConsumerWarps);
        }
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // The next kernel on the stream may start its own prologue now; it reads
    // nothing of ours before its griddepcontrol.wait.
    pdl_launch_dependents();

    const int my_tiles =
        (int)blockIdx.x < a.n_tiles ? (a.n_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const int total = my_tiles * a.ksteps;

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tq);
            prefetch_tensormap(&td);
            prefetch_tensormap(&tx);
            const uint64_t pw = policy_evict_first(), px = policy_evict_last();
            auto issue_weights = [&](int it) {
                const int slot = it % a.stages;
                const int t = (int)blockIdx.x + (it / a.ksteps) * (int)gridDim.x;
                const int ks = it % a.ksteps;
                const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
                const uint32_t full = full0 + 8 * slot;
                const int g0 = t * a.TG, c0 = ks * a.CS;
                mbar_arrive_expect_tx(full, a.tx_bytes);
                tma_load_3d(st, &tq, full, 0, c0, g0, pw);
                tma_load_3d(st + a.d_off, &td, full, 0, c0 >> 1, g0, pw);
                if (SWIGLU) {
                    tma_load_3d(st + a.q_half, &tq, full, 0, c0, g0 + a.up_group0, pw);
                    tma_load_3d(st + a.d_off + a.d_half, &td, full, 0, c0 >> 1, g0 + a.up_group0, pw);
                }
            };
            auto issue_x = [&](int it) {
                const int slot = it % a.stages;
                const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
                const int c0 = (it % a.ksteps) * a.CS;
                tma_load_3d(st + a.x_off, &tx, full0 + 8 * slot, 0, c0, 0, px);
            };
            const int pro = total < a.stages ? total : a.stages;
            int it = 0;
            for (; it < pro; ++it) issue_weights(it);  // weights do not depend on the previous grid
            pdl_wait();                                // activations do
            for (int k = 0; k < pro; ++k) issue_x(k);
            for (; it < total; ++it) {
                const int slot = it % a.stages;
                if (!mbar_wait(empty0 + 8 * slot, ((it / a.stages) & 1) ^ 1, abort_flag)) break;
                issue_weights(it);
                issue_x(it);
            }
            *issued = it;
        }
    } else {
        // ------------------------------ consumers -----------------------------
        const int cw = warp, r = lane & 7, j = lane >> 3;
        int gA, gB, q0, qs;
        if (a.TG >= 8) {
            gA = cw;
            gB = (a.TG == 16) ? cw + 8 : -1;
            q0 = 0;
            qs = 1;
        } else {
            gA = cw % a.TG;
            gB = -1;
            q0 = cw / a.TG;
            qs = kConsumerWarps / a.TG;
        }
        pdl_wait();  // outputs may still be read by the previous grid
        int it = 0;
        for (int tl = 0; tl < my_tiles; ++tl) {
            const int t = (int)blockIdx.x + tl * (int)gridDim.x;
            float acc[2][NMAX];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int n = 0; n < NMAX; ++n) acc[h][n] = 0.f;
            for (int ks = 0; ks < a.ksteps; ++ks, ++it) {
                const int slot = it % a.stages;
                if (mbar_wait(full0 + 8 * slot, (it / a.stages) & 1, abort_flag)) {
                    const uint8_t *st = smem + (size_t)slot * a.stage_bytes;
                    const int cols = min(a.CS, a.C - ks * a.CS);
                    const int nq = (cols + 3) >> 2;
                    for (int cq = q0; cq < nq; cq += qs) {
                        const int col = 4 * cq + j;
                        if (MODE == kModeQ8Q8) {
                            const int blk = min((ks * a.CS + col) >> 1, a.B - 1);
                            tile_process_column_q8<NMAX>(st, a, col, blk, r, j, gA, acc);
                            if (gB >= 0) {
                                float tmp[2][NMAX];
#pragma unroll
                                for (int n = 0; n < NMAX; ++n) tmp[0][n] = acc[1][n];
                                tile_process_column_q8<NMAX>(st, a, col, blk, r, j, gB, tmp);
#pragma unroll
                                for (int n = 0; n < NMAX; ++n) acc[1][n] = tmp[0][n];
                            }
                        } else if (col < cols) {
                            tile_process_column<NMAX, SWIGLU>(st, a, col, r, gA, gB, acc);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty0 + 8 * slot);
            }
            // lanes r, r+8, r+16, r+24 hold the same row
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int n = 0; n < NMAX; ++n) {
                    acc[h][n] += __shfl_xor_sync(0xffffffffu, acc[h][n], 8);
                    acc[h][n] += __shfl_xor_sync(0xffffffffu, acc[h][n], 16);
                }
            if (a.TG >= 8) {
                if (j == 0) {
                    if (SWIGLU) {
                        tile_store<NMAX, true>(a, t, gA, r, acc[0], acc[1]);
                    } else {
                        tile_store<NMAX, false>(a, t, gA, r, acc[0], acc[0]);
                        if (gB >= 0) tile_store<NMAX, false>(a, t, gB, r, acc[1], acc[1]);
                    }
                }
            } else {
                if (j == 0) {
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) red[((cw * 2 + h) * NMAX + n) * 8 + r] = acc[h][n];
                }
                named_barrier(1, kConsumerWarps * 32);
                if (cw < a.TG && j == 0) {
                    float v0[NMAX], v1[NMAX];
#pragma unroll
                    for (int n = 0; n < NMAX; ++n) v0[n] = v1[n] = 0.f;
                    for (int w = cw; w < kConsumerWarps; w += a.TG) {
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) {
                            v0[n] += red[((w * 2 + 0) * NMAX + n) * 8 + r];
                            v1[n] += red[((w * 2 + 1) * NMAX + n) * 8 + r];
                        }
                    }
                    tile_store<NMAX, SWIGLU>(a, t, cw, r, v0, v1);
                }
                named_barrier(1, kConsumerWarps * 32);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        // A wait gave up: make sure no copy is still landing in this CTA's
        // shared memory before it exits.
        const int n_issued = *issued;
        for (int it = n_issued > a.stages ? n_issued - a.stages : 0; it < n_issued; ++it)
            mbar_drain(full0 + 8 * (it % a.stages), (it / a.stages) & 1);
    }
}

}  // namespace q8
