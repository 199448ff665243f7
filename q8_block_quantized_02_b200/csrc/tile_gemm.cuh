// tile_gemm.cuh -- S2/S3/S4/S8: Q8_0 weight products for N = 1..16 activation
// columns: fp32 activations (GEMV / small-batch GEMM), the fused
// SiLU(gate) * up epilogue, and Q8_0 activations (int32 block dots).
//
// Work split (one persistent CTA per SM):
//   * the output rows are taken in packed groups of 8 ("units"; for SwiGLU a
//     unit is a gate group together with its up group).  CTA c owns the
//     contiguous, balanced unit range [U*c/grid, U*(c+1)/grid) and walks it in
//     tiles of up to TG units (the last tile may be partial);
//   * a tile is streamed over K in stages of CS 16-byte columns.  Each stage
//     is one TMA box per unit for the q bytes ([CS][8 rows x 16 B], the
//     tensor cores' core-matrix order), one per unit for the scales
//     ([CS/2][8] fp16) and one for the activations ([N][CS][16 elements]);
//   * warp 8 produces: one thread issues the boxes into a ring of `stages`
//     buffers guarded by full/empty mbarriers.  Weight boxes of the first
//     stages are issued before griddepcontrol.wait, so they stream while the
//     previous kernel on the stream is still finishing; activation boxes are
//     issued after it;
//   * warps 0..7 consume.  Lane (r = lane & 7, j = lane >> 3) works on row r
//     of column 4*cq + j; the 8 lanes of a column read 128 contiguous bytes,
//     so shared-memory reads are conflict-free.  A tile of >= 8 units gives
//     each warp one or two whole units (no cross-warp traffic).  A smaller
//     tile splits its (unit, 4-column quad) pairs evenly over the 8 warps;
//     the warps' partial sums are then added in shared memory in warp order;
//   * fp32 modes dequantise each 16-byte piece once (byte permute + paired
//     subtract) and take the 16-term dot with packed f32x2 FMAs, then scale
//     by the block's d.  The Q8Q8 mode takes exact int32 dots on the dp4a
//     units and adds d_w * d_x * dot in fp32;
//   * every output is summed in a fixed order, so results are bit-identical
//     from run to run.
// Every wait is bounded (see q8_device.cuh); a stalled pipeline records an
// error, drains its in-flight copies and exits.
#pragma once

#include "q8_device.cuh"

namespace q8 {

constexpr int kConsumerWarps = 8;
constexpr int kTileThreads = (kConsumerWarps + 1) * 32;
constexpr int kModeF32 = 0, kModeSwiGLU = 1, kModeQ8Q8 = 2;

struct TileArgs {
    float *y;            // [N][M_out]
    const uint16_t *xd;  // Q8Q8: activation scales [N][B] (read through L1)
    int M_out;           // output rows
    int N;               // activation columns
    int C;               // 16-byte columns per row (K / 16)
    int B;               // blocks per row (K / 32)
    int units;           // output row groups (SwiGLU: gate groups)
    int TG;              // max units per tile
    int CS;              // columns per stage (multiple of 8)
    int ksteps;          // stages per tile = ceil(C / CS)
    int NQ;              // 4-column quads over K = ceil(C / 4)
    int up_group0;       // SwiGLU: group index of the first up row (I / 8)
    int stages;          // ring depth
    uint32_t q_box;      // bytes of one unit's q box (CS * 128)
    uint32_t d_box;      // bytes of one unit's scale box (CS * 8)
    uint32_t d_slot;     // shared-memory stride of scale boxes (128-aligned)
    uint32_t x_box;      // bytes of the activation box
    uint32_t q_half;     // TG * q_box
    uint32_t d_off;      // offset of the scale region
    uint32_t d_half;     // TG * d_slot
    uint32_t x_off;      // offset of the activation region
    uint32_t stage_bytes;
};

template <int MODE>
__host__ __device__ constexpr int tile_acc_sets() {
    return MODE == kModeSwiGLU ? 4 : 2;
}
__host__ __device__ constexpr int tile_red_floats(int nmax, int sets) {
    return kConsumerWarps * sets * nmax * 8;
}

__device__ __forceinline__ int dp4a_s8(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

struct ColPiece {
    uint64_t w[8];
    float d;
};

__device__ __forceinline__ void load_piece(const uint8_t *st, const TileArgs &a, uint32_t qoff,
                                           uint32_t doff, int g, int col, int r, ColPiece &p) {
    const uint4 q = *reinterpret_cast<const uint4 *>(st + qoff + g * a.q_box + col * kColBytes + r * 16);
    p.d = __half2float(*reinterpret_cast<const __half *>(st + a.d_off + doff + g * a.d_slot +
                                                         (col >> 1) * 16 + r * 2));
    dequant16_x2(q, p.w);
}

// fp32 activations: one column of row r for one or two weight pieces that
// share the activation values (two units of a tile, or gate and up).
template <int NMAX>
__device__ __forceinline__ void fp32_column(const uint8_t *st, const TileArgs &a, int col,
                                            const ColPiece &p0, const ColPiece *p1,
                                            float (&acc0)[NMAX], float (&acc1)[NMAX]) {
    const uint8_t *xcol = st + a.x_off + col * 64;
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        if (n < a.N) {
            const ulonglong2 *xv = reinterpret_cast<const ulonglong2 *>(xcol + n * a.CS * 64);
            const ulonglong2 x0 = xv[0], x1 = xv[1], x2 = xv[2], x3 = xv[3];
            acc0[n] = fmaf(dot16_x2(p0.w, x0, x1, x2, x3), p0.d, acc0[n]);
            if (p1) acc1[n] = fmaf(dot16_x2(p1->w, x0, x1, x2, x3), p1->d, acc1[n]);
        }
    }
}

// Q8 x Q8: one 16-byte column (half a block) of row r for unit g; lanes j and
// j^1 hold the two halves of one block, so their int32 partials are joined by
// a shuffle before the block's scales are applied (by the even lane).  Every
// lane of the warp calls this (the shuffle needs them all); columns past the
// end of K lie in the zero-filled part of the TMA box and add nothing.
template <int NMAX>
__device__ __forceinline__ void q8_column(const uint8_t *st, const TileArgs &a, int col, int blk,
                                          int r, int j, int g, float (&acc)[NMAX]) {
    const uint4 qb = *reinterpret_cast<const uint4 *>(st + g * a.q_box + col * kColBytes + r * 16);
    // stored bytes are q + 128; flipping the top bit gives signed int8 again
    const uint32_t w0 = qb.x ^ 0x80808080u, w1 = qb.y ^ 0x80808080u, w2 = qb.z ^ 0x80808080u,
                   w3 = qb.w ^ 0x80808080u;
    const float dw = __half2float(*reinterpret_cast<const __half *>(
        st + a.d_off + g * a.d_slot + (col >> 1) * 16 + r * 2));
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
                acc[n] = fmaf((float)dot, dw * dx, acc[n]);
            }
        }
    }
}

// One column of unit g into accumulator set s (SwiGLU: gate -> 2s, up -> 2s+1).
template <int NMAX, int MODE>
__device__ __forceinline__ void unit_column(const uint8_t *st, const TileArgs &a, int ks, int col,
                                            int r, int j, int g, int s,
                                            float (&acc)[tile_acc_sets<MODE>()][NMAX]) {
    if (MODE == kModeQ8Q8) {
        const int blk = min((ks * a.CS + col) >> 1, a.B - 1);
        q8_column<NMAX>(st, a, col, blk, r, j, g, acc[s]);
    } else if (MODE == kModeSwiGLU) {
        ColPiece pg, pu;
        load_piece(st, a, 0, 0, g, col, r, pg);
        load_piece(st, a, a.q_half, a.d_half, g, col, r, pu);
        fp32_column<NMAX>(st, a, col, pg, &pu, acc[2 * s], acc[2 * s + 1]);
    } else {
        ColPiece p;
        load_piece(st, a, 0, 0, g, col, r, p);
        fp32_column<NMAX>(st, a, col, p, nullptr, acc[s], acc[s]);
    }
}

template <int NMAX, int MODE>
__device__ __forceinline__ void store_unit(const TileArgs &a, int unit, int r, const float *v0,
                                           const float *v1) {
    const int row = unit * kGroupRows + r;
    if (row >= a.M_out) return;
#pragma unroll
    for (int n = 0; n < NMAX; ++n)
        if (n < a.N)
            a.y[(size_t)n * a.M_out + row] = MODE == kModeSwiGLU ? silu_mul(v0[n], v1[n]) : v0[n];
}

template <int NMAX, int MODE>
__global__ void __launch_bounds__(kTileThreads, 1)
    tile_gemm_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap td,
                     const __grid_constant__ CUtensorMap tx, const TileArgs a) {
    constexpr int SETS = tile_acc_sets<MODE>();
    constexpr int HALVES = MODE == kModeSwiGLU ? 2 : 1;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)a.stages * a.stage_bytes);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);
    float *red = reinterpret_cast<float *>(bars + 2 * a.stages);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(red + tile_red_floats(NMAX, SETS));
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
    // The next kernel on the stream may start its prologue now; it reads
    // nothing this kernel writes before its own griddepcontrol.wait.
    pdl_launch_dependents();

    const int u0 = (int)(((int64_t)a.units * blockIdx.x) / gridDim.x);
    const int u1 = (int)(((int64_t)a.units * (blockIdx.x + 1)) / gridDim.x);
    const int n_tiles = (u1 - u0 + a.TG - 1) / a.TG;
    const int total = n_tiles * a.ksteps;

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tq);
            prefetch_tensormap(&td);
            prefetch_tensormap(&tx);
            const uint64_t pw = policy_evict_first(), px = policy_evict_last();
            auto issue_weights = [&](int it) {
                const int slot = it % a.stages;
                const int ut = u0 + (it / a.ksteps) * a.TG;
                const int tga = min(a.TG, u1 - ut);
                const int c0 = (it % a.ksteps) * a.CS;
                const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
                const uint32_t full = full0 + 8 * slot;
                mbar_arrive_expect_tx(full, HALVES * tga * (a.q_box + a.d_box) + a.x_box);
                for (int g = 0; g < tga; ++g) {
                    tma_load_3d(st + g * a.q_box, &tq, full, 0, c0, ut + g, pw);
                    tma_load_3d(st + a.d_off + g * a.d_slot, &td, full, 0, c0 >> 1, ut + g, pw);
                    if (MODE == kModeSwiGLU) {
                        tma_load_3d(st + a.q_half + g * a.q_box, &tq, full, 0, c0,
                                    ut + g + a.up_group0, pw);
                        tma_load_3d(st + a.d_off + a.d_half + g * a.d_slot, &td, full, 0, c0 >> 1,
                                    ut + g + a.up_group0, pw);
                    }
                }
            };
            auto issue_x = [&](int it) {
                const int slot = it % a.stages;
                const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
                tma_load_3d(st + a.x_off, &tx, full0 + 8 * slot, 0, (it % a.ksteps) * a.CS, 0, px);
            };
            const int pro = total < a.stages ? total : a.stages;
            int it = 0;
            for (; it < pro; ++it) issue_weights(it);  // weights never depend on the previous grid
            pdl_wait();                                // activations may
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
        pdl_wait();  // outputs may still be read by the previous grid
        int it = 0;
        for (int tl = 0; tl < n_tiles; ++tl) {
            const int ut = u0 + tl * a.TG;
            const int tga = min(a.TG, u1 - ut);
            const bool whole = tga >= 8;  // each warp owns whole units
            // split mode: this warp's contiguous range of (unit, quad) pairs
            const int P = tga * a.NQ;
            const int p_lo = (P * cw) / kConsumerWarps, p_hi = (P * (cw + 1)) / kConsumerWarps;
            const int gs0 = p_lo / a.NQ;
            const int gs1 = p_hi > p_lo ? (p_hi - 1) / a.NQ : gs0;
            float acc[SETS][NMAX];
#pragma unroll
            for (int h = 0; h < SETS; ++h)
#pragma unroll
                for (int n = 0; n < NMAX; ++n) acc[h][n] = 0.f;
            for (int ks = 0; ks < a.ksteps; ++ks, ++it) {
                const int slot = it % a.stages;
                if (mbar_wait(full0 + 8 * slot, (it / a.stages) & 1, abort_flag)) {
                    const uint8_t *st = smem + (size_t)slot * a.stage_bytes;
                    const int cols = min(a.CS, a.C - ks * a.CS);
                    const int nq = (cols + 3) >> 2;
                    if (whole) {
                        const int gB = cw + 8 < tga ? cw + 8 : -1;
                        for (int cq = 0; cq < nq; ++cq) {
                            const int col = 4 * cq + j;
                            if (MODE == kModeF32 && gB >= 0) {
                                if (col < cols) {
                                    ColPiece p0, p1;
                                    load_piece(st, a, 0, 0, cw, col, r, p0);
                                    load_piece(st, a, 0, 0, gB, col, r, p1);
                                    fp32_column<NMAX>(st, a, col, p0, &p1, acc[0], acc[1]);
                                }
                            } else if (MODE == kModeQ8Q8 || col < cols) {
                                unit_column<NMAX, MODE>(st, a, ks, col, r, j, cw, 0, acc);
                                if (gB >= 0) unit_column<NMAX, MODE>(st, a, ks, col, r, j, gB, 1, acc);
                            }
                        }
                    } else {
                        const int qs0 = ks * (a.CS >> 2);
                        for (int s = 0; s < 2; ++s) {
                            const int g = s == 0 ? gs0 : gs1;
                            if (s == 1 && gs1 == gs0) break;
                            const int lo = max(max(p_lo - g * a.NQ, 0), qs0);
                            const int hi = min(min(p_hi - g * a.NQ, a.NQ), qs0 + nq);
                            for (int qk = lo; qk < hi; ++qk) {
                                const int col = 4 * (qk - qs0) + j;
                                if (MODE == kModeQ8Q8 || col < cols)
                                    unit_column<NMAX, MODE>(st, a, ks, col, r, j, g, s, acc);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty0 + 8 * slot);
            }
            // lanes r, r+8, r+16, r+24 hold partial sums of the same row
#pragma unroll
            for (int h = 0; h < SETS; ++h)
#pragma unroll
                for (int n = 0; n < NMAX; ++n) {
                    acc[h][n] += __shfl_xor_sync(0xffffffffu, acc[h][n], 8);
                    acc[h][n] += __shfl_xor_sync(0xffffffffu, acc[h][n], 16);
                }
            if (whole) {
                if (j == 0) {
                    if (MODE == kModeSwiGLU) {
                        store_unit<NMAX, MODE>(a, ut + cw, r, acc[0], acc[1]);
                    } else {
                        store_unit<NMAX, MODE>(a, ut + cw, r, acc[0], acc[0]);
                        if (cw + 8 < tga) store_unit<NMAX, MODE>(a, ut + cw + 8, r, acc[1], acc[1]);
                    }
                }
            } else {
                if (j == 0) {
#pragma unroll
                    for (int h = 0; h < SETS; ++h)
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) red[((cw * SETS + h) * NMAX + n) * 8 + r] = acc[h][n];
                }
                named_barrier(1, kConsumerWarps * 32);
                if (cw < tga && j == 0) {
                    // unit cw: add the partials of every warp whose range touches it, in warp order
                    constexpr int PER = SETS / 2;  // accumulator sets per unit slot
                    float v[PER][NMAX];
#pragma unroll
                    for (int h = 0; h < PER; ++h)
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) v[h][n] = 0.f;
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        const int wl = (P * w) / kConsumerWarps, wh = (P * (w + 1)) / kConsumerWarps;
                        if (wh <= wl || wl >= (cw + 1) * a.NQ || wh <= cw * a.NQ) continue;
                        const int slot = (wl / a.NQ == cw) ? 0 : 1;
#pragma unroll
                        for (int h = 0; h < PER; ++h)
#pragma unroll
                            for (int n = 0; n < NMAX; ++n)
                                v[h][n] += red[((w * SETS + slot * PER + h) * NMAX + n) * 8 + r];
                    }
                    store_unit<NMAX, MODE>(a, ut + cw, r, v[0], v[PER - 1]);
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
