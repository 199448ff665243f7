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
    float *y;            // [N][M_out] (may be null when best is set)
    unsigned long long *best;  // arg-max keys [N] (q8_gemv_argmax; null otherwise)
    const float *res;    // fp32 GEMV: [N][M_out] added to the outputs (q8_gemv_residual; may be y)
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
    uint32_t d_slot;     // shared-memory stride of unit scale boxes (= d_box)
    uint32_t x_box;      // bytes of the activation box
    uint32_t q_half;     // TG * q_box
    uint32_t d_off;      // offset of the scale region
    uint32_t d_half;     // TG * d_slot
    uint32_t x_off;      // offset of the activation region
    uint32_t stage_bytes;
    int CB;              // resident kernel: columns per weight box
    int nchunks;         // resident kernel: weight boxes per row group (CS = nchunks * CB)
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
    if (row >= a.M_out || !a.y) return;
#pragma unroll
    for (int n = 0; n < NMAX; ++n)
        if (n < a.N) {
            const size_t o = (size_t)n * a.M_out + row;
            a.y[o] = MODE == kModeSwiGLU ? silu_mul(v0[n], v1[n])
                     : (MODE == kModeF32 && a.res) ? __fadd_rn(v0[n], a.res[o])  // read, then write: y may be res
                                                   : v0[n];
        }
}

// Arg-max key of output value v at row `row`: the float's bits mapped to an
// unsigned order (negative values below positive ones, -0 taken as +0) in
// the high word, 0xFFFFFFFF - row in the low word, so the largest key is the
// largest value and, among equal values, the lowest row.
__device__ __forceinline__ unsigned long long argmax_key(float v, int row) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)ord << 32) | (0xFFFFFFFFu - (uint32_t)row);
}

// Zeroes the n arg-max keys of q8_gemv_argmax ahead of its GEMV, as a kernel
// of the dependent-launch chain (a memset node would stop the GEMV from
// starting early): it waits for the previous grid, which may still combine
// keys into the same buffer, clears them, and lets the GEMV proceed.
__global__ void clear_keys_kernel(unsigned long long *keys, int n) {
    pdl_wait();
    for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = 0ull;
    pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// producer: one elected thread streams the tiles' TMA boxes into the ring
// ---------------------------------------------------------------------------
template <int MODE>
__device__ __forceinline__ void tile_produce(uint8_t *smem, uint32_t full0, uint32_t empty0,
                                             volatile int *abort_flag, volatile int *issued,
                                             const TileArgs &a, int u0, int u1, int total,
                                             const CUtensorMap *tq, const CUtensorMap *td,
                                             const CUtensorMap *tq1, const CUtensorMap *td1,
                                             const CUtensorMap *tx) {
    constexpr int HALVES = MODE == kModeSwiGLU ? 2 : 1;
    const uint64_t pw = policy_evict_first(), px = policy_evict_last();
    // A full tile is one box of TG units for the q bytes and one for the
    // scales (two TMA instructions: each costs tens of ns to issue); the
    // partial last tile of a CTA's range is fetched unit by unit so that
    // nothing outside the range is read.
    // The ring position (slot, phase) and the tile position (tile, k step) of
    // iteration `it` are carried along, not divided out of `it` (an integer
    // division by a runtime value costs tens of instructions).
    auto issue_weights = [&](int slot, int tile, int ks) {
        const int ut = u0 + tile * a.TG;
        const int tga = min(a.TG, u1 - ut);
        const int c0 = ks * a.CS;
        const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
        const uint32_t full = full0 + 8 * slot;
        mbar_arrive_expect_tx(full, HALVES * tga * (a.q_box + a.d_box) + a.x_box);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
            const int g0 = ut + (h ? a.up_group0 : 0);
            const uint32_t qd = st + (h ? a.q_half : 0u), dd = st + a.d_off + (h ? a.d_half : 0u);
            if (tga == a.TG) {
                tma_load_3d(qd, tq, full, 0, c0, g0, pw);
                tma_load_3d(dd, td, full, 0, c0 >> 1, g0, pw);
            } else {
                for (int g = 0; g < tga; ++g) {
                    tma_load_3d(qd + g * a.q_box, tq1, full, 0, c0, g0 + g, pw);
                    tma_load_3d(dd + g * a.d_box, td1, full, 0, c0 >> 1, g0 + g, pw);
                }
            }
        }
    };
    auto issue_x = [&](int slot, int ks) {
        const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
        tma_load_3d(st + a.x_off, tx, full0 + 8 * slot, 0, ks * a.CS, 0, px);
    };
    const int pro = total < a.stages ? total : a.stages;
    int it = 0, tile = 0, ks = 0;
    for (; it < pro; ++it) {  // weights never depend on the previous grid
        issue_weights(it, tile, ks);
        if (++ks == a.ksteps) { ks = 0; ++tile; }
    }
    pdl_wait_and_trigger();  // activations may
    {
        int kx = 0;
        for (int k = 0; k < pro; ++k) {
            issue_x(k, kx);
            if (++kx == a.ksteps) kx = 0;
        }
    }
    int slot = pro % a.stages, phase = pro / a.stages;  // ring position of iteration `pro`
    for (; it < total; ++it) {
        if (!mbar_wait(empty0 + 8 * slot, (phase & 1) ^ 1, abort_flag)) break;
        issue_weights(slot, tile, ks);
        issue_x(slot, ks);
        if (++ks == a.ksteps) { ks = 0; ++tile; }
        if (++slot == a.stages) { slot = 0; ++phase; }
    }
    *issued = it;
}

// A wait gave up somewhere: make sure no copy is still landing in this CTA's
// shared memory before it exits.
__device__ __forceinline__ void tile_drain(uint32_t full0, const TileArgs &a, int n_issued) {
    for (int it = n_issued > a.stages ? n_issued - a.stages : 0; it < n_issued; ++it)
        mbar_drain(full0 + 8 * (it % a.stages), (it / a.stages) & 1);
}

// ---------------------------------------------------------------------------
// Column-owner kernel (N <= 4)
// ---------------------------------------------------------------------------
// Consumer warp lw of group cg takes the 4-column quads cq = lw, lw + 8, ...
// of every stage whose index is cg modulo the number of groups; a lane keeps
// its column's activations in registers and runs every unit of the tile
// against them, so each column gives TGM independent dequant + dot chains and
// activations are read once per column.  At the end of a tile each warp
// leaves its partial sums in a double-buffered shared area and moves on; a
// reducer warp adds the partials of every unit in warp order and stores the
// outputs, so no consumer ever waits on a CTA-wide barrier.
template <int NMAX, int MODE, int CW_>
struct ColsCfg {
    static constexpr int CW = CW_;                           // consumer warps (8 or 16)
    static constexpr int WPG = 8;                            // warps per consumer group
    static constexpr int GROUPS = CW / WPG;                  // groups alternate stages
    static constexpr int TGM = (MODE == kModeSwiGLU ? 4 : 8) / (NMAX == 4 ? 2 : 1);
    static constexpr int H = MODE == kModeSwiGLU ? 2 : 1;
    static constexpr int THREADS = (CW + 2) * 32;            // + producer + reducer
    static constexpr int RED_FLOATS = 2 * CW * TGM * H * NMAX * 8;
};

// One column of every unit of the tile for lane (r, j).  GUARD = false is the
// full-tile path: no per-unit branch, so the compiler can overlap the
// independent per-unit chains (shared loads, dequantisation, dot products).
template <int NMAX, int MODE, int TGM, bool GUARD>
__device__ __forceinline__ void cols_step(const uint8_t *st, const TileArgs &a, int ks, int col,
                                          int cols, int r, int j, int tga,
                                          float (&acc)[TGM][MODE == kModeSwiGLU ? 2 : 1][NMAX]) {
    constexpr int H = MODE == kModeSwiGLU ? 2 : 1;
    if (MODE == kModeQ8Q8) {
        // every lane takes part (the block halves meet in a shuffle); columns
        // past K are zero-filled and add nothing
        const int blk = min((ks * a.CS + col) >> 1, a.B - 1);
        uint4 xv[NMAX];
        float dx[NMAX];
#pragma unroll
        for (int n = 0; n < NMAX; ++n) {
            if (n < a.N) {
                xv[n] = *reinterpret_cast<const uint4 *>(st + a.x_off + (n * a.CS + col) * 16);
                dx[n] = __half2float(__ushort_as_half(__ldg(a.xd + (size_t)n * a.B + blk)));
            }
        }
#pragma unroll
        for (int g = 0; g < TGM; ++g) {
            if (!GUARD || g < tga) {
                const uint4 qb = *reinterpret_cast<const uint4 *>(st + g * a.q_box + col * kColBytes + r * 16);
                const uint32_t w0 = qb.x ^ 0x80808080u, w1 = qb.y ^ 0x80808080u, w2 = qb.z ^ 0x80808080u,
                               w3 = qb.w ^ 0x80808080u;
                const float dw = __half2float(*reinterpret_cast<const __half *>(
                    st + a.d_off + g * a.d_slot + (col >> 1) * 16 + r * 2));
#pragma unroll
                for (int n = 0; n < NMAX; ++n) {
                    if (n < a.N) {
                        int dot = dp4a_s8(w0, xv[n].x, 0);
                        dot = dp4a_s8(w1, xv[n].y, dot);
                        dot = dp4a_s8(w2, xv[n].z, dot);
                        dot = dp4a_s8(w3, xv[n].w, dot);
                        dot += __shfl_xor_sync(0xffffffffu, dot, 8);
                        if ((j & 1) == 0) acc[g][0][n] = fmaf((float)dot, dw * dx[n], acc[g][0][n]);
                    }
                }
            }
        }
    } else if (col < cols) {
        ulonglong2 xr[NMAX][4];
#pragma unroll
        for (int n = 0; n < NMAX; ++n) {
            if (n < a.N) {
                const ulonglong2 *xv = reinterpret_cast<const ulonglong2 *>(st + a.x_off + (n * a.CS + col) * 64);
                xr[n][0] = xv[0];
                xr[n][1] = xv[1];
                xr[n][2] = xv[2];
                xr[n][3] = xv[3];
            }
        }
#pragma unroll
        for (int g = 0; g < TGM; ++g) {
            if (!GUARD || g < tga) {
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    ColPiece pc;
                    load_piece(st, a, h ? a.q_half : 0u, h ? a.d_half : 0u, g, col, r, pc);
#pragma unroll
                    for (int n = 0; n < NMAX; ++n)
                        if (n < a.N)
                            acc[g][h][n] = fmaf(dot16_x2(pc.w, xr[n][0], xr[n][1], xr[n][2], xr[n][3]), pc.d,
                                                acc[g][h][n]);
                }
            }
        }
    }
}

template <int NMAX, int MODE, int CW_>
__global__ void __launch_bounds__(ColsCfg<NMAX, MODE, CW_>::THREADS, 1)
    cols_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap td,
                const __grid_constant__ CUtensorMap tq1, const __grid_constant__ CUtensorMap td1,
                const __grid_constant__ CUtensorMap tx, const TileArgs a) {
    using Cfg = ColsCfg<NMAX, MODE, CW_>;
    constexpr int TGM = Cfg::TGM, H = Cfg::H, CW = Cfg::CW, WPG = Cfg::WPG;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)a.stages * a.stage_bytes);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);
    const uint32_t redfull0 = smem_u32(bars + 2 * a.stages), redfree0 = redfull0 + 16;
    float *red = reinterpret_cast<float *>(bars + 2 * a.stages + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(red + Cfg::RED_FLOATS);
    volatile int *issued = abort_flag + 1;

    // units * grid < 2^31 is checked on the host, so 32-bit math is exact here
    const int u0 = (int)(((unsigned)a.units * blockIdx.x) / gridDim.x);
    const int u1 = (int)(((unsigned)a.units * (blockIdx.x + 1)) / gridDim.x);
    const int n_tiles = (u1 - u0 + a.TG - 1) / a.TG;
    const int total = n_tiles * a.ksteps;
    const int used_stages = total < a.stages ? total : a.stages;
    if (threadIdx.x == 0) {
        for (int s = 0; s < used_stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, WPG);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(redfull0 + 8 * p, CW);
            mbar_init(redfree0 + 8 * p, 1);
        }
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CW) {
        if (lane == 0)
            tile_produce<MODE>(smem, full0, empty0, abort_flag, issued, a, u0, u1, total, &tq, &td,
                               &tq1, &td1, &tx);
        else
            pdl_wait_and_trigger();
    } else if (warp == CW + 1) {
        // ------------------------------ reducer -------------------------------
        pdl_wait_and_trigger();  // the outputs may still be read by the previous grid
        unsigned long long bestk[NMAX];  // q8_gemv_argmax: this lane's best key per column
#pragma unroll
        for (int n = 0; n < NMAX; ++n) bestk[n] = 0ull;
        for (int tl = 0; tl < n_tiles; ++tl) {
            const int p = tl & 1;
            const bool ok = mbar_wait(redfull0 + 8 * p, (tl >> 1) & 1, abort_flag);
            const int ut = u0 + tl * a.TG;
            const int tga = min(a.TG, u1 - ut);
            if (ok) {
                for (int o = lane; o < tga * 8; o += 32) {
                    const int g = o >> 3, rr = o & 7;
                    float v[H][NMAX];
#pragma unroll
                    for (int h = 0; h < H; ++h)
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) {
                            float sum = 0.f;
#pragma unroll
                            for (int w = 0; w < CW; ++w)
                                sum += red[(((((p * CW + w) * TGM + g) * H + h) * NMAX + n) << 3) + rr];
                            v[h][n] = sum;
                        }
                    store_unit<NMAX, MODE>(a, ut + g, rr, v[0], v[H - 1]);
                    const int row = (ut + g) * kGroupRows + rr;
                    if (MODE == kModeF32 && a.best && row < a.M_out) {
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) {
                            const unsigned long long k = argmax_key(v[0][n], row);
                            bestk[n] = k > bestk[n] ? k : bestk[n];
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(redfree0 + 8 * p);
        }
        if (MODE == kModeF32 && a.best) {
            // one atomic per column and CTA; the keys were zeroed before the launch
#pragma unroll
            for (int n = 0; n < NMAX; ++n) {
                unsigned long long k = bestk[n];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const unsigned long long t = __shfl_xor_sync(0xffffffffu, k, o);
                    k = t > k ? t : k;
                }
                if (lane == 0 && n < a.N && k != 0ull) atomicMax(a.best + n, k);
            }
        }
    } else {
        // ------------------------------ consumers -----------------------------
        const int cw = warp, cg = cw / WPG, lw = cw % WPG, r = lane & 7, j = lane >> 3;
        pdl_wait_and_trigger();  // Q8Q8: activation scales are read straight from memory
        int it = 0, slot = 0, phase = 0;  // ring position of iteration `it`, carried along
        for (int tl = 0; tl < n_tiles; ++tl) {
            const int ut = u0 + tl * a.TG;
            const int tga = min(a.TG, u1 - ut);
            float acc[TGM][H][NMAX];
#pragma unroll
            for (int g = 0; g < TGM; ++g)
#pragma unroll
                for (int h = 0; h < H; ++h)
#pragma unroll
                    for (int n = 0; n < NMAX; ++n) acc[g][h][n] = 0.f;
            for (int ks = 0; ks < a.ksteps;
                 ++ks, ++it, slot = slot + 1 == a.stages ? 0 : slot + 1, phase ^= slot == 0 ? 1 : 0) {
                if (it % Cfg::GROUPS != cg) continue;
                // With two groups a slot can pass from one group to the other
                // (odd ring): wait for the release of the slot's previous
                // stage, as the producer does, before waiting for this fill.
                // Otherwise, while that stage is still in flight, the previous
                // phase of `full` has the parity this wait asks for.
                bool ready = true;
                if (Cfg::GROUPS > 1 && it >= a.stages)
                    ready = mbar_wait(empty0 + 8 * slot, phase ^ 1, abort_flag);
                if (ready && mbar_wait(full0 + 8 * slot, phase, abort_flag)) {
                    const uint8_t *st = smem + (size_t)slot * a.stage_bytes;
                    const int cols = min(a.CS, a.C - ks * a.CS);
                    const int nq = (cols + 3) >> 2;
                    for (int cq = lw; cq < nq; cq += WPG) {
                        const int col = 4 * cq + j;
                        if (tga == TGM)
                            cols_step<NMAX, MODE, TGM, false>(st, a, ks, col, cols, r, j, tga, acc);
                        else
                            cols_step<NMAX, MODE, TGM, true>(st, a, ks, col, cols, r, j, tga, acc);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty0 + 8 * slot);
            }
            // lanes r, r+8, r+16, r+24 hold partial sums of the same row
#pragma unroll
            for (int g = 0; g < TGM; ++g)
#pragma unroll
                for (int h = 0; h < H; ++h)
#pragma unroll
                    for (int n = 0; n < NMAX; ++n) {
                        acc[g][h][n] += __shfl_xor_sync(0xffffffffu, acc[g][h][n], 8);
                        acc[g][h][n] += __shfl_xor_sync(0xffffffffu, acc[g][h][n], 16);
                    }
            const int p = tl & 1;
            if (tl >= 2) mbar_wait(redfree0 + 8 * p, ((tl >> 1) - 1) & 1, abort_flag);
            if (j == 0) {
#pragma unroll
                for (int g = 0; g < TGM; ++g)
#pragma unroll
                    for (int h = 0; h < H; ++h)
#pragma unroll
                        for (int n = 0; n < NMAX; ++n)
                            red[(((((p * CW + cw) * TGM + g) * H + h) * NMAX + n) << 3) + r] = acc[g][h][n];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(redfull0 + 8 * p);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) tile_drain(full0, a, *issued);
}

// ---------------------------------------------------------------------------
// Group-owner kernel (N >= 5)
// ---------------------------------------------------------------------------
// Group owners (N >= 5): a tile of >= 8 units gives each warp one or two whole
// units (no cross-warp traffic); a smaller tile splits its (unit, quad) pairs
// evenly over the warps and adds their partial sums in warp order.
template <int NMAX, int MODE>
__device__ __forceinline__ void consume_groups(uint8_t *smem, uint32_t full0, uint32_t empty0,
                                               float *red, volatile int *abort_flag,
                                               const TileArgs &a, int u0, int u1, int n_tiles) {
    constexpr int SETS = tile_acc_sets<MODE>();
    const int cw = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane & 7, j = lane >> 3;
    pdl_wait_and_trigger();  // outputs may still be read by the previous grid
    int it = 0, slot = 0, phase = 0;  // ring position of iteration `it`, carried along
    for (int tl = 0; tl < n_tiles; ++tl) {
        const int ut = u0 + tl * a.TG;
        const int tga = min(a.TG, u1 - ut);
        const bool whole = tga >= 8;
        const int P = tga * a.NQ;
        const int p_lo = (P * cw) / kConsumerWarps, p_hi = (P * (cw + 1)) / kConsumerWarps;
        const int gs0 = p_lo / a.NQ;
        const int gs1 = p_hi > p_lo ? (p_hi - 1) / a.NQ : gs0;
        float acc[SETS][NMAX];
#pragma unroll
        for (int h = 0; h < SETS; ++h)
#pragma unroll
            for (int n = 0; n < NMAX; ++n) acc[h][n] = 0.f;
        for (int ks = 0; ks < a.ksteps;
             ++ks, ++it, slot = slot + 1 == a.stages ? 0 : slot + 1, phase ^= slot == 0 ? 1 : 0) {
            if (mbar_wait(full0 + 8 * slot, phase, abort_flag)) {
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
                constexpr int PER = SETS / 2;
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

// The group-owner kernel comes in two builds: one CTA per SM (no register
// limit but the SM's), and CTAS = 2, two CTAs per SM, each within half of it
// (96 registers a thread): twice the warps to hide the FMA latency when a
// matrix has row groups enough to fill both.  SwiGLU at 16 columns keeps one
// (its gate and up accumulators need the registers).
__host__ __device__ constexpr bool tile_two_ctas_ok(int nmax, int mode) {
    return !(mode == kModeSwiGLU && nmax == 16);
}

template <int NMAX, int MODE, int CTAS>
__global__ void __launch_bounds__(kTileThreads, CTAS)
    tile_gemm_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap td,
                     const __grid_constant__ CUtensorMap tq1, const __grid_constant__ CUtensorMap td1,
                     const __grid_constant__ CUtensorMap tx, const TileArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)a.stages * a.stage_bytes);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);
    float *red = reinterpret_cast<float *>(bars + 2 * a.stages);
    volatile int *abort_flag =
        reinterpret_cast<volatile int *>(red + tile_red_floats(NMAX, tile_acc_sets<MODE>()));
    volatile int *issued = abort_flag + 1;

    const int u0 = (int)(((unsigned)a.units * blockIdx.x) / gridDim.x);
    const int u1 = (int)(((unsigned)a.units * (blockIdx.x + 1)) / gridDim.x);
    const int n_tiles = (u1 - u0 + a.TG - 1) / a.TG;
    const int total = n_tiles * a.ksteps;
    const int used_stages = total < a.stages ? total : a.stages;
    if (threadIdx.x == 0) {
        for (int s = 0; s < used_stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kConsumerWarps);
        }
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        if (lane == 0)
            tile_produce<MODE>(smem, full0, empty0, abort_flag, issued, a, u0, u1, total, &tq, &td,
                               &tq1, &td1, &tx);
        else
            pdl_wait_and_trigger();
    } else {
        consume_groups<NMAX, MODE>(smem, full0, empty0, red, abort_flag, a, u0, u1, n_tiles);
    }
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) tile_drain(full0, a, *issued);
}

}  // namespace q8
