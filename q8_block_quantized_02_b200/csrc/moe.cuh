// moe.cuh -- S6: grouped MoE GEMV over the routed experts, in two launches.
//
//   launch 1 (gate/up): for every selected expert and for the shared expert,
//     h = SiLU(gate x) * up x for the tokens that use it.  Work units are
//     (expert, 8-row gate group) pairs, so an expert picked by several tokens
//     streams its weights once and serves all of them.  A routed pair's h is
//     stored already multiplied by its routing weight, in expert-sorted pair
//     order (pairs of one expert are consecutive rows of the workspace).
//   launch 2 (down + sum): for every 8-row group of the output, the K stream
//     is the concatenation of the selected experts' down rows (ascending
//     expert id) and the shared expert's; each stage multiplies one slice of
//     one expert by that expert's workspace rows, so y[t] is accumulated in a
//     fixed order without atomics.
//
// Each CTA rebuilds the same expert table from idx at start (after waiting for
// the router): experts present in idx, ascending; for each, its (token, slot)
// pairs in token order.  The weight pipeline is the tile kernels' (producer
// warp issuing TMA boxes into an mbarrier ring, bounded waits, drain on
// abort); consumers use the column-owner mapping with activations read from
// the staged box for each token of the current expert.
#pragma once

#include "tile_gemm.cuh"

namespace q8 {

constexpr int kMoeMaxT = 16;
constexpr int kMoeMaxK = 8;
constexpr int kMoeMaxE = 256;
constexpr int kMoeMaxPairs = kMoeMaxT * kMoeMaxK;
constexpr int kMoeMaxSeg = kMoeMaxPairs + 1;  // routed experts + shared expert
constexpr int kMoeWarps = 8;                  // consumer warps
constexpr int kMoeThreads = (kMoeWarps + 1) * 32;

struct MoeArgs {
    int T, E, k, H, I, Is;  // Is = 0: no shared expert
    const int32_t *idx;     // [T][k]
    const float *w;         // [T][k]
    float *hbuf;            // workspace: [T*k][I] routed h (expert-sorted pairs)
    float *hsh;             // workspace: [T][Is] shared h
    float *y;               // [T][H]
    int units_out;          // launch 2: H / 8
    int TG, CS, stages;
    uint32_t q_box, d_box, x_box, q_half, d_off, d_half, x_off, stage_bytes;
};

struct MoeTable {
    int n_seg;                         // routed segments, then the shared one (if any)
    int n_routed;
    int seg_expert[kMoeMaxSeg];        // expert id, -1 for the shared expert
    int seg_row0[kMoeMaxSeg];          // first pair row (routed)
    int seg_cnt[kMoeMaxSeg];           // tokens using it
    int seg_unit0[kMoeMaxSeg + 1];     // launch 1: first flattened unit
    int seg_kstep0[kMoeMaxSeg + 1];    // launch 2: first stage of the segment in a tile
    short pair_tok[kMoeMaxPairs];      // pair row -> token
    short pair_slot[kMoeMaxPairs];     // pair row -> slot
    signed char box_row[kMoeMaxSeg][kMoeMaxT];  // launch 2: token -> row of the x box, or -1
    int counts[kMoeMaxE];
};

// Build the table with all threads of the CTA (idx must be readable).
__device__ __forceinline__ void moe_build_table(MoeTable &tb, const MoeArgs &a, int stage_kind) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int P = a.T * a.k;
    for (int e = tid; e < kMoeMaxE; e += nthr) tb.counts[e] = 0;
    __syncthreads();
    for (int p = tid; p < P; p += nthr) {
        int e = a.idx[p];
        if (e < 0 || e >= a.E) {
            record_error(kErrBadExpert);
            continue;  // an out-of-range pick contributes nothing
        }
        atomicAdd(&tb.counts[e], 1);
    }
    __syncthreads();
    if (tid < 32) {
        // ascending scan over experts: segment index and first pair row
        int seg_base = 0, row_base = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + tid;
            const int c = e < a.E ? tb.counts[e] : 0;
            const unsigned present = __ballot_sync(0xffffffffu, c > 0);
            int incl = c;  // inclusive prefix of counts over lanes
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (tid >= off) incl += v;
            }
            if (c > 0) {
                const int sidx = seg_base + __popc(present & ((1u << tid) - 1u));
                tb.seg_expert[sidx] = e;
                tb.seg_cnt[sidx] = c;
                tb.seg_row0[sidx] = row_base + incl - c;
            }
            seg_base += __popc(present);
            row_base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) {
            tb.n_routed = seg_base;
            int n = seg_base;
            if (a.Is > 0) {
                tb.seg_expert[n] = -1;
                tb.seg_cnt[n] = a.T;
                tb.seg_row0[n] = 0;
                ++n;
            }
            tb.n_seg = n;
        }
    }
    __syncthreads();
    // pair rows: pair p = t*k + s goes to row seg_row0[its segment] + (earlier pairs of the same expert)
    for (int p = tid; p < P; p += nthr) {
        const int e = a.idx[p];
        if (e < 0 || e >= a.E) continue;
        int before = 0;
        for (int q = 0; q < p; ++q) before += (a.idx[q] == e);
        // segment of expert e: experts present below e
        int lo = 0, hi = tb.n_routed - 1;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (tb.seg_expert[mid] < e) lo = mid + 1; else hi = mid;
        }
        const int row = tb.seg_row0[lo] + before;
        tb.pair_tok[row] = (short)(p / a.k);
        tb.pair_slot[row] = (short)(p % a.k);
    }
    __syncthreads();
    if (tid == 0) {
        // launch 1 unit offsets; launch 2 stage offsets (per tile)
        int u = 0, ks = 0;
        const int c_routed = a.I / 16, c_shared = a.Is / 16;
        for (int s = 0; s < tb.n_seg; ++s) {
            tb.seg_unit0[s] = u;
            tb.seg_kstep0[s] = ks;
            const bool shared = tb.seg_expert[s] < 0;
            u += (shared ? a.Is : a.I) / kGroupRows;
            ks += ((shared ? c_shared : c_routed) + a.CS - 1) / a.CS;
        }
        tb.seg_unit0[tb.n_seg] = u;
        tb.seg_kstep0[tb.n_seg] = ks;
    }
    if (stage_kind == 2) {
        for (int i = tid; i < kMoeMaxSeg * kMoeMaxT; i += nthr) (&tb.box_row[0][0])[i] = -1;
        __syncthreads();
        for (int s = tid; s < tb.n_seg; s += nthr) {
            if (tb.seg_expert[s] < 0) {
                for (int t = 0; t < a.T; ++t) tb.box_row[s][t] = (signed char)t;
            } else {
                for (int i = 0; i < tb.seg_cnt[s]; ++i)
                    tb.box_row[s][tb.pair_tok[tb.seg_row0[s] + i]] = (signed char)i;
            }
        }
    }
    __syncthreads();
}

__device__ __forceinline__ void moe_load_piece(const uint8_t *st, const MoeArgs &a, uint32_t qoff,
                                               uint32_t doff, int g, int col, int r, ColPiece &p) {
    const uint4 q = *reinterpret_cast<const uint4 *>(st + qoff + g * a.q_box + col * kColBytes + r * 16);
    p.d = __half2float(*reinterpret_cast<const __half *>(st + a.d_off + doff + g * a.d_box +
                                                         (col >> 1) * 16 + r * 2));
    dequant16_x2(q, p.w);
}

// index of the segment holding flattened launch-1 unit u
__device__ __forceinline__ int moe_seg_of_unit(const MoeTable &tb, int u) {
    int lo = 0, hi = tb.n_seg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb.seg_unit0[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ int moe_seg_of_kstep(const MoeTable &tb, int ks) {
    int lo = 0, hi = tb.n_seg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb.seg_kstep0[mid] <= ks) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Tiles of launch 1: runs of <= TG consecutive units of one segment inside the
// CTA's range.  Walk them with this cursor.
struct MoeTile {
    int seg, ut, tga;  // segment, first unit (flattened), units
};

__device__ __forceinline__ MoeTile moe_tile1(const MoeTable &tb, const MoeArgs &a, int u, int u1) {
    MoeTile t;
    t.seg = moe_seg_of_unit(tb, u);
    t.ut = u;
    t.tga = min(min(a.TG, u1 - u), tb.seg_unit0[t.seg + 1] - u);
    return t;
}

template <int STAGE, int NMAX, int TGM>
__global__ void __launch_bounds__(kMoeThreads, 1)
    moe_kernel(const __grid_constant__ CUtensorMap tq_r, const __grid_constant__ CUtensorMap td_r,
               const __grid_constant__ CUtensorMap tq_s, const __grid_constant__ CUtensorMap td_s,
               const __grid_constant__ CUtensorMap tx_r, const __grid_constant__ CUtensorMap tx_s,
               const MoeArgs a) {
    constexpr int H = STAGE == 1 ? 2 : 1;  // launch 1 keeps gate and up sums
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)a.stages * a.stage_bytes);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);
    MoeTable &tb = *reinterpret_cast<MoeTable *>(bars + 2 * a.stages);
    float *red = reinterpret_cast<float *>(&tb + 1);
    constexpr int RED = kMoeWarps * TGM * H * NMAX * 8;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(red + RED);
    volatile int *issued = abort_flag + 1;

    pdl_wait_and_trigger();  // idx, w (router) and the activations come from earlier kernels
    moe_build_table(tb, a, STAGE);

    // this CTA's range of units
    const int U = STAGE == 1 ? tb.seg_unit0[tb.n_seg] : a.units_out;
    const int u0 = (int)(((long long)U * blockIdx.x) / gridDim.x);
    const int u1 = (int)(((long long)U * (blockIdx.x + 1)) / gridDim.x);
    const int ksteps2 = tb.seg_kstep0[tb.n_seg];  // launch 2: stages per tile
    const int ksteps1 = (a.H / 16 + a.CS - 1) / a.CS;
    const int ksteps = STAGE == 1 ? ksteps1 : ksteps2;
    // count the tiles and stages of this CTA
    int n_tiles = 0;
    for (int u = u0; u < u1;) {
        const int step = STAGE == 1 ? moe_tile1(tb, a, u, u1).tga : min(a.TG, u1 - u);
        u += step;
        ++n_tiles;
    }
    const int total = n_tiles * ksteps;
    const int used_stages = total < a.stages ? total : a.stages;
    if (threadIdx.x == 0) {
        for (int s = 0; s < used_stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kMoeWarps);
        }
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kMoeWarps) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            const uint64_t pw = policy_evict_first(), px = policy_evict_last();
            int it = 0, u = u0;
            for (int tl = 0; tl < n_tiles; ++tl) {
                MoeTile t;
                if (STAGE == 1) {
                    t = moe_tile1(tb, a, u, u1);
                } else {
                    t.seg = 0;
                    t.ut = u;
                    t.tga = min(a.TG, u1 - u);
                }
                u += t.tga;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int slot = it % a.stages;
                    if (it >= a.stages && !mbar_wait(empty0 + 8 * slot, ((it / a.stages) & 1) ^ 1, abort_flag)) {
                        *issued = it;
                        goto producer_done;
                    }
                    {
                        const int seg = STAGE == 1 ? t.seg : moe_seg_of_kstep(tb, ks);
                        const bool shared = tb.seg_expert[seg] < 0;
                        const int c0 = (STAGE == 1 ? ks : ks - tb.seg_kstep0[seg]) * a.CS;
                        const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
                        const uint32_t full = full0 + 8 * slot;
                        const CUtensorMap *mq = shared ? &tq_s : &tq_r;
                        const CUtensorMap *md = shared ? &td_s : &td_r;
                        mbar_arrive_expect_tx(full, H * t.tga * (a.q_box + a.d_box) + a.x_box);
                        int g0, up;
                        if (STAGE == 1) {
                            const int in_seg = t.ut - tb.seg_unit0[seg];
                            const int gates = (shared ? a.Is : a.I) / kGroupRows;
                            g0 = (shared ? 0 : tb.seg_expert[seg] * 2 * gates) + in_seg;
                            up = gates;
                        } else {
                            g0 = (shared ? 0 : tb.seg_expert[seg] * (a.H / kGroupRows)) + t.ut;
                            up = 0;
                        }
                        for (int g = 0; g < t.tga; ++g)
#pragma unroll
                            for (int h = 0; h < H; ++h) {
                                tma_load_3d(st + (h ? a.q_half : 0u) + g * a.q_box, mq, full, 0, c0, g0 + g + h * up, pw);
                                tma_load_3d(st + a.d_off + (h ? a.d_half : 0u) + g * a.d_box, md, full, 0, c0 >> 1,
                                            g0 + g + h * up, pw);
                            }
                        if (STAGE == 1)
                            tma_load_3d(st + a.x_off, &tx_r, full, 0, c0, 0, px);
                        else if (shared)
                            tma_load_3d(st + a.x_off, &tx_s, full, 0, c0, 0, px);
                        else
                            tma_load_3d(st + a.x_off, &tx_r, full, 0, c0, tb.seg_row0[seg], px);
                    }
                }
            }
            *issued = it;
        producer_done:;
        }
    } else {
        // ------------------------------ consumers -----------------------------
        const int cw = warp, r = lane & 7, j = lane >> 3;
        int it = 0, u = u0;
        for (int tl = 0; tl < n_tiles; ++tl) {
            MoeTile t;
            if (STAGE == 1) {
                t = moe_tile1(tb, a, u, u1);
            } else {
                t.seg = 0;
                t.ut = u;
                t.tga = min(a.TG, u1 - u);
            }
            u += t.tga;
            float acc[TGM][H][NMAX];
#pragma unroll
            for (int g = 0; g < TGM; ++g)
#pragma unroll
                for (int h = 0; h < H; ++h)
#pragma unroll
                    for (int n = 0; n < NMAX; ++n) acc[g][h][n] = 0.f;
            for (int ks = 0; ks < ksteps; ++ks, ++it) {
                const int slot = it % a.stages;
                if (mbar_wait(full0 + 8 * slot, (it / a.stages) & 1, abort_flag)) {
                    const uint8_t *st = smem + (size_t)slot * a.stage_bytes;
                    const int seg = STAGE == 1 ? t.seg : moe_seg_of_kstep(tb, ks);
                    const bool shared = tb.seg_expert[seg] < 0;
                    const int cseg = (shared ? a.Is : (STAGE == 1 ? a.H : a.I)) / 16;
                    const int c_here = (STAGE == 1 ? a.H / 16 : cseg);
                    const int c0 = (STAGE == 1 ? ks : ks - tb.seg_kstep0[seg]) * a.CS;
                    const int cols = min(a.CS, c_here - c0);
                    const int nq = (cols + 3) >> 2;
                    const int cnt = tb.seg_cnt[seg];
                    for (int cq = cw; cq < nq; cq += kMoeWarps) {
                        const int col = 4 * cq + j;
                        if (col >= cols) continue;
#pragma unroll
                        for (int g = 0; g < TGM; ++g) {
                            if (g < t.tga) {
#pragma unroll
                                for (int h = 0; h < H; ++h) {
                                    ColPiece pc;
                                    moe_load_piece(st, a, h ? a.q_half : 0u, h ? a.d_half : 0u, g, col, r, pc);
#pragma unroll
                                    for (int n = 0; n < NMAX; ++n) {
                                        // launch 1: entry n of the segment's token list;
                                        // launch 2: token n, read from its box row
                                        int row;
                                        if (STAGE == 1)
                                            row = n < cnt ? (shared ? n : tb.pair_tok[tb.seg_row0[seg] + n]) : -1;
                                        else
                                            row = n < a.T ? tb.box_row[seg][n] : -1;
                                        if (row >= 0) {
                                            const ulonglong2 *xv = reinterpret_cast<const ulonglong2 *>(
                                                st + a.x_off + (row * a.CS + col) * 64);
                                            acc[g][h][n] = fmaf(dot16_x2(pc.w, xv[0], xv[1], xv[2], xv[3]), pc.d,
                                                                acc[g][h][n]);
                                        }
                                    }
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty0 + 8 * slot);
            }
#pragma unroll
            for (int g = 0; g < TGM; ++g)
#pragma unroll
                for (int h = 0; h < H; ++h)
#pragma unroll
                    for (int n = 0; n < NMAX; ++n) {
                        acc[g][h][n] += __shfl_xor_sync(0xffffffffu, acc[g][h][n], 8);
                        acc[g][h][n] += __shfl_xor_sync(0xffffffffu, acc[g][h][n], 16);
                    }
            if (j == 0) {
#pragma unroll
                for (int g = 0; g < TGM; ++g)
#pragma unroll
                    for (int h = 0; h < H; ++h)
#pragma unroll
                        for (int n = 0; n < NMAX; ++n)
                            red[((((cw * TGM + g) * H + h) * NMAX + n) << 3) + r] = acc[g][h][n];
            }
            named_barrier(1, kMoeWarps * 32);
            // outputs: (unit g, row r, entry n), warps' partials added in warp order
            const int seg = t.seg;
            const bool shared = STAGE == 1 && tb.seg_expert[seg] < 0;
            const int cnt = STAGE == 1 ? tb.seg_cnt[seg] : a.T;
            for (int o = threadIdx.x; o < t.tga * 8 * NMAX; o += kMoeWarps * 32) {
                const int n = o % NMAX, rr = (o / NMAX) & 7, g = o / (NMAX * 8);
                if (n >= cnt) continue;
                float v[H];
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    float s = 0.f;
#pragma unroll
                    for (int w = 0; w < kMoeWarps; ++w) s += red[((((w * TGM + g) * H + h) * NMAX + n) << 3) + rr];
                    v[h] = s;
                }
                if (STAGE == 1) {
                    const float hval = silu_mul(v[0], v[H - 1]);
                    const int row = (t.ut - tb.seg_unit0[seg] + g) * kGroupRows + rr;
                    if (shared) {
                        a.hsh[(size_t)n * a.Is + row] = hval;
                    } else {
                        const int pr = tb.seg_row0[seg] + n;
                        a.hbuf[(size_t)pr * a.I + row] = hval * a.w[tb.pair_tok[pr] * a.k + tb.pair_slot[pr]];
                    }
                } else {
                    a.y[(size_t)n * a.H + (t.ut + g) * kGroupRows + rr] = v[0];
                }
            }
            named_barrier(1, kMoeWarps * 32);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        const int n_issued = *issued;
        for (int it = n_issued > a.stages ? n_issued - a.stages : 0; it < n_issued; ++it)
            mbar_drain(full0 + 8 * (it % a.stages), (it / a.stages) & 1);
    }
}

}  // namespace q8
