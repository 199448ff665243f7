// moe.cuh -- S6: grouped MoE GEMV over the routed experts, in three launches.
//
// A "segment" is one expert in use (the experts present in idx, ascending
// id) or the shared expert (last); it serves cnt tokens.  Both weight
// launches walk (segment, 8-row group) work items, so a selected expert's
// weights stream once for all of its tokens and nothing else is read:
//
//   launch 1 (gate/up): items are (segment, gate group); each computes
//     h = SiLU(gate x) * up x for the segment's tokens.  A routed pair's h is
//     stored already multiplied by its routing weight, in expert-sorted pair
//     order (pairs of one expert are consecutive rows of the workspace);
//   launch 2 (down): items are (segment, output group); each multiplies the
//     segment's down rows by the segment's h rows and writes that segment's
//     partial output for each of its tokens, at the pair's original index
//     t * k + s (shared expert: after them);
//   launch 3 (sum): y[t] = the token's partials in ascending expert id, then
//     the shared expert's: a fixed order, so results are bit-identical from
//     run to run, and no atomics.
//
// Each CTA of launches 1 and 2 rebuilds the same expert table from idx at
// start (after waiting for the router).  The weight pipeline is the tile
// kernels' (a producer thread issuing TMA boxes into an mbarrier ring,
// bounded waits, drain on abort).  A stage holds CS 16-byte columns of the
// tile's items and one TMA box per token of the segment (only the segment's
// own activation rows); consumers use the column-owner mapping.
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
    float *hbuf;            // workspace: [T*k][I] routed h (expert-sorted pair rows)
    float *hsh;             // workspace: [T][Is] shared h
    float *part;            // workspace: [T*k + T][H] partial outputs of launch 2
    float *y;               // [T][H]
    int TG, CS, stages;
    uint32_t q_box;         // bytes of one item's q box (CS * 128)
    uint32_t d_box;         // bytes of one item's scale box (CS * 8)
    uint32_t x_row;         // bytes of one token's activation box (CS * 64)
    uint32_t q_half, d_off, d_half, x_off, stage_bytes;
};

struct MoeTable {
    int n_seg;                         // routed segments, then the shared one (if any)
    int n_routed;
    int seg_expert[kMoeMaxSeg];        // expert id, -1 for the shared expert
    int seg_row0[kMoeMaxSeg];          // first pair row (routed)
    int seg_cnt[kMoeMaxSeg];           // tokens using it
    int seg_unit0[kMoeMaxSeg + 1];     // first work item (flattened, for this launch)
    short pair_tok[kMoeMaxPairs];      // pair row -> token
    short pair_slot[kMoeMaxPairs];     // pair row -> slot
    int counts[kMoeMaxE];
};

// Build the table with all threads of the CTA (idx must be readable).
// `items_routed` / `items_shared`: work items of one routed / the shared
// segment in this launch.
__device__ __forceinline__ void moe_build_table(MoeTable &tb, const MoeArgs &a, int items_routed,
                                                int items_shared) {
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
    if (tid == 0) {
        int u = 0;
        for (int s = 0; s < tb.n_seg; ++s) {
            tb.seg_unit0[s] = u;
            u += tb.seg_expert[s] < 0 ? items_shared : items_routed;
        }
        tb.seg_unit0[tb.n_seg] = u;
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

// index of the segment holding flattened work item u
__device__ __forceinline__ int moe_seg_of_unit(const MoeTable &tb, int u) {
    int lo = 0, hi = tb.n_seg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb.seg_unit0[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Tiles: runs of <= TG consecutive items of one segment inside the CTA's
// range.  Walk them with this cursor.
struct MoeTile {
    int seg, ut, tga;  // segment, first item (flattened), items
};

__device__ __forceinline__ MoeTile moe_tile(const MoeTable &tb, const MoeArgs &a, int u, int u1) {
    MoeTile t;
    t.seg = moe_seg_of_unit(tb, u);
    t.ut = u;
    t.tga = min(min(a.TG, u1 - u), tb.seg_unit0[t.seg + 1] - u);
    return t;
}

// K of a segment in 16-byte columns: launch 1 reads x (H wide) for every
// segment; launch 2 reads the segment's h (I wide, Is for the shared expert).
template <int STAGE>
__device__ __forceinline__ int moe_seg_cols(const MoeArgs &a, bool shared) {
    return STAGE == 1 ? a.H / 16 : (shared ? a.Is : a.I) / 16;
}

// The stages of one tile for a consumer warp: NX >= cnt token entries (a
// compile-time bound, so the per-token chains unroll), TGM items with no
// per-item branch (a tile with fewer items recomputes its last one; those
// sums are never stored).  Leaves the warp's per-row partials in `red`.
template <int STAGE, int NX, int TGM, int NMAX>
__device__ __forceinline__ void moe_tile_compute(const uint8_t *smem, const MoeArgs &a, uint32_t full0,
                                                 uint32_t empty0, volatile int *abort_flag, int &it, int ks_n,
                                                 int cols_seg, int tga, int cnt, float *red) {
    constexpr int H = STAGE == 1 ? 2 : 1;
    const int cw = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane & 7, j = lane >> 3;
    float acc[TGM][H][NX];
#pragma unroll
    for (int g = 0; g < TGM; ++g)
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
            for (int n = 0; n < NX; ++n) acc[g][h][n] = 0.f;
    for (int ks = 0; ks < ks_n; ++ks, ++it) {
        const int slot = it % a.stages;
        if (mbar_wait_warp(full0 + 8 * slot, (it / a.stages) & 1, abort_flag)) {
            const uint8_t *st = smem + (size_t)slot * a.stage_bytes;
            const int cols = min(a.CS, cols_seg - ks * a.CS);
            const int nq = (cols + 3) >> 2;
            for (int cq = cw; cq < nq; cq += kMoeWarps) {
                const int col = 4 * cq + j;
                if (col >= cols) continue;
                // token entries past cnt read row cnt - 1 again (unstored); up to
                // four tokens' activations stay in registers for all items
                constexpr int XR = NX <= 4 ? NX : 1;
                ulonglong2 xr[XR][4];
                if (NX <= 4) {
#pragma unroll
                    for (int n = 0; n < XR; ++n) {
                        const int nn = n < cnt ? n : cnt - 1;
                        const ulonglong2 *xv =
                            reinterpret_cast<const ulonglong2 *>(st + a.x_off + nn * a.x_row + col * 64);
                        xr[n][0] = xv[0];
                        xr[n][1] = xv[1];
                        xr[n][2] = xv[2];
                        xr[n][3] = xv[3];
                    }
                }
#pragma unroll
                for (int g = 0; g < TGM; ++g) {
                    const int gu = g < tga ? g : tga - 1;
#pragma unroll
                    for (int h = 0; h < H; ++h) {
                        ColPiece pc;
                        moe_load_piece(st, a, h ? a.q_half : 0u, h ? a.d_half : 0u, gu, col, r, pc);
#pragma unroll
                        for (int n = 0; n < NX; ++n) {
                            if (NX <= 4) {
                                acc[g][h][n] = fmaf(dot16_x2(pc.w, xr[n % XR][0], xr[n % XR][1], xr[n % XR][2],
                                                             xr[n % XR][3]),
                                                    pc.d, acc[g][h][n]);
                            } else {
                                const int nn = n < cnt ? n : cnt - 1;
                                const ulonglong2 *xv =
                                    reinterpret_cast<const ulonglong2 *>(st + a.x_off + nn * a.x_row + col * 64);
                                acc[g][h][n] = fmaf(dot16_x2(pc.w, xv[0], xv[1], xv[2], xv[3]), pc.d, acc[g][h][n]);
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
            for (int n = 0; n < NX; ++n) {
                acc[g][h][n] += __shfl_xor_sync(0xffffffffu, acc[g][h][n], 8);
                acc[g][h][n] += __shfl_xor_sync(0xffffffffu, acc[g][h][n], 16);
            }
    if (j == 0) {
#pragma unroll
        for (int g = 0; g < TGM; ++g)
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
                for (int n = 0; n < NX; ++n)
                    red[((((cw * TGM + g) * H + h) * NMAX + n) << 3) + r] = acc[g][h][n];
    }
}

// First work item of CTA c of `grid`: the first item starting at or after
// work position W * c / grid, where an item's work is its segment's stage
// count and W the total.  Monotone in c, 0 at c = 0 and U at c = grid, so the
// CTAs' ranges partition the items.
template <int STAGE>
__device__ __forceinline__ int moe_work_split(const MoeTable &tb, const MoeArgs &a, int c, int grid) {
    long long W = 0;
    for (int s = 0; s < tb.n_seg; ++s) {
        const int ks = (moe_seg_cols<STAGE>(a, tb.seg_expert[s] < 0) + a.CS - 1) / a.CS;
        W += (long long)(tb.seg_unit0[s + 1] - tb.seg_unit0[s]) * ks;
    }
    const long long P = W * c / grid;
    long long w0 = 0;
    for (int s = 0; s < tb.n_seg; ++s) {
        const int ks = (moe_seg_cols<STAGE>(a, tb.seg_expert[s] < 0) + a.CS - 1) / a.CS;
        const long long ws = (long long)(tb.seg_unit0[s + 1] - tb.seg_unit0[s]) * ks;
        if (P < w0 + ws) return tb.seg_unit0[s] + (int)((P - w0 + ks - 1) / ks);
        w0 += ws;
    }
    return tb.seg_unit0[tb.n_seg];
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
    moe_build_table(tb, a, (STAGE == 1 ? a.I : a.H) / kGroupRows, (STAGE == 1 ? a.Is : a.H) / kGroupRows);

    // this CTA's range of work items, balanced by work (an item's stages:
    // the shared expert's down items are longer), then its tiles and stages
    const int u0 = moe_work_split<STAGE>(tb, a, blockIdx.x, gridDim.x);
    const int u1 = moe_work_split<STAGE>(tb, a, blockIdx.x + 1, gridDim.x);
    int n_tiles = 0, total = 0;
    for (int u = u0; u < u1;) {
        const MoeTile t = moe_tile(tb, a, u, u1);
        u += t.tga;
        ++n_tiles;
        total += (moe_seg_cols<STAGE>(a, tb.seg_expert[t.seg] < 0) + a.CS - 1) / a.CS;
    }
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
                const MoeTile t = moe_tile(tb, a, u, u1);
                u += t.tga;
                const bool shared = tb.seg_expert[t.seg] < 0;
                const int ks_n = (moe_seg_cols<STAGE>(a, shared) + a.CS - 1) / a.CS;
                const int cnt = tb.seg_cnt[t.seg], row0 = tb.seg_row0[t.seg];
                const int in_seg = t.ut - tb.seg_unit0[t.seg];
                // packed group of the tile's first item, and the gate -> up distance
                int g0, up;
                if (STAGE == 1) {
                    const int gates = (shared ? a.Is : a.I) / kGroupRows;
                    g0 = (shared ? 0 : tb.seg_expert[t.seg] * 2 * gates) + in_seg;
                    up = gates;
                } else {
                    g0 = (shared ? 0 : tb.seg_expert[t.seg] * (a.H / kGroupRows)) + in_seg;
                    up = 0;
                }
                const CUtensorMap *mq = shared ? &tq_s : &tq_r;
                const CUtensorMap *md = shared ? &td_s : &td_r;
                const CUtensorMap *mx = (STAGE == 2 && shared) ? &tx_s : &tx_r;
                for (int ks = 0; ks < ks_n; ++ks, ++it) {
                    const int slot = it % a.stages;
                    if (it >= a.stages && !mbar_wait(empty0 + 8 * slot, ((it / a.stages) & 1) ^ 1, abort_flag)) {
                        *issued = it;
                        goto producer_done;
                    }
                    {
                        const int c0 = ks * a.CS;
                        const uint32_t st = smem_u32(smem + (size_t)slot * a.stage_bytes);
                        const uint32_t full = full0 + 8 * slot;
                        mbar_arrive_expect_tx(full, H * t.tga * (a.q_box + a.d_box) + cnt * a.x_row);
                        for (int g = 0; g < t.tga; ++g)
#pragma unroll
                            for (int h = 0; h < H; ++h) {
                                tma_load_3d(st + (h ? a.q_half : 0u) + g * a.q_box, mq, full, 0, c0, g0 + g + h * up, pw);
                                tma_load_3d(st + a.d_off + (h ? a.d_half : 0u) + g * a.d_box, md, full, 0, c0 >> 1,
                                            g0 + g + h * up, pw);
                            }
                        // the segment's own activation rows, one box each
                        for (int n = 0; n < cnt; ++n) {
                            const int row = shared ? n : (STAGE == 1 ? (int)tb.pair_tok[row0 + n] : row0 + n);
                            tma_load_3d(st + a.x_off + n * a.x_row, mx, full, 0, c0, row, px);
                        }
                    }
                }
            }
            *issued = it;
        producer_done:;
        }
    } else {
        // ------------------------------ consumers -----------------------------
        int it = 0, u = u0;
        for (int tl = 0; tl < n_tiles; ++tl) {
            const MoeTile t = moe_tile(tb, a, u, u1);
            u += t.tga;
            const bool shared = tb.seg_expert[t.seg] < 0;
            const int cols_seg = moe_seg_cols<STAGE>(a, shared);
            const int ks_n = (cols_seg + a.CS - 1) / a.CS;
            const int cnt = tb.seg_cnt[t.seg];
            // the segment's token count, rounded up to a power of two <= NMAX
            if (NMAX == 1 || cnt <= 1)
                moe_tile_compute<STAGE, 1, TGM, NMAX>(smem, a, full0, empty0, abort_flag, it, ks_n, cols_seg, t.tga, cnt, red);
            else if (NMAX == 2 || cnt <= 2)
                moe_tile_compute<STAGE, (NMAX < 2 ? NMAX : 2), TGM, NMAX>(smem, a, full0, empty0, abort_flag, it, ks_n,
                                                                          cols_seg, t.tga, cnt, red);
            else if (NMAX == 4 || cnt <= 4)
                moe_tile_compute<STAGE, (NMAX < 4 ? NMAX : 4), TGM, NMAX>(smem, a, full0, empty0, abort_flag, it, ks_n,
                                                                          cols_seg, t.tga, cnt, red);
            else if (NMAX == 8 || cnt <= 8)
                moe_tile_compute<STAGE, (NMAX < 8 ? NMAX : 8), TGM, NMAX>(smem, a, full0, empty0, abort_flag, it, ks_n,
                                                                          cols_seg, t.tga, cnt, red);
            else
                moe_tile_compute<STAGE, NMAX, TGM, NMAX>(smem, a, full0, empty0, abort_flag, it, ks_n, cols_seg,
                                                         t.tga, cnt, red);
            named_barrier(1, kMoeWarps * 32);
            // outputs: (item g, row rr, token entry n), warps' partials added in warp order
            const int in_seg = t.ut - tb.seg_unit0[t.seg];
            const int row0 = tb.seg_row0[t.seg];
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
                const int row = (in_seg + g) * kGroupRows + rr;  // row of h (launch 1) or of y (launch 2)
                if (STAGE == 1) {
                    const float hval = silu_mul(v[0], v[H - 1]);
                    if (shared) {
                        a.hsh[(size_t)n * a.Is + row] = hval;
                    } else {
                        const int pr = row0 + n;
                        a.hbuf[(size_t)pr * a.I + row] = hval * a.w[tb.pair_tok[pr] * a.k + tb.pair_slot[pr]];
                    }
                } else {
                    const int dst = shared ? a.T * a.k + n : tb.pair_tok[row0 + n] * a.k + tb.pair_slot[row0 + n];
                    a.part[(size_t)dst * a.H + row] = v[0];
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

// Launch 3: y[t][h] = the token's routed partials in ascending expert id (a
// repeated pick of one expert in slot order), then the shared expert's.  An
// out-of-range pick contributes nothing.
__global__ void moe_sum_kernel(const int32_t *__restrict__ idx, const float *__restrict__ part,
                               float *__restrict__ y, int T, int E, int k, int H, int has_shared) {
    pdl_wait_and_trigger();
    const int total = T * H;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
        const int t = i / H, h = i - t * H;
        float s = 0.f;
        int last = -1;  // key e * k + slot of the pick added last
        for (int r = 0; r < k; ++r) {
            int best = -1, best_key = 0x7fffffff;
            for (int q = 0; q < k; ++q) {
                const int e = idx[t * k + q];
                if (e < 0 || e >= E) continue;
                const int key = e * k + q;
                if (key > last && key < best_key) {
                    best_key = key;
                    best = q;
                }
            }
            if (best < 0) break;
            s += part[(size_t)(t * k + best) * H + h];
            last = best_key;
        }
        if (has_shared) s += part[(size_t)(T * k + t) * H + h];
        y[i] = s;
    }
}

}  // namespace q8
