// moe.cuh -- S6: grouped MoE GEMV over the routed experts, in one persistent
// launch.
//
// A "segment" is one expert in use (the experts present in idx, ascending id)
// or the shared expert; it serves cnt tokens.  The work is a list of items,
// each 8 rows of one segment's weights applied to all of its tokens:
//
//   phase 1 (gate/up): item (segment, gate group) computes
//     h = SiLU(gate x) * up x for the segment's tokens.  A routed pair's h is
//     stored already multiplied by its routing weight, in expert-sorted pair
//     order (the pairs of one expert are consecutive workspace rows); the
//     shared expert's h goes to a [T][I_shared] buffer;
//   phase 2 (down): item (segment, output group) multiplies the segment's 8
//     down rows by its h rows and stores one partial output row per token, at
//     the pair's index t * k + s.  The shared expert's down projection (K =
//     I_shared, several times a routed expert's K) is split along K into
//     nsplit chunks about as long as a routed expert's, each an item of its
//     own with its own partial row (T * k + chunk * T + t), so every phase-2
//     item is about as long and tiles fill their stages;
//   final sum: y[t] = the token's partials in ascending expert id, then the
//     shared expert's chunks in order -- a fixed order, so results are
//     bit-identical from run to run.  It is taken, per output group, by the CTA that finishes that
//     group's last phase-2 item (a counter per group says which one).
//
// A selected expert's weights stream once for all of its tokens, and nothing
// else is read.  One CTA runs per SM.  CTA c owns an even slice of each of
// four lists, walked in this order: the shared expert's phase-1 items (known
// before the router's output is), the routed phase-1 items, the shared
// expert's phase-2 items and the routed phase-2 items.  So the shared
// expert's gate/up weights are requested before griddepcontrol.wait and
// stream while the previous kernel on the stream finishes; every CTA's first
// phase-2 items multiply the shared expert's h, which is complete first; and
// phase-2 weights stream into free ring slots while the h they multiply is
// still being finished by other CTAs.
//
// Warp roles (CW + 3 warps):
//   * warps 0..CW-1 consume.  Warp w takes column quad w & 7 of every stage
//     and, with CW = 16, half w >> 3 of the tile's items; lane (r = lane & 7,
//     j = lane >> 3) works on row r of column 4 * (w & 7) + j, as in the tile
//     kernels;
//   * warp CW issues the weight boxes of each stage (TMA, into a ring of
//     `stages` slots guarded by full/empty mbarriers);
//   * warp CW + 1 issues the activation boxes of each stage (token rows for phase
//     1, h rows for phase 2).  Before the first stage of a phase-2 tile it
//     waits until the tile's segment has all of its phase-1 items counted
//     done (a release/acquire counter in the workspace);
//   * warp CW + 2 builds the expert table from idx (warp intrinsics only), then
//     takes each tile's epilogue: the 8 column warps' partial sums (in warp
//     order), SiLU(gate) * up or the partial outputs, the counters, and the
//     final sums of the output groups it completes.  The consumers hand it
//     their sums through kMoeRedBufs buffers and never wait for the stores.
// The workspace counters are zero between calls: the CTA that finishes a
// group's sum clears its counter and the last CTA to finish clears the
// segment counters, so a workspace must be zero-filled once before its first
// call (q8_moe_workspace_init).  Every wait is bounded (see q8_device.cuh); a
// stalled pipeline records an error, drains its in-flight copies and exits.
#pragma once

#include "tile_gemm.cuh"

namespace q8 {

constexpr int kMoeMaxT = 16;
constexpr int kMoeMaxK = 8;
constexpr int kMoeMaxE = 256;
constexpr int kMoeMaxPairs = kMoeMaxT * kMoeMaxK;
constexpr int kMoeMaxSeg = kMoeMaxPairs;       // routed segments (the shared one is apart)
// Consumer warps: 16 (8 column quads x 2 item halves) for one or two tokens,
// 8 (each warp all of a tile's items) for more, where a lane's accumulators
// need the registers that 3 warps per SM sub-partition leave (5 leave 96).
// Warps CW, CW + 1 and CW + 2 are the weight producer, the activation
// producer and the table / epilogue warp.
__host__ __device__ constexpr int moe_cw(int nmax) { return nmax <= 2 ? 16 : 8; }
__host__ __device__ constexpr int moe_threads(int nmax) { return (moe_cw(nmax) + 3) * 32; }
constexpr int kMoeCS = 32;                     // 16-byte columns per stage
constexpr uint32_t kMoeQBox = kMoeCS * kColBytes;  // one item's q box
constexpr uint32_t kMoeDBox = kMoeCS * 8;          // one item's scale box ([CS/2][8] fp16)
constexpr uint32_t kMoeXRow = kMoeCS * 64;         // one token's activation box
constexpr int kMoeMaxStages = 8;
constexpr int kMoeRedBufs = 3;                 // partial-sum buffers between consumers and the epilogue warp
constexpr int kMoeBarBytes = 256;              // mbarriers: full, empty (<= 8 each), red full/free (4 each), table
constexpr int kMoeRedMax = 64;                 // partial-sum slots per column quad and tile
constexpr int kMoePend = 32;                   // phase-2 tiles the epilogue warp counts at once
constexpr int kMoeMaxSplit = 8;                // K chunks of the shared down projection, at most

// workspace counters (32-bit words)
constexpr int kCtrCta = 0;                     // CTAs finished
constexpr int kCtrShared = 1;                  // phase-1 items done, shared expert
constexpr int kCtrRouted = 2;                  // ... routed segment s at kCtrRouted + s
constexpr int kCtrGroups = kCtrRouted + kMoeMaxSeg;  // phase-2 segments done, output group o

// Token bucket of a segment serving cnt tokens: the compile-time token count
// its tiles are computed for.
__host__ __device__ constexpr int moe_nx(int cnt) {
    return cnt <= 1 ? 1 : cnt <= 2 ? 2 : cnt <= 4 ? 4 : cnt <= 8 ? 8 : 16;
}
// Items per tile: 8 down items, or 6 gate|up pairs for up to two tokens (one
// token's gate/up slice of about 5 items stays one tile), 4 for four tokens;
// fewer for 8 and 16 tokens, so that a lane holds at most 32 accumulators
// (its items x halves x tokens).
__host__ __device__ constexpr int moe_tg(int phase, int nx) {
    return phase == 1 ? (nx <= 2 ? 6 : nx <= 4 ? 4 : 16 / nx) : (nx <= 4 ? 8 : 32 / nx);
}
__host__ __device__ constexpr int moe_halves(int phase) { return phase == 1 ? 2 : 1; }
// Relative consumer work of an item of a segment with cnt tokens: per 16
// weights, one dequantisation (~24 instructions) and one dot per token (~10).
// The routed lists are split over the CTAs by this work, not by item count.
__host__ __device__ constexpr int moe_item_work(int cnt) { return 24 + 10 * moe_nx(cnt); }
constexpr int kMoeTile1 = moe_tg(1, 1), kMoeTile2 = moe_tg(2, 1);  // the largest tiles
// A stage: the weight boxes ([half][item] q boxes, then scale boxes), then
// one activation box per token.
__host__ __device__ constexpr uint32_t moe_x_off(int phase, int nx) {
    return (uint32_t)(moe_halves(phase) * moe_tg(phase, nx)) * (kMoeQBox + kMoeDBox);
}
__host__ __device__ constexpr uint32_t moe_stage_bytes(int phase, int nx) {
    return moe_x_off(phase, nx) + (uint32_t)nx * kMoeXRow;
}

struct MoeArgs {
    int T, E, k, H, I, Is;  // Is = 0: no shared expert
    const int32_t *idx;     // [T][k]
    const float *w;         // [T][k]
    float *hbuf;            // workspace: [T*k][I] routed h (expert-sorted pair rows)
    float *hsh;             // workspace: [T][Is] shared h
    float *part;            // workspace: [T*k + nsplit*T][H] partial outputs
    float *y;               // [T][H]
    unsigned *ctr;          // workspace counters, zero between calls
    int nsplit;             // K chunks of the shared expert's down projection (0: no shared expert)
    int cc;                 // 16-byte columns per chunk (even; the last chunk may be shorter)
    int stages;             // ring slots
    uint32_t slot_bytes;    // bytes of one slot (the largest stage of this token bucket)
    int red_a;              // partial-sum slots per column quad (<= kMoeRedMax)
};

struct MoeTable {
    int n_routed;
    int seg_expert[kMoeMaxSeg];
    int seg_row0[kMoeMaxSeg];          // first pair row
    int seg_cnt[kMoeMaxSeg];           // tokens using it (<= T: picks of a token are distinct)
    int seg_w0[kMoeMaxSeg + 1];        // work of the segments before it (moe_item_work per item)
    short pair_tok[kMoeMaxPairs];      // pair row -> token
    short pair_slot[kMoeMaxPairs];     // pair row -> slot
    float pair_w[kMoeMaxPairs];        // pair row -> routing weight
    signed char tok_order[kMoeMaxT][kMoeMaxK];  // token's slots by ascending expert id, -1 after
    int pick[kMoeMaxPairs];            // idx, -1 where the pick was rejected
    union {
        int counts[kMoeMaxE];          // while building: per-expert pick count, then expert -> segment
        int last_o[kMoePend * kMoeTile2];  // at the end: output groups whose sums this CTA takes
    };
    // epilogue warp: phase-2 tiles stored but not yet counted (first group, groups)
    int pend_o0[kMoePend];
    int pend_n[kMoePend];
    int n_last;                        // groups in last_o whose sums the CTA takes at its end
    int r0, r1, v0, v1;                // this CTA's routed slices (gate/up, down), set with the table
};

static_assert(kMoeMaxE == kMoePend * kMoeTile2, "the table's counts and last_o share storage");

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_relaxed_gpu_add(unsigned *p, unsigned v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_acq_rel_gpu_add(unsigned *p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
// Orders this thread's generic-proxy accesses of global memory with its later
// TMA (async-proxy) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Wait until *p >= target (a counter other CTAs raise with release
// semantics).  Bounded like mbar_wait; false (and *abort raised) on timeout.
__device__ __forceinline__ bool wait_counter_geq(const unsigned *p, unsigned target, volatile int *abort) {
    if (ld_acquire_gpu(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        __nanosleep(64);
        if (ld_acquire_gpu(p) >= target) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(kErrWaitTimeout);
            *abort = 1;
            return false;
        }
    }
}

// Build the table with one warp (idx must be readable).  A pick outside
// [0, E), or a token's second pick of an expert, is rejected: it records
// kErrBadExpert and contributes nothing.  Everything here is a pure function
// of idx, so every CTA builds the same table.
__device__ __forceinline__ void moe_build_table(MoeTable &tb, const MoeArgs &a, int lane) {
    const int P = a.T * a.k;
    const int chunks = (P + 31) >> 5;  // <= 4
    for (int e = lane; e < a.E; e += 32) tb.counts[e] = 0;
    float wv[4];  // routing weights, loaded with idx (one round trip for both)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int p = c * 32 + lane;
        wv[c] = c < chunks && p < P ? __ldcg(a.w + p) : 0.f;
        if (c < chunks && p < P) tb.pick[p] = __ldcg(a.idx + p);
    }
    __syncwarp();
    int ev[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int p = c * 32 + lane;
        int e = -1;
        if (c < chunks && p < P) {
            e = tb.pick[p];
            bool ok = e >= 0 && e < a.E;
            const int t = p / a.k, s = p - t * a.k;
            for (int s2 = 0; ok && s2 < s; ++s2) ok = tb.pick[t * a.k + s2] != e;
            if (!ok) {
                record_error(kErrBadExpert);
                e = -1;
            }
        }
        ev[c] = e;
    }
    __syncwarp();
    // ranks within each expert in pick order, one 32-pick chunk at a time
    const unsigned lt = (1u << lane) - 1u;
    int rk[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        rk[c] = 0;
        if (c < chunks) {
            const int p = c * 32 + lane;
            if (p < P) tb.pick[p] = ev[c];
            const int e = ev[c];
            const unsigned m = __match_any_sync(0xffffffffu, e >= 0 ? e : (1 << 20) + lane);
            const int base = e >= 0 ? tb.counts[e] : 0;
            rk[c] = base + __popc(m & lt);
            __syncwarp();
            if (e >= 0 && lane == __ffs(m) - 1) tb.counts[e] = base + __popc(m);
            __syncwarp();
        }
    }
    // ascending scan over experts: segment index and first pair row
    int seg_base = 0, row_base = 0;
    for (int e0 = 0; e0 < a.E; e0 += 32) {
        const int e = e0 + lane;
        const int c = e < a.E ? tb.counts[e] : 0;
        const unsigned present = __ballot_sync(0xffffffffu, c > 0);
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (c > 0) {
            const int sidx = seg_base + __popc(present & lt);
            tb.seg_expert[sidx] = e;
            tb.seg_cnt[sidx] = c;
            tb.seg_row0[sidx] = row_base + incl - c;
            tb.counts[e] = sidx;
        }
        seg_base += __popc(present);
        row_base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tb.n_routed = seg_base;
    __syncwarp();
    // prefix of the segments' work (<= 128 segments: 4 per lane, then a scan)
    {
        int w[4], sum = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int sg = lane * 4 + i;
            w[i] = sg < seg_base ? moe_item_work(tb.seg_cnt[sg]) : 0;
            sum += w[i];
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int sg = lane * 4 + i;
            if (sg <= seg_base) tb.seg_w0[sg] = run;
            run += w[i];
        }
        if (lane == 31) tb.seg_w0[seg_base] = run;  // the total (also when seg_base = 128)
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int p = c * 32 + lane;
        if (c < chunks && ev[c] >= 0) {
            const int row = tb.seg_row0[tb.counts[ev[c]]] + rk[c];
            tb.pair_tok[row] = (short)(p / a.k);
            tb.pair_slot[row] = (short)(p % a.k);
            tb.pair_w[row] = wv[c];
        }
    }
    // each token's valid slots by ascending expert id (its picks are distinct)
    if (lane < a.T) {
        const int t = lane;
        int n = 0;
        for (int s = 0; s < a.k; ++s) {
            const int e = tb.pick[t * a.k + s];
            if (e < 0) continue;
            int i = n++;
            while (i > 0 && tb.pick[t * a.k + tb.tok_order[t][i - 1]] > e) {
                tb.tok_order[t][i] = tb.tok_order[t][i - 1];
                --i;
            }
            tb.tok_order[t][i] = (signed char)s;
        }
        for (int s = n; s < a.k; ++s) tb.tok_order[t][s] = -1;
    }
    __syncwarp();
}

// The same table for one token (the decode case), in registers and shuffles:
// lane j < k holds pick j; its segment is its rank among the valid picks by
// expert id, and every segment serves the one token.
__device__ __forceinline__ void moe_build_table_t1(MoeTable &tb, const MoeArgs &a, int lane) {
    const bool in = lane < a.k;
    const int e = in ? __ldcg(a.idx + lane) : -1;
    const float wv = in ? __ldcg(a.w + lane) : 0.f;
    bool ok = in && e >= 0 && e < a.E;
    // a repeated pick: valid only at its first slot
    const unsigned same = __match_any_sync(0xffffffffu, ok ? e : (1 << 20) + lane);
    if (ok && (same & ((1u << lane) - 1u))) ok = false;
    if (in && !ok) record_error(kErrBadExpert);
    const unsigned valid = __ballot_sync(0xffffffffu, ok);
    int rank = 0;
    for (int j = 0; j < a.k; ++j) {
        const int ej = __shfl_sync(0xffffffffu, e, j);
        rank += ((valid >> j) & 1u) && ej < e;
    }
    if (ok) {
        tb.seg_w0[rank] = rank * moe_item_work(1);
        tb.seg_expert[rank] = e;
        tb.seg_cnt[rank] = 1;
        tb.seg_row0[rank] = rank;
        tb.pair_tok[rank] = 0;
        tb.pair_slot[rank] = (short)lane;
        tb.pair_w[rank] = wv;
        tb.tok_order[0][rank] = (signed char)lane;
    }
    const int n = __popc(valid);
    if (lane >= n && lane < a.k) tb.tok_order[0][lane] = -1;
    if (lane == 0) tb.seg_w0[n] = n * moe_item_work(1);
    if (lane == 0) tb.n_routed = n;
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Work lists and the tile cursor (walked identically by every role)
// ---------------------------------------------------------------------------
struct MoeRanges {
    int s0, s1;   // phase-1 shared items
    int r0, r1;   // phase-1 routed items, flattened segment-major (I/8 per segment)
    int q0, q1;   // phase-2 shared items, chunk-major (H/8 per chunk)
    int v0, v1;   // phase-2 routed items, flattened segment-major (H/8 per segment)
    bool table;   // r*, q*, v* are set
};

// The shared expert's items split evenly: known without idx.
__device__ __forceinline__ MoeRanges moe_ranges_shared(const MoeArgs &a) {
    MoeRanges rg{};
    const long long S1 = a.Is / kGroupRows, S2 = (long long)a.nsplit * (a.H / kGroupRows);
    rg.s0 = (int)(S1 * blockIdx.x / gridDim.x);
    rg.s1 = (int)(S1 * (blockIdx.x + 1) / gridDim.x);
    rg.q0 = (int)(S2 * blockIdx.x / gridDim.x);
    rg.q1 = (int)(S2 * (blockIdx.x + 1) / gridDim.x);
    rg.table = false;
    return rg;
}

// Each list is split over the CTAs (the shared ones evenly, the routed ones
// by work), and a CTA walks its slices in list order: shared gate/up (no idx
// needed), routed gate/up, shared down (its h completes first: every CTA
// starts with the shared gate/up items), routed down.
// First item of CTA c in a routed list of n items per segment, split by work:
// the first item starting at or after work position W * c / grid.  Monotone
// in c, 0 at c = 0 and the item count at c = grid.
__device__ __forceinline__ int moe_split_routed(const MoeTable &tb, int n, int c, int grid) {
    // 32-bit throughout: W <= 8192 items x 128 segments x 184 < 2^31, and
    // W * c / grid = (W / grid) * c + (W % grid) * c / grid exactly
    const int W = n * tb.seg_w0[tb.n_routed];
    const int P = (W / grid) * c + (W % grid) * c / grid;
    if (P >= W) return tb.n_routed * n;
    int lo = 0, hi = tb.n_routed - 1;  // the segment holding position P
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (n * tb.seg_w0[mid] <= P) lo = mid; else hi = mid - 1;
    }
    const int w = tb.seg_w0[lo + 1] - tb.seg_w0[lo];  // one item's work in segment lo
    const int in = (P - n * tb.seg_w0[lo] + w - 1) / w;
    return lo * n + (in < n ? in : n);
}

// The routed slices, computed once (by the table warp, lanes 0-3) into the
// table; every role then copies them.
__device__ __forceinline__ void moe_split_routed_all(MoeTable &tb, const MoeArgs &a, int lane) {
    const int c = blockIdx.x, G = gridDim.x;
    if (lane == 0) tb.r0 = moe_split_routed(tb, a.I / kGroupRows, c, G);
    if (lane == 1) tb.r1 = moe_split_routed(tb, a.I / kGroupRows, c + 1, G);
    if (lane == 2) tb.v0 = moe_split_routed(tb, a.H / kGroupRows, c, G);
    if (lane == 3) tb.v1 = moe_split_routed(tb, a.H / kGroupRows, c + 1, G);
    __syncwarp();
}
__device__ __forceinline__ void moe_ranges_routed(MoeRanges &rg, const MoeTable &tb, const MoeArgs &a) {
    rg.r0 = tb.r0;
    rg.r1 = tb.r1;
    rg.v0 = tb.v0;
    rg.v1 = tb.v1;
    rg.table = true;
}

struct MoeTile {
    int phase;   // 1 or 2
    int seg;     // routed segment, -1 for the shared expert
    int in_seg;  // first item within the segment
    int tga;     // items
    int cnt;     // tokens of the segment
    int nx;      // token bucket (compile-time token count of the compute)
    int cols;    // 16-byte columns of K (from column c0)
    int c0;      // first column: the shared down chunk's, else 0
    int split;   // shared down chunk
    int ks_n;    // stages
};

struct MoeCursor {
    int kind;  // 0: phase-1 shared, 1: phase-1 routed, 2: phase-2 shared, 3: phase-2 routed, 4: done
    int u;
};

// Next tile of this CTA.  Without the table it stops (false) at the end of
// the shared phase-1 list; call again once rg.table is set.
__device__ __forceinline__ bool moe_next(MoeCursor &cur, const MoeRanges &rg, const MoeTable &tb,
                                         const MoeArgs &a, MoeTile &t) {
    if (cur.kind == 0) {
        if (cur.u < rg.s1) {
            t.phase = 1;
            t.seg = -1;
            t.in_seg = cur.u;
            t.cnt = a.T;
            t.nx = moe_nx(a.T);
            t.tga = min(moe_tg(1, t.nx), rg.s1 - cur.u);
            t.cols = a.H / 16;
            goto found;
        }
        if (!rg.table) return false;
        cur.kind = 1;
        cur.u = rg.r0;
    }
    if (cur.kind == 1) {
        if (cur.u < rg.r1) {
            const int ipg = a.I / kGroupRows;
            t.phase = 1;
            t.seg = cur.u / ipg;
            t.in_seg = cur.u - t.seg * ipg;
            t.cnt = tb.seg_cnt[t.seg];
            t.nx = moe_nx(t.cnt);
            t.tga = min(min(moe_tg(1, t.nx), rg.r1 - cur.u), ipg - t.in_seg);
            t.cols = a.H / 16;
            goto found;
        }
        cur.kind = 2;
        cur.u = rg.q0;
    }
    if (cur.kind == 2) {
        if (cur.u < rg.q1) {
            const int opg = a.H / kGroupRows;
            t.phase = 2;
            t.seg = -1;
            t.split = cur.u / opg;
            t.in_seg = cur.u - t.split * opg;
            t.cnt = a.T;
            t.nx = moe_nx(a.T);
            t.tga = min(min(moe_tg(2, t.nx), rg.q1 - cur.u), opg - t.in_seg);
            t.c0 = t.split * a.cc;
            t.cols = min(a.cc, a.Is / 16 - t.c0);
            goto found;
        }
        cur.kind = 3;
        cur.u = rg.v0;
    }
    if (cur.kind == 3) {
        if (cur.u < rg.v1) {
            const int opg = a.H / kGroupRows;
            t.phase = 2;
            t.seg = cur.u / opg;
            t.in_seg = cur.u - t.seg * opg;
            t.cnt = tb.seg_cnt[t.seg];
            t.nx = moe_nx(t.cnt);
            t.tga = min(min(moe_tg(2, t.nx), rg.v1 - cur.u), opg - t.in_seg);
            t.cols = a.I / 16;
            goto found;
        }
        cur.kind = 4;
    }
    return false;
found:
    if (t.phase == 1 || t.seg >= 0) t.c0 = t.split = 0;
    cur.u += t.tga;
    t.ks_n = (t.cols + kMoeCS - 1) / kMoeCS;
    return true;
}

// ---------------------------------------------------------------------------
// Consumers: the stages of one tile
// ---------------------------------------------------------------------------
// Lane (r, j) of warp (quad, hf) accumulates, for its column of each stage,
// NP = (TG / (CW / 8)) * halves pieces (its share of the items; a tile with fewer
// items repeats its last one, whose sums are never stored) times NX tokens
// (token entries past cnt repeat token cnt - 1, never stored).  Up to two
// tokens' activations stay in registers for all pieces; more tokens go four
// at a time, each piece dequantised once per four tokens.
// Position in the stage ring: the stage count `it`, its slot and the phase
// parity, carried along (a division by the runtime slot count per stage
// costs tens of instructions).
struct MoeRing {
    int it = 0, slot = 0, phase = 0;
    __device__ __forceinline__ void next(int stages) {
        ++it;
        if (++slot == stages) {
            slot = 0;
            phase ^= 1;
        }
    }
};

template <int PH, int NX, int CW, bool FULL>
__device__ __forceinline__ void moe_consume(const uint8_t *smem, const MoeArgs &a, uint32_t full0,
                                            uint32_t empty0, volatile int *abort_flag, MoeRing &it,
                                            const MoeTile &t, int quad, int hf, int lane,
                                            float (&acc)[(moe_tg(PH, NX) / (CW / 8)) * moe_halves(PH)][NX]) {
    constexpr int HH = moe_halves(PH), TG = moe_tg(PH, NX), TGH = TG / (CW / 8), NP = TGH * HH;
    constexpr uint32_t XOFF = moe_x_off(PH, NX);
    const int r = lane & 7, j = lane >> 3, col = 4 * quad + j;
    // piece p: item g(p) = (p / HH) * (CW / 8) + hf (the two warp halves take
    // alternate items), half p % HH.  A partial tile (FULL = false) skips the
    // pieces of items past its end: its stages cost in proportion to its
    // items, spread over both halves.
    const int gl = t.tga - 1;
    const bool any = FULL || hf < t.tga;  // this warp has items in the tile
    const uint32_t q_lane = col * kColBytes + r * 16;
    const uint32_t d_lane = (uint32_t)HH * TG * kMoeQBox + (col >> 1) * 16 + r * 2;
#define Q8_MOE_G(p) ((p) / HH * (CW / 8) + hf)
#define Q8_MOE_B(p) ((p) % HH * TG + min(Q8_MOE_G(p), gl))
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
        for (int n = 0; n < NX; ++n) acc[p][n] = 0.f;
    for (int ks = 0; ks < t.ks_n; ++ks, it.next(a.stages)) {
        const int slot = it.slot;
        if (mbar_wait_warp(full0 + 8 * slot, it.phase, abort_flag)) {
            const uint8_t *st = smem + (size_t)slot * a.slot_bytes;
            const int cols = min(kMoeCS, t.cols - ks * kMoeCS);
            if (col < cols && any) {
                if (NX <= 2) {
                    ulonglong2 xr[NX][4];
#pragma unroll
                    for (int n = 0; n < NX; ++n) {
                        const int nn = n < t.cnt ? n : t.cnt - 1;
                        const ulonglong2 *xv = reinterpret_cast<const ulonglong2 *>(st + XOFF + nn * kMoeXRow + col * 64);
                        xr[n][0] = xv[0];
                        xr[n][1] = xv[1];
                        xr[n][2] = xv[2];
                        xr[n][3] = xv[3];
                    }
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        if (!FULL && Q8_MOE_G(p) > gl) continue;
                        const int b = Q8_MOE_B(p);
                        const uint4 q = *reinterpret_cast<const uint4 *>(st + b * kMoeQBox + q_lane);
                        const float d = __half2float(*reinterpret_cast<const __half *>(st + b * kMoeDBox + d_lane));
                        uint64_t w[8];
                        dequant16_x2(q, w);
#pragma unroll
                        for (int n = 0; n < NX; ++n)
                            acc[p][n] = fmaf(dot16_x2(w, xr[n][0], xr[n][1], xr[n][2], xr[n][3]), d, acc[p][n]);
                    }
                } else {
                    // tokens four at a time: their activations in registers,
                    // each piece dequantised once per four tokens
#pragma unroll
                    for (int n0 = 0; n0 < NX; n0 += 4) {
                        ulonglong2 xr[4][4];
#pragma unroll
                        for (int n = 0; n < 4; ++n) {
                            const int nn = n0 + n < t.cnt ? n0 + n : t.cnt - 1;
                            const ulonglong2 *xv = reinterpret_cast<const ulonglong2 *>(st + XOFF + nn * kMoeXRow + col * 64);
                            xr[n][0] = xv[0];
                            xr[n][1] = xv[1];
                            xr[n][2] = xv[2];
                            xr[n][3] = xv[3];
                        }
#pragma unroll
                        for (int p = 0; p < NP; ++p) {
                            if (!FULL && Q8_MOE_G(p) > gl) continue;
                            const int b = Q8_MOE_B(p);
                            const uint4 q = *reinterpret_cast<const uint4 *>(st + b * kMoeQBox + q_lane);
                            const float d = __half2float(*reinterpret_cast<const __half *>(st + b * kMoeDBox + d_lane));
                            uint64_t w[8];
                            dequant16_x2(q, w);
#pragma unroll
                            for (int n = 0; n < 4; ++n)
                                acc[p][n0 + n] =
                                    fmaf(dot16_x2(w, xr[n][0], xr[n][1], xr[n][2], xr[n][3]), d, acc[p][n0 + n]);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * slot);
    }
#undef Q8_MOE_B
#undef Q8_MOE_G
    // lanes r, r+8, r+16, r+24 hold partial sums of the same row
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
        for (int n = 0; n < NX; ++n) {
            acc[p][n] += __shfl_xor_sync(0xffffffffu, acc[p][n], 8);
            acc[p][n] += __shfl_xor_sync(0xffffffffu, acc[p][n], 16);
        }
}

// One tile for a consumer warp: the stages, then its sums into red buffer
// tl % kMoeRedBufs (slot (item * halves + half) * NX + token of its column
// quad).
template <int PH, int NX, int CW>
__device__ __forceinline__ void moe_consume_tile(const uint8_t *smem, const MoeArgs &a, uint32_t full0,
                                                 uint32_t empty0, uint32_t redfull0, uint32_t redfree0,
                                                 float *red, volatile int *abort_flag, MoeRing &it, int tl,
                                                 const MoeTile &t, int quad, int hf, int lane) {
    constexpr int HH = moe_halves(PH), TGH = moe_tg(PH, NX) / (CW / 8), NP = TGH * HH;
    float acc[NP][NX];
    if (t.tga == moe_tg(PH, NX))
        moe_consume<PH, NX, CW, true>(smem, a, full0, empty0, abort_flag, it, t, quad, hf, lane, acc);
    else
        moe_consume<PH, NX, CW, false>(smem, a, full0, empty0, abort_flag, it, t, quad, hf, lane, acc);
    const int pb = tl % kMoeRedBufs;
    if (tl >= kMoeRedBufs) mbar_wait_warp(redfree0 + 8 * pb, ((tl / kMoeRedBufs) - 1) & 1, abort_flag);
    if ((lane >> 3) == 0) {
        float *rq = red + (size_t)(pb * 8 + quad) * a.red_a * 8;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const int g = p / HH * (CW / 8) + hf, h = p % HH;
#pragma unroll
            for (int n = 0; n < NX; ++n) rq[(((g * HH + h) * NX + n) << 3) + (lane & 7)] = acc[p][n];
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(redfull0 + 8 * pb);
}

template <int PH, int NMAX, int CW>
__device__ __forceinline__ void moe_consume_any(const uint8_t *smem, const MoeArgs &a, uint32_t full0,
                                                uint32_t empty0, uint32_t redfull0, uint32_t redfree0,
                                                float *red, volatile int *abort_flag, MoeRing &it, int tl,
                                                const MoeTile &t, int quad, int hf, int lane) {
#define Q8_MOE_TILE(NXV)                                                                                  \
    moe_consume_tile<PH, (NXV < NMAX ? NXV : NMAX), CW>(smem, a, full0, empty0, redfull0, redfree0, red,     \
                                                     abort_flag, it, tl, t, quad, hf, lane)
    if (NMAX == 1 || t.nx == 1) Q8_MOE_TILE(1);
    else if (NMAX == 2 || t.nx == 2) Q8_MOE_TILE(2);
    else if (NMAX == 4 || t.nx == 4) Q8_MOE_TILE(4);
    else if (NMAX == 8 || t.nx == 8) Q8_MOE_TILE(8);
    else Q8_MOE_TILE(16);
#undef Q8_MOE_TILE
}

// ---------------------------------------------------------------------------
// Epilogue warp
// ---------------------------------------------------------------------------
// y for the output groups tb.last_o[0..n): every token's partials in
// ascending expert id, then the shared expert's chunks.  Run by the CTA whose
// phase-2 items completed the groups (after the acquire), by threads tid of
// nthr; the partials are read from L2, each output's loads in flight
// together.
__device__ __forceinline__ void moe_final_sum(const MoeTable &tb, const MoeArgs &a, int n, int tid, int nthr) {
    const int per = a.T * kGroupRows, total = n * per;
#pragma unroll 2
    for (int q = tid; q < total; q += nthr) {
        const int gi = q / per, qq = q - gi * per;
        const int o = tb.last_o[gi];
        const int t = qq >> 3, row = o * kGroupRows + (qq & 7);
        // every partial's load first (independent), then the fixed-order sum
        float v[kMoeMaxK], vs[kMoeMaxSplit];
        int sl[kMoeMaxK];
#pragma unroll
        for (int j = 0; j < kMoeMaxK; ++j) {
            sl[j] = j < a.k ? tb.tok_order[t][j] : -1;
            v[j] = sl[j] >= 0 ? __ldcg(a.part + (size_t)(t * a.k + sl[j]) * a.H + row) : 0.f;
        }
#pragma unroll
        for (int sp = 0; sp < kMoeMaxSplit; ++sp)
            vs[sp] = sp < a.nsplit ? __ldcg(a.part + (size_t)(a.T * a.k + sp * a.T + t) * a.H + row) : 0.f;
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < kMoeMaxK; ++j)
            if (sl[j] >= 0) s += v[j];
#pragma unroll
        for (int sp = 0; sp < kMoeMaxSplit; ++sp)
            if (sp < a.nsplit) s += vs[sp];
        a.y[(size_t)t * a.H + row] = s;
    }
}

// Count the phase-2 tiles pending in tb.pend_*: one fence for all of their
// stores, then one atomic per (tile, output group), 32 at a time.  The groups
// this CTA completed are appended to tb.last_o; their sums are taken by the
// whole CTA at its end (or here, by this warp, when `now`: the pending list
// filled up before the CTA's last tile).
__device__ __forceinline__ void moe_flush_phase2(MoeTable &tb, const MoeArgs &a, int &npend, int n_seg, int lane,
                                                 bool now) {
    if (npend == 0) return;
    __threadfence();
    __syncwarp();
    int total = 0;
    for (int e = 0; e < npend; ++e) total += tb.pend_n[e];
    int nlast = tb.n_last;
    for (int i0 = 0; i0 < total; i0 += 32) {
        // the (i0 + lane)-th (tile, group) pair
        int i = i0 + lane, e = 0;
        while (e < npend && i >= tb.pend_n[e]) i -= tb.pend_n[e++];
        bool last = false;
        int o = 0;
        if (e < npend) {
            o = tb.pend_o0[e] + i;
            last = atomicAdd(a.ctr + kCtrGroups + o, 1u) == (unsigned)(n_seg - 1);
        }
        const unsigned m = __ballot_sync(0xffffffffu, last);
        if (last) tb.last_o[nlast + __popc(m & ((1u << lane) - 1u))] = o;
        nlast += __popc(m);
    }
    npend = 0;
    if (now) {
        __syncwarp();
        if (nlast) {
            __threadfence();  // acquire: the other CTAs' partials
            moe_final_sum(tb, a, nlast, lane, 32);
            for (int i = lane; i < nlast; i += 32) a.ctr[kCtrGroups + tb.last_o[i]] = 0u;
        }
        nlast = 0;
    }
    if (lane == 0) tb.n_last = nlast;
    __syncwarp();
}

// Tile t's outputs; `next` (nullable) is the tile after it, so that a
// segment's phase-1 items are counted once, after its last tile here.
__device__ __forceinline__ void moe_epilogue(MoeTable &tb, const MoeArgs &a, const float *red,
                                             uint32_t redfull0, uint32_t redfree0, volatile int *abort_flag,
                                             int tl, const MoeTile &t, const MoeTile *next, unsigned &p1_items,
                                             int &npend, int n_seg, int lane) {
    const int pb = tl % kMoeRedBufs;
    const bool ok = mbar_wait_warp(redfull0 + 8 * pb, (tl / kMoeRedBufs) & 1, abort_flag);
    const int HH = t.phase == 1 ? 2 : 1;
    const bool shared = t.seg < 0;
    const int row0 = shared ? 0 : tb.seg_row0[t.seg];
    const int n_out = t.tga * kGroupRows * t.cnt;
    if (ok) {
        for (int o = lane; o < n_out; o += 32) {
            const int n = o % t.cnt, rr = (o / t.cnt) & 7, g = o / (t.cnt * kGroupRows);
            float v[2] = {0.f, 0.f};
            for (int h = 0; h < HH; ++h) {
                const int slot = (g * HH + h) * t.nx + n;
                float s = 0.f;
#pragma unroll
                for (int qd = 0; qd < 8; ++qd) s += red[((size_t)(pb * 8 + qd) * a.red_a + slot) * 8 + rr];
                v[h] = s;
            }
            const int row = (t.in_seg + g) * kGroupRows + rr;
            if (t.phase == 1) {
                const float hval = silu_mul(v[0], v[1]);
                if (shared) {
                    a.hsh[(size_t)n * a.Is + row] = hval;
                } else {
                    const int pr = row0 + n;
                    a.hbuf[(size_t)pr * a.I + row] = hval * tb.pair_w[pr];
                }
            } else {
                const int dst = shared ? a.T * a.k + t.split * a.T + n
                                       : tb.pair_tok[row0 + n] * a.k + tb.pair_slot[row0 + n];
                a.part[(size_t)dst * a.H + row] = v[0];
            }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(redfree0 + 8 * pb);
    if (!ok) return;
    if (t.phase == 1) {
        // publish the segment's items once its last tile here is stored:
        // every lane's stores (each lane's fence), then the counter
        p1_items += (unsigned)t.tga;
        if (next == nullptr || next->phase != 1 || next->seg != t.seg) {
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                fence_proxy_async_global();  // h is read back by TMA
                red_relaxed_gpu_add(a.ctr + (shared ? kCtrShared : kCtrRouted + t.seg), p1_items);
            }
            p1_items = 0;
        }
    } else {
        if (lane == 0) {
            tb.pend_o0[npend] = t.in_seg;
            tb.pend_n[npend] = t.tga;
        }
        __syncwarp();
        ++npend;
        if (next == nullptr || npend == kMoePend) moe_flush_phase2(tb, a, npend, n_seg, lane, next != nullptr);
    }
}

// ---------------------------------------------------------------------------
// Producers
// ---------------------------------------------------------------------------
// Weight maps: [phase 1 | 2][routed stack | shared][q | scales][box depth
// 1, 2, 4, 8 groups].  A tile's items are consecutive packed groups, so a
// stage of tga items takes one box per set bit of tga (and half) instead of
// one per item: an SM's TMA unit accepts about one instruction per 70 ns,
// which per-item boxes of 4 KB would make the stream's limit.
constexpr int kMoeDepths = 4;
struct MoeMaps {
    CUtensorMap w[2][2][2][kMoeDepths];
    CUtensorMap x1, x1s;              // x [T][H]: one token per box, all T tokens per box
    CUtensorMap h2r, h2s;             // routed h [T*k][I] (one pair row per box), shared h [T][Is] (T rows)
};

// Weight boxes of one tile's stages, by the whole warp: lane 0 waits for the
// slot and arms its barrier, then the lanes issue the boxes in parallel.
// Returns false (warp-uniform) when a wait failed.
__device__ __forceinline__ bool moe_issue_weights(uint8_t *smem, const MoeArgs &a, const MoeMaps &m,
                                                  const MoeTable &tb, uint32_t full0, uint32_t empty0,
                                                  volatile int *abort_flag, MoeRing &it, const MoeTile &t,
                                                  uint64_t pw, int lane) {
    const int HH = t.phase == 1 ? 2 : 1, TG = moe_tg(t.phase, t.nx);
    const bool shared = t.seg < 0;
    // packed group of the tile's first item, and the gate -> up distance
    int g0, up = 0;
    if (t.phase == 1) {
        const int gates = (shared ? a.Is : a.I) / kGroupRows;
        g0 = (shared ? 0 : tb.seg_expert[t.seg] * 2 * gates) + t.in_seg;
        up = gates;
    } else {
        g0 = (shared ? 0 : tb.seg_expert[t.seg] * (a.H / kGroupRows)) + t.in_seg;
    }
    const CUtensorMap(&maps)[2][kMoeDepths] = m.w[t.phase - 1][shared ? 1 : 0];
    const int bits = __popc(t.tga), per = bits * HH;  // boxes per half, per stage (q; scales alike)
    const uint32_t dbase = (uint32_t)HH * TG * kMoeQBox;
    for (int ks = 0; ks < t.ks_n; ++ks, it.next(a.stages)) {
        const int slot = it.slot;
        if (it.it >= a.stages && !mbar_wait_warp(empty0 + 8 * slot, it.phase ^ 1, abort_flag))
            return false;
        const uint32_t st = smem_u32(smem + (size_t)slot * a.slot_bytes);
        const uint32_t full = full0 + 8 * slot;
        if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)(HH * t.tga) * (kMoeQBox + kMoeDBox));
        __syncwarp();
        for (int i = lane; i < 2 * per; i += 32) {
            const bool dbox = i >= per;
            const int j = dbox ? i - per : i, h = j / bits, k = j - h * bits;
            // the k-th set bit of tga, from the largest: box depth and first item
            int d = 3, off = 0, n = 0;
            for (; d >= 0; --d)
                if ((t.tga >> d) & 1) {
                    if (n == k) break;
                    off += 1 << d;
                    ++n;
                }
            const int grp = g0 + off + h * up, b = h * TG + off;
            if (dbox)
                tma_load_3d(st + dbase + b * kMoeDBox, &maps[1][d], full, 0, (t.c0 >> 1) + ks * (kMoeCS / 2), grp, pw);
            else
                tma_load_3d(st + b * kMoeQBox, &maps[0][d], full, 0, t.c0 + ks * kMoeCS, grp, pw);
        }
    }
    return true;
}

// Activation boxes of one tile's stages (phase 2: after the segment's h is
// complete).  Returns false when a wait failed.
__device__ __forceinline__ bool moe_issue_acts(uint8_t *smem, const MoeArgs &a, const MoeMaps &m,
                                               const MoeTable &tb, uint32_t full0, uint32_t empty0,
                                               volatile int *abort_flag, MoeRing &it, const MoeTile &t,
                                               uint64_t px) {
    const bool shared = t.seg < 0;
    if (t.phase == 2) {
        const unsigned target = (unsigned)((shared ? a.Is : a.I) / kGroupRows);
        if (!wait_counter_geq(a.ctr + (shared ? kCtrShared : kCtrRouted + t.seg), target, abort_flag))
            return false;
        fence_proxy_async_global();
    }
    const uint32_t xoff = moe_x_off(t.phase, t.nx);
    const int row0 = shared ? 0 : tb.seg_row0[t.seg];
    for (int ks = 0; ks < t.ks_n; ++ks, it.next(a.stages)) {
        const int slot = it.slot;
        if (it.it >= a.stages && !mbar_wait(empty0 + 8 * slot, it.phase ^ 1, abort_flag)) return false;
        const uint32_t st = smem_u32(smem + (size_t)slot * a.slot_bytes) + xoff;
        const uint32_t full = full0 + 8 * slot;
        mbar_arrive_expect_tx(full, (uint32_t)t.cnt * kMoeXRow);
        if (shared) {
            tma_load_3d(st, t.phase == 1 ? &m.x1s : &m.h2s, full, 0, t.c0 + ks * kMoeCS, 0, px);
        } else {
            for (int n = 0; n < t.cnt; ++n) {
                const int row = t.phase == 1 ? (int)tb.pair_tok[row0 + n] : row0 + n;
                tma_load_3d(st + n * kMoeXRow, t.phase == 1 ? &m.x1 : &m.h2r, full, 0, ks * kMoeCS, row, px);
            }
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
// Shared memory: the ring (stages x slot_bytes), the mbarriers (kMoeBarBytes),
// the red buffers (kMoeRedBufs x 8 quads x red_a slots x 8 rows), the table,
// and three flags.  NMAX: the largest token bucket (T rounded up to a power of 2).
template <int NMAX>
__global__ void __launch_bounds__(moe_threads(NMAX), 1)
    moe_fused_kernel(const __grid_constant__ MoeMaps maps, const MoeArgs a) {
    constexpr int CW = moe_cw(NMAX);
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *tail = smem + (size_t)a.stages * a.slot_bytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(tail);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kMoeMaxStages);
    const uint32_t redfull0 = smem_u32(bars + 2 * kMoeMaxStages), redfree0 = redfull0 + 8 * kMoeRedBufs;
    const uint32_t tbl_ready = redfree0 + 8 * kMoeRedBufs;
    float *red = reinterpret_cast<float *>(tail + kMoeBarBytes);
    MoeTable &tb = *reinterpret_cast<MoeTable *>(red + kMoeRedBufs * 8 * a.red_a * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(&tb + 1);
    volatile int *issued_w = abort_flag + 1;
    volatile int *issued_x = abort_flag + 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(full0 + 8 * s, 2);  // weight and activation producers
            mbar_init(empty0 + 8 * s, CW);
        }
        for (int p = 0; p < kMoeRedBufs; ++p) {
            mbar_init(redfull0 + 8 * p, CW);
            mbar_init(redfree0 + 8 * p, 1);
        }
        mbar_init(tbl_ready, 1);
        *abort_flag = 0;
        *issued_w = 0;
        *issued_x = 0;
        fence_mbar_init();
    }
    __syncthreads();

    MoeRanges rg = moe_ranges_shared(a);
    MoeCursor cur{0, rg.s0};
    MoeTile t;
    if (warp == CW) {
        // ------------------------- weight producer -------------------------
        {
            const uint64_t pw = policy_evict_first();
            MoeRing it;
            bool ok = true;
            // the shared expert's gate|up boxes need nothing from earlier kernels
            while (ok && moe_next(cur, rg, tb, a, t))
                ok = moe_issue_weights(smem, a, maps, tb, full0, empty0, abort_flag, it, t, pw, lane);
            pdl_wait_and_trigger();
            if (ok && mbar_wait_warp(tbl_ready, 0, abort_flag)) {
                moe_ranges_routed(rg, tb, a);
                while (ok && moe_next(cur, rg, tb, a, t))
                    ok = moe_issue_weights(smem, a, maps, tb, full0, empty0, abort_flag, it, t, pw, lane);
            }
            if (lane == 0) *issued_w = it.it;
        }
    } else if (warp == CW + 1) {
        // ----------------------- activation producer -----------------------
        pdl_wait_and_trigger();  // x comes from the previous kernel
        if (lane == 0) {
            const uint64_t px = policy_evict_last();
            MoeRing it;
            bool ok = true;
            while (ok && moe_next(cur, rg, tb, a, t)) ok = moe_issue_acts(smem, a, maps, tb, full0, empty0, abort_flag, it, t, px);
            if (ok && mbar_wait(tbl_ready, 0, abort_flag)) {
                moe_ranges_routed(rg, tb, a);
                while (ok && moe_next(cur, rg, tb, a, t))
                    ok = moe_issue_acts(smem, a, maps, tb, full0, empty0, abort_flag, it, t, px);
            }
            *issued_x = it.it;
        }
    } else if (warp == CW + 2) {
        // ------------------------ table + epilogues ------------------------
        pdl_wait_and_trigger();  // idx and w come from the router
        if (lane == 0) tb.n_last = 0;
        if (a.T == 1)
            moe_build_table_t1(tb, a, lane);
        else
            moe_build_table(tb, a, lane);
        moe_split_routed_all(tb, a, lane);
        if (lane == 0) mbar_arrive(tbl_ready);
        moe_ranges_routed(rg, tb, a);
        const int n_seg = tb.n_routed + a.nsplit;  // phase-2 contributions per output group
        if (n_seg == 0) {
            // no valid pick and no shared expert: y is zero (slice per CTA)
            const long long n = (long long)a.T * a.H;
            for (long long i = n * blockIdx.x / gridDim.x + lane; i < n * (blockIdx.x + 1) / gridDim.x; i += 32)
                a.y[i] = 0.f;
        }
        int tl = 0, npend = 0;
        unsigned p1_items = 0;
        bool has = moe_next(cur, rg, tb, a, t);
        while (has) {
            MoeTile nt;
            const bool hn = moe_next(cur, rg, tb, a, nt);
            moe_epilogue(tb, a, red, redfull0, redfree0, abort_flag, tl++, t, hn ? &nt : nullptr, p1_items, npend,
                         n_seg, lane);
            t = nt;
            has = hn;
        }
    } else {
        // ----------------------------- consumers ----------------------------
        const int quad = warp & 7, hf = warp >> 3;
        pdl_wait_and_trigger();
        MoeRing it;
        int tl = 0;
        for (;;) {
            if (!moe_next(cur, rg, tb, a, t)) {
                if (rg.table || !mbar_wait_warp(tbl_ready, 0, abort_flag)) break;
                moe_ranges_routed(rg, tb, a);
                continue;
            }
            if (t.phase == 1)
                moe_consume_any<1, NMAX, CW>(smem, a, full0, empty0, redfull0, redfree0, red, abort_flag, it, tl++, t, quad, hf, lane);
            else
                moe_consume_any<2, NMAX, CW>(smem, a, full0, empty0, redfull0, redfree0, red, abort_flag, it, tl++, t, quad, hf, lane);
        }
    }
    __syncthreads();
    if (!*abort_flag && tb.n_last > 0) {
        // the sums of the output groups this CTA completed, by all threads
        __threadfence();  // acquire: the other CTAs' partials
        moe_final_sum(tb, a, tb.n_last, threadIdx.x, blockDim.x);
        for (int i = threadIdx.x; i < tb.n_last; i += blockDim.x) a.ctr[kCtrGroups + tb.last_o[i]] = 0u;
    }
    if (threadIdx.x == 0) {
        if (*abort_flag) {
            // complete the stages one producer armed and the other did not,
            // then wait (bounded) for every copy still in flight
            const int iw = *issued_w, ix = *issued_x, hi = iw > ix ? iw : ix;
            const int lo = hi > a.stages ? hi - a.stages : 0;
            for (int it = lo; it < hi; ++it) {
                if (it >= iw) mbar_arrive(full0 + 8 * (it % a.stages));
                if (it >= ix) mbar_arrive(full0 + 8 * (it % a.stages));
            }
            for (int it = lo; it < hi; ++it) mbar_drain(full0 + 8 * (it % a.stages), (it / a.stages) & 1);
        } else {
            // the last CTA to finish clears the segment counters
            __threadfence();
            if (atom_acq_rel_gpu_add(a.ctr + kCtrCta, 1u) == gridDim.x - 1) {
                a.ctr[kCtrShared] = 0u;
                for (int s = 0; s < tb.n_routed; ++s) a.ctr[kCtrRouted + s] = 0u;
                __threadfence();
                a.ctr[kCtrCta] = 0u;
            }
        }
    }
}

// Zeroes n words of a counter area ahead of a kernel that needs them at zero,
// as a kernel of the dependent-launch chain: the next kernel may start (and
// prefetch) at once, and its own dependency wait covers this kernel's stores,
// which come after this kernel's wait for the grid before it (the previous
// user of the area).
__global__ void clear_words_kernel(unsigned *p, int n) {
    pdl_launch_dependents();
    pdl_wait();
    for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = 0u;
}

}  // namespace q8
