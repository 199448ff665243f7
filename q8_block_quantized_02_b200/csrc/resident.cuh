// resident.cuh -- S2/S4 at N = 1 for small matrices (the projections of a
// small model's decode step): each CTA holds its whole share of the weights
// in shared memory.  In a decode step these products run back to back, each
// waiting for the one before, so what matters is the time from the release
// of that dependency to the kernel's last store; at these sizes that time is
// mostly fixed costs per launch (the dependency release, the first L2 read of
// x, one barrier), and the kernel keeps its code straight-line: loops with a
// runtime trip count cost a branch resolution per iteration that few warps
// cannot hide.
#pragma once

#include "tile_gemm.cuh"

namespace q8 {

// ---------------------------------------------------------------------------
// Resident kernel (small matrices, N <= 4)
// ---------------------------------------------------------------------------
// For matrices whose row groups spread to at most 8 per CTA, with all of a
// CTA's weights fitting in shared memory (the decode projections of small
// models).  Every weight box of the CTA is issued at kernel start, before
// griddepcontrol.wait, so the weights stream in while the previous kernel on
// the stream still runs.  After the wait the activations are copied with
// plain 16-byte loads (one L2 round trip), the CTA computes all of its rows
// from shared memory in one pass with the column-owner lane mapping above,
// and the eight warps' partial sums meet in shared memory behind a single
// barrier, added in warp order.  There is no ring, no per-stage barrier and
// no reducer warp: a dependent decode step pays for none of them.
constexpr int kResTGM = 8;   // row groups per CTA at most

// Warps of a CTA.  (16 warps for the multi-group and SwiGLU cases measured
// slower in a decode chain: 512 threads of 84 registers leave too little of
// the SM to the neighbouring kernels of the chain.)
template <int MODE, int TGM>
__host__ __device__ constexpr int res_warps() {
    return 8;
}

constexpr int kResColsPerThread = 2;  // one-group path: C <= 512 columns
constexpr int kResOneThreads = 256;   // one-group path: threads

template <int NMAX, int MODE, int TGM>
__host__ __device__ constexpr int res_red_floats() {
    // column-owner partials, or the one-group path's [row][thread] partials
    return res_warps<MODE, TGM>() * TGM * (MODE == kModeSwiGLU ? 2 : 1) * NMAX * 8 > 8 * 32 * res_warps<MODE, TGM>()
               ? res_warps<MODE, TGM>() * TGM * (MODE == kModeSwiGLU ? 2 : 1) * NMAX * 8
               : 8 * 32 * res_warps<MODE, TGM>();
}

// One row group, fp32 activations, N = 1: thread t owns the 16-byte columns
// t and t + 256 of the group.  It loads their activations straight from
// memory, reads each column's 8 x 16 B core matrix a row at a time starting at
// row t % 8 (the eight lanes of a quarter-warp then read eight different
// 16-byte bank groups), and keeps one partial sum per row, in that rotated
// order.  Partials meet in shared memory as [row][thread]; warp r adds row
// r's in thread order and then across its lanes by a fixed shuffle tree.
// With a single row group per CTA the column-owner mapping would have eight
// lanes read every activation; here each is read once.  (With several
// groups or the SwiGLU pair the column-owner mapping reuses the activations
// across groups and stays faster.)
__device__ __forceinline__ void res_one_group(const uint8_t *smem, const TileArgs &a,
                                              const float *__restrict__ x, int unit, uint32_t wbar,
                                              volatile int *abort_flag, float *red) {
    const int t = threadIdx.x, rot = t & 7, lane = t & 31, warp = t >> 5;
    ulonglong2 xa[kResColsPerThread][4];
#pragma unroll
    for (int k = 0; k < kResColsPerThread; ++k) {
        const int c = t + k * kResOneThreads;
        if (c < a.C) {
            const ulonglong2 *xg = reinterpret_cast<const ulonglong2 *>(x + (size_t)c * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) xa[k][i] = __ldg(xg + i);
        }
    }
    const bool ok = mbar_wait_warp(wbar, 0, abort_flag);
    float accr[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) accr[i] = 0.f;
    if (ok) {
#pragma unroll
        for (int k = 0; k < kResColsPerThread; ++k) {
            const int c = t + k * kResOneThreads;
            if (c < a.C) {
                const uint8_t *qc = smem + c * kColBytes;
                const uint8_t *dc = smem + a.d_off + (c >> 1) * 16;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = (i + rot) & 7;
                    const uint4 qv = *reinterpret_cast<const uint4 *>(qc + r * 16);
                    const float d = __half2float(*reinterpret_cast<const __half *>(dc + r * 2));
                    uint64_t w[8];
                    dequant16_x2(qv, w);
                    accr[i] = fmaf(dot16_x2(w, xa[k][0], xa[k][1], xa[k][2], xa[k][3]), d, accr[i]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[((i + rot) & 7) * kResOneThreads + t] = accr[i];
    __syncthreads();
    if (ok && warp < 8) {
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < kResOneThreads / 32; ++i) sum += red[warp * kResOneThreads + lane + 32 * i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            const int row = unit * kGroupRows + warp;
            if (row < a.M_out) a.y[row] = a.res ? __fadd_rn(sum, a.res[row]) : sum;
        }
    }
}

// One column of the CTA's TGM row groups for lane (r, j), with no per-group
// branch so that the groups' independent chains (shared loads,
// dequantisation, dot products) overlap.  A CTA holding fewer groups (tga <
// TGM) reads its last group again in place of each missing one; those sums
// are never stored.
template <int NMAX, int MODE, int TGM>
__device__ __forceinline__ void res_step(const uint8_t *st, const TileArgs &a, int col, int r, int tga,
                                         float (&acc)[TGM][MODE == kModeSwiGLU ? 2 : 1][NMAX]) {
    constexpr int H = MODE == kModeSwiGLU ? 2 : 1;
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
        const int gu = g < tga ? g : tga - 1;
#pragma unroll
        for (int h = 0; h < H; ++h) {
            ColPiece pc;
            load_piece(st, a, h ? a.q_half : 0u, h ? a.d_half : 0u, gu, col, r, pc);
#pragma unroll
            for (int n = 0; n < NMAX; ++n)
                if (n < a.N)
                    acc[g][h][n] = fmaf(dot16_x2(pc.w, xr[n][0], xr[n][1], xr[n][2], xr[n][3]), pc.d, acc[g][h][n]);
        }
    }
}

// TGM: the plan's row groups per CTA (1..kResTGM).
template <int NMAX, int MODE, int TGM>
__global__ void __launch_bounds__(res_warps<MODE, TGM>() * 32, 1)
    resident_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap td,
                    const __grid_constant__ CUtensorMap tq1, const __grid_constant__ CUtensorMap td1,
                    const float *__restrict__ x, const TileArgs a) {
    constexpr int H = MODE == kModeSwiGLU ? 2 : 1;
    constexpr int kResWarps = res_warps<MODE, TGM>();
    constexpr int kResThreads = kResWarps * 32;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *red = reinterpret_cast<float *>(smem + a.stage_bytes);
    uint64_t *bar = reinterpret_cast<uint64_t *>(red + res_red_floats<NMAX, MODE, TGM>());
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar + 1);
    const uint32_t wbar = smem_u32(bar);
    // units * grid < 2^31 is checked on the host, so 32-bit math is exact here
    const int u0 = (int)(((unsigned)a.units * blockIdx.x) / gridDim.x);
    const int u1 = (int)(((unsigned)a.units * (blockIdx.x + 1)) / gridDim.x);
    const int tga = u1 - u0;  // 1..TGM (planned on the host)
    if (threadIdx.x == 0) {
        mbar_init(wbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t pw = policy_evict_first();
        const uint32_t st = smem_u32(smem);
        mbar_arrive_expect_tx(wbar, (uint32_t)(H * tga) * (a.q_box + a.d_box));
        if (a.nchunks == 1) {
            // one box per half covers all of the CTA's row groups (a map of that
            // depth): 2 or 4 TMA instructions, so thread 0 reaches its
            // dependency wait early (an SM's TMA unit takes tens of ns per
            // instruction)
            const CUtensorMap *mq = tga == TGM ? &tq : &tq1;
            const CUtensorMap *md = tga == TGM ? &td : &td1;
            for (int h = 0; h < H; ++h) {
                const int grp = u0 + (h ? a.up_group0 : 0);
                tma_load_3d(st + h * a.q_half, mq, wbar, 0, 0, grp, pw);
                tma_load_3d(st + a.d_off + h * a.d_half, md, wbar, 0, 0, grp, pw);
            }
        } else {
            // rows longer than one box: a box per group and chunk (depth-1 maps)
            for (int h = 0; h < H; ++h)
                for (int g = 0; g < tga; ++g) {
                    const int grp = u0 + g + (h ? a.up_group0 : 0);
                    for (int c = 0; c < a.nchunks; ++c) {
                        tma_load_3d(st + h * a.q_half + g * a.q_box + c * a.CB * kColBytes, &tq, wbar, 0,
                                    c * a.CB, grp, pw);
                        tma_load_3d(st + a.d_off + h * a.d_half + g * a.d_slot + c * a.CB * 8, &td, wbar, 0,
                                    c * a.CB / 2, grp, pw);
                    }
                }
        }
    }
    // the activations, and the outputs, belong to the previous grid until here;
    // only now may the next kernel on the stream start and prefetch
    pdl_wait_and_trigger();
    if (MODE == kModeF32 && NMAX == 1 && TGM == 1 && a.C <= kResColsPerThread * kResThreads) {
        res_one_group(smem, a, x, u0, wbar, abort_flag, red);
        if (threadIdx.x == 0 && *abort_flag) mbar_drain(wbar, 0);
        return;
    }
    {
        // activations -> shared memory as [n][column][16 floats]; every load of a
        // thread is issued before its first store, so the copy costs one round trip
        constexpr int XB = 8;
        const int k4 = a.C * 4;  // float4 per activation row
        const int total = a.N * k4;
        float4 *xs = reinterpret_cast<float4 *>(smem + a.x_off);
        const float4 *xg = reinterpret_cast<const float4 *>(x);
        for (int base = threadIdx.x; base < total; base += XB * kResThreads) {
            float4 v[XB];
#pragma unroll
            for (int u = 0; u < XB; ++u) {
                const int i = base + u * kResThreads;
                if (i < total) v[u] = __ldg(xg + i);
            }
#pragma unroll
            for (int u = 0; u < XB; ++u) {
                const int i = base + u * kResThreads;
                if (i < total) {
                    const int n = i / k4;
                    xs[n * a.CS * 4 + (i - n * k4)] = v[u];
                }
            }
        }
    }
    __syncthreads();
    const bool ok = mbar_wait_warp(wbar, 0, abort_flag);
    const int r = lane & 7, j = lane >> 3;
    float acc[TGM][H][NMAX];
#pragma unroll
    for (int g = 0; g < TGM; ++g)
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
            for (int n = 0; n < NMAX; ++n) acc[g][h][n] = 0.f;
    if (ok) {
        const int nq = (a.C + 3) >> 2;
        for (int cq = warp; cq < nq; cq += kResWarps) {
            const int col = 4 * cq + j;
            if (col < a.C) res_step<NMAX, MODE, TGM>(smem, a, col, r, tga, acc);
        }
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
    if (j == 0) {
#pragma unroll
        for (int g = 0; g < TGM; ++g)
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
                for (int n = 0; n < NMAX; ++n)
                    red[((((warp * TGM + g) * H + h) * NMAX + n) << 3) + r] = acc[g][h][n];
    }
    __syncthreads();
    if (ok) {
        for (int o = threadIdx.x; o < tga * 8; o += kResThreads) {
            const int g = o >> 3, rr = o & 7;
            float v[H][NMAX];
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
                for (int n = 0; n < NMAX; ++n) {
                    float sum = 0.f;
#pragma unroll
                    for (int w = 0; w < kResWarps; ++w)
                        sum += red[((((w * TGM + g) * H + h) * NMAX + n) << 3) + rr];
                    v[h][n] = sum;
                }
            store_unit<NMAX, MODE>(a, u0 + g, rr, v[0], v[H - 1]);
        }
    } else if (threadIdx.x == 0) {
        mbar_drain(wbar, 0);  // no weight copy may still land after the CTA exits
    }
}


}  // namespace q8
