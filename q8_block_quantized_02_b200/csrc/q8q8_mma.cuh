// q8q8_mma.cuh -- S8 on the tensor cores: Q8_0 weights times Q8_0 activations
// for 5..16 activation columns, where the product is a dense integer
// contraction worth a tcgen05.mma (kind::i8).
//
// A Q8_0 block dot needs its own pair of scales, so the tensor cores take one
// 32-deep block at a time: D[m][n] = sum_i A[m][i] * xq[n][i] over one block,
// exact in int32, and the epilogue adds float(dot) * d_w[m] * d_x[n] into fp32
// registers.  (The block-dot-then-scale order is the integer path of "Add
// Qwen1.5-MoE Q8_0 ... - #144", "Key implementation notes": each activation
// block quantised to int8, then int8 x int8 accumulation with the Q8_0
// scales; the weights are the raw GGUF Q8_0 blocks of the
// "skuznetsov/cogni-ml" README's Q8_0 GEMV probe, "Build Qwen CLIs".)
//
// Operands straight from the packed layout (include/q8.h):
//   * A = weights, M = 128 rows (16 packed groups) x K = 32 bytes.  A group's
//     16-byte column is an 8 x 16 B core matrix, so the q bytes of a tile load
//     with one TMA box into [group][column][8 rows x 16 B] and feed the MMA as
//     a K-major, no-swizzle operand: the two core matrices of a block are
//     128 B apart (leading offset), groups CS * 128 B apart (stride offset).
//     Stored bytes are q + 128, so A is read as unsigned 8-bit;
//   * B = activations, N = 16 rows (zero padded past N) x 32 bytes, loaded
//     as [column][row][16 B] (core matrices of 8 rows), read as signed 8-bit;
//   * D = 128 lanes x 16 int32 columns of tensor memory per block.  A half
//     stage (4 blocks, 64 columns) fills the next slot of a ring of 8 such
//     slots (all 512 columns), so the MMAs run up to two stages ahead of the
//     epilogue and their latency stays off its path; each epilogue warp
//     loads its columns of a half before one wait, paying the load latency
//     once per 4 blocks.
// Because A holds q + 128, the tensor cores return dot + 128 * sum_i xq[n][i];
// the epilogue removes that term exactly.  Its int -> float conversion adds
// the correction to 0x4B400000 (the bits of 1.5 * 2^23) and subtracts
// 1.5 * 2^23 as a float, exact for |dot| < 2^22 (here |dot| <= 32 * 127 * 128).
//
// Work split: output rows in tiles of 128; a cluster of `split` CTAs shares a
// contiguous tile range and splits K into `split` contiguous block ranges
// (small M).  Partial sums meet in the cluster leader's registers, taken from
// the peers' shared memory in rank order, so results are bit-identical from
// run to run.  Warp 0 issues TMA (weight boxes of the first stages before
// griddepcontrol.wait), warp 1 owns tensor memory and issues the MMAs, warps
// 2..9 are the epilogue (warp w reads TMEM lanes 32 * (w % 4) ..; the two
// warps of a lane quarter split the 16 activation columns).
// Every wait is bounded; a stalled pipeline records an error, waits for its
// copies and MMAs in flight, frees its tensor memory and exits.
#pragma once

#include <type_traits>

#include "q8_device.cuh"

namespace q8 {

constexpr int kMmaTileGroups = 16;                 // 128 output rows per tile
constexpr int kMmaN = 16;                          // MMA N: activation columns (padded)
constexpr int kMmaCS = 32;                         // 16-byte columns per stage: 4 KB of each group
constexpr int kMmaSB = kMmaCS / 2;                 // blocks per stage
constexpr int kMmaHalfBlocks = 4;                  // blocks per TMEM half (one ld each)
constexpr int kMmaHalves = kMmaSB / kMmaHalfBlocks;   // TMEM halves per stage
constexpr int kMmaTSlots = 8;                         // TMEM ring of halves (two stages)
constexpr uint32_t kMmaSlotCols = kMmaHalfBlocks * kMmaN;      // 64 columns a half
constexpr uint32_t kMmaTmemCols = kMmaTSlots * kMmaSlotCols;  // 512 columns
constexpr int kMmaEpiGroups = 2;                   // epilogue warp groups, split over n
constexpr int kMmaNPG = kMmaN / kMmaEpiGroups;     // activation columns per group
constexpr int kMmaEpiThreads = kMmaEpiGroups * 128;
constexpr int kMmaThreads = 64 + kMmaEpiThreads;   // producer, MMA, epilogue
constexpr int kMmaMaxSplit = 8;

constexpr uint32_t kMmaQBytes = kMmaCS * kMmaTileGroups * kColBytes;  // 64 KB
constexpr uint32_t kMmaDBytes = kMmaSB * kMmaTileGroups * 16;         // 4 KB
constexpr uint32_t kMmaXBytes = kMmaCS * kMmaN * 16;                  // 8 KB
constexpr uint32_t kMmaTabBytes = kMmaSB * kMmaN * 8;                 // 2 KB
constexpr uint32_t kMmaDOff = kMmaQBytes;
constexpr uint32_t kMmaXOff = kMmaDOff + kMmaDBytes;
constexpr uint32_t kMmaTabOff = kMmaXOff + kMmaXBytes;
constexpr uint32_t kMmaStageBytes = kMmaTabOff + kMmaTabBytes;
constexpr uint32_t kMmaTxBytes = kMmaQBytes + kMmaDBytes + kMmaXBytes;
constexpr uint32_t kMmaRedBytes = kMmaN * 128 * 4;                    // one tile's partials

// Shared-memory carve-up (host and device): stages, barriers, partials, misc.
__host__ __device__ constexpr uint32_t mma_bar_off(int stages) { return stages * kMmaStageBytes; }
__host__ __device__ constexpr uint32_t mma_nbars(int stages) { return 2 * stages + 2 * kMmaTSlots + 3; }
__host__ __device__ constexpr uint32_t mma_red_off(int stages) {
    return (mma_bar_off(stages) + 8 * mma_nbars(stages) + 127) / 128 * 128;
}
__host__ __device__ constexpr uint32_t mma_misc_off(int stages, bool split) {
    return mma_red_off(stages) + (split ? kMmaRedBytes : 0);
}
__host__ __device__ constexpr uint32_t mma_smem_bytes(int stages, bool split) {
    return mma_misc_off(stages, split) + 16;
}

// Instruction descriptor: D s32, A unsigned 8-bit, B signed 8-bit, both
// K-major, N = 16, M = 128 (PTX ISA, tcgen05 instruction descriptor table).
constexpr uint32_t kMmaIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kMmaN >> 3) << 17) |
                               ((uint32_t)(128 >> 4) << 24);

struct MmaArgs {
    float *y;            // [N][M]
    const uint16_t *xd;  // activation scales [N][B], binary16
    int M, N, B;
    int tiles;           // ceil(groups / 16)
    int split;           // CTAs per cluster (K split)
    int stages;
};

// ---------------------------------------------------------------------------
// tcgen05 / cluster wrappers (PTX ISA for sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, no swizzle: start, leading and stride byte
// offsets in 16-byte units, descriptor version 1 (bits 46-47).
__device__ __forceinline__ uint64_t mma_smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
           ((uint64_t)(sbo >> 4) << 32) | (1ull << 46);
}

// D = A * B (the accumulator input is off: every block starts from zero).
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(0)
        : "memory");
}

// Arrive on a local mbarrier once every MMA this thread issued has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Column loads of 32 lanes without waiting: the registers are undefined until
// tmem_wait_ld8, which names them as operands so that no use of them is
// scheduled before the wait.
__device__ __forceinline__ void tmem_ld8_async(uint32_t taddr, uint32_t *v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                   "=r"(v[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld4_async(uint32_t taddr, uint32_t *v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld1_async(uint32_t taddr, uint32_t *v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v[0]) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_ld2_async(uint32_t taddr, uint32_t *v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                 : "=r"(v[0]), "=r"(v[1])
                 : "r"(taddr)
                 : "memory");
}
// Waits for every earlier tcgen05.ld of the thread; names 8 of the loaded
// registers so that no use of them is scheduled before it (called once per
// 8 registers: the later calls return at once).
__device__ __forceinline__ void tmem_wait_ld8(uint32_t *v) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]),
                   "+r"(v[7])
                 :
                 : "memory");
}


__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t o;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(o) : "r"(smem_addr), "r"(rank));
    return o;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// mbar_wait with cluster-scope acquire (arrivals come from peer CTAs).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    if (*abort) return false;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_acq_cluster(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                record_error(kErrWaitTimeout);
                *abort = 1;
                return false;
            }
        }
    }
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
// Every thread of every CTA of the cluster; all of them reach it (every wait
// before it is bounded).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                     "memory");
}

__device__ __forceinline__ int byte_sum_s8(uint4 w, int acc) {
    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(w.x), "r"(0x01010101));
    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(w.y), "r"(0x01010101));
    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(w.z), "r"(0x01010101));
    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(w.w), "r"(0x01010101));
    return acc;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kMmaThreads, 1)
    q8q8_mma_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap td,
                    const __grid_constant__ CUtensorMap tx, const MmaArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.split;
    const uint32_t full0 = smem_u32(smem + mma_bar_off(a.stages));
    const uint32_t empty0 = full0 + 8 * a.stages;
    const uint32_t tfull0 = empty0 + 8 * a.stages;
    const uint32_t tempty0 = tfull0 + 8 * kMmaTSlots;
    const uint32_t done_bar = tempty0 + 8 * kMmaTSlots;
    const uint32_t redfull = done_bar + 8, redfree = redfull + 8;
    float *red = reinterpret_cast<float *>(smem + mma_red_off(a.stages));
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + mma_misc_off(a.stages, S > 1));
    volatile uint32_t *tmem_slot = misc;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
    volatile int *issued = reinterpret_cast<volatile int *>(misc + 2);

    {
        // the launch must match the plan this kernel was given: uniform over
        // the grid, so every CTA leaves here together (no cluster barrier yet)
        uint32_t dyn, nct = 1;
        asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if (S > 1) asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(nct));
        if (dyn < mma_smem_bytes(a.stages, S > 1) || nct != (uint32_t)S || gridDim.x % S != 0) {
            if (threadIdx.x == 0) record_error(kErrLaunchConfig);
            return;
        }
    }
    const int rank = S > 1 ? (int)cluster_ctarank() : 0;
    const int ci = blockIdx.x / S, P = gridDim.x / S;
    const int t0 = (int)(((long long)a.tiles * ci) / P);
    const int t1 = (int)(((long long)a.tiles * (ci + 1)) / P);
    const int b_lo = (int)(((long long)a.B * rank) / S);
    const int b_hi = (int)(((long long)a.B * (rank + 1)) / S);
    const int nblk = b_hi - b_lo;
    const int ksteps = (nblk + kMmaSB - 1) / kMmaSB;
    int n_tiles = t1 - t0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1 + kMmaEpiThreads / 32);  // MMA commit + epilogue warps
        }
        for (int h = 0; h < kMmaTSlots; ++h) {
            mbar_init(tfull0 + 8 * h, 1);
            mbar_init(tempty0 + 8 * h, kMmaEpiThreads / 32);
        }
        mbar_init(done_bar, 1);
        mbar_init(redfull, S > 1 ? kMmaEpiThreads * (S - 1) : 1);
        mbar_init(redfree, kMmaEpiThreads);
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(misc), kMmaTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    if (S > 1) cluster_sync_all();  // peers' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if ((tmem >> 16) != 0 || (tmem & 0xFFFFu) + kMmaTmemCols > 512) {  // lane 0, columns in range
        if (threadIdx.x == 0) record_error(kErrLaunchConfig);
        n_tiles = 0;
    }
    const int total = n_tiles * ksteps;

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0 && total > 0) {
            const uint64_t pw = policy_evict_first(), px = policy_evict_last();
            // ring slot/phase and (tile, k step) are carried along: no
            // division by a runtime value per stage
            auto issue_w = [&](int slot, int tile, int ks) {
                const int b0 = b_lo + ks * kMmaSB;
                const uint32_t st = smem_u32(smem + (size_t)slot * kMmaStageBytes);
                const uint32_t full = full0 + 8 * slot;
                mbar_arrive_expect_tx(full, kMmaTxBytes);
                tma_load_3d(st, &tq, full, 0, 2 * b0, kMmaTileGroups * (t0 + tile), pw);
                tma_load_3d(st + kMmaDOff, &td, full, 0, b0, kMmaTileGroups * (t0 + tile), pw);
            };
            auto issue_x = [&](int slot, int ks) {
                const int b0 = b_lo + ks * kMmaSB;
                const uint32_t st = smem_u32(smem + (size_t)slot * kMmaStageBytes);
                tma_load_3d(st + kMmaXOff, &tx, full0 + 8 * slot, 0, 0, 2 * b0, px);
            };
            const int pro = total < a.stages ? total : a.stages;
            int it = 0, tile = 0, ks = 0;
            for (; it < pro; ++it) {  // weights never depend on the previous grid
                issue_w(it, tile, ks);
                if (++ks == ksteps) { ks = 0; ++tile; }
            }
            pdl_wait_and_trigger();  // activations may
            for (int k = 0, kx = 0; k < pro; ++k) {
                issue_x(k, kx);
                if (++kx == ksteps) kx = 0;
            }
            int slot = pro % a.stages, phase = pro / a.stages;  // ring position of iteration `pro`
            for (; it < total; ++it) {
                if (!mbar_wait(empty0 + 8 * slot, (phase & 1) ^ 1, abort_flag)) break;
                issue_w(slot, tile, ks);
                issue_x(slot, ks);
                if (++ks == ksteps) { ks = 0; ++tile; }
                if (++slot == a.stages) { slot = 0; ++phase; }
            }
            *issued = it;
        } else {
            pdl_wait_and_trigger();
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        pdl_wait_and_trigger();  // its inputs arrive after the producer's wait anyway
        if (lane == 0) {
            // Half h of each stage (blocks 4h .. 4h + 3) goes to the next slot
            // of a ring of kMmaTSlots TMEM slots of 64 columns (block jj of
            // the half at column 16 jj), handed to the epilogue by one commit;
            // the MMAs run up to four stages ahead of the epilogue's reads.
            bool ok = true;
            int ts = 0, tph = 0;  // TMEM slot and its phase, carried along
            int slot = 0, phase = 0, ks = 0;  // ring position and k step of iteration `it`
            for (int it = 0; it < total && ok;
                 ++it, ks = ks + 1 == ksteps ? 0 : ks + 1, slot = slot + 1 == a.stages ? 0 : slot + 1,
                     phase ^= slot == 0 ? 1 : 0) {
                if (!mbar_wait(full0 + 8 * slot, phase, abort_flag)) break;
                tc_fence_after();
                const int nb = min(kMmaSB, nblk - ks * kMmaSB);
                const uint32_t st = smem_u32(smem + (size_t)slot * kMmaStageBytes);
                for (int h = 0; h < kMmaHalves; ++h) {
                    // the epilogue has read this slot's previous half
                    if (!mbar_wait(tempty0 + 8 * ts, tph ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = h * kMmaHalfBlocks; j < (h + 1) * kMmaHalfBlocks && j < nb; ++j) {
                        // block j: columns 2j, 2j+1 (128 B apart); groups kMmaCS * 128 B apart
                        const uint64_t ad = mma_smem_desc(st + j * 2 * kColBytes, kColBytes, kMmaCS * kColBytes);
                        // activations [column][16 rows][16 B]: columns 256 B apart, 8-row halves 128 B
                        const uint64_t bd = mma_smem_desc(st + kMmaXOff + j * 2 * (kMmaN * 16), kMmaN * 16, 8 * 16);
                        mma_i8(tmem + ts * kMmaSlotCols + (j - h * kMmaHalfBlocks) * kMmaN, ad, bd, kMmaIdesc);
                    }
                    // past the end of K the half holds no new block: the commit
                    // still arrives, once the earlier MMAs are done
                    mma_commit(tfull0 + 8 * ts);
                    if (++ts == kMmaTSlots) { ts = 0; tph ^= 1; }
                }
                if (ok) mma_commit(empty0 + 8 * slot);
            }
            // nothing may still read shared memory or write TMEM when the CTA
            // frees them
            mma_commit(done_bar);
            mbar_drain(done_bar, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------ epilogue ------------------------------
        // Warp w reads TMEM lanes 32 * (w % 4) ..; the two warps of a lane
        // quarter take activation columns [0, 8) and [8, 16).
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int grp = (warp - 2) >> 2;        // column group
        const int n0 = grp * kMmaNPG;
        const int row = 32 * q + lane;          // tile row = TMEM lane
        const int g = row >> 3, r = row & 7;    // packed group and row in it
        const int e = threadIdx.x - 64;         // table entry of this thread (< 128)
        const bool tab_thread = e < kMmaSB * kMmaN;
        const int jt = (e >> 4) & (kMmaSB - 1), nt = e & 15;  // (block in stage, activation row)
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + n0;
        pdl_wait_and_trigger();  // activation scales and outputs belong to the previous grid until now
        auto dx_load = [&](int it, int ks) -> float {  // ks: the k step of iteration it
            if (it >= total || !tab_thread) return 0.f;
            const int b = b_lo + ks * kMmaSB + jt;
            return (b < b_hi && nt < a.N) ? __half2float(__ushort_as_half(__ldg(a.xd + (size_t)nt * a.B + b)))
                                          : 0.f;
        };
        float dx_next = dx_load(0, 0);
        uint64_t acc2[kMmaNPG / 2];  // fp32 pairs (n0 + 2p, n0 + 2p + 1)
        // acc += float(dot) * d_w * d_x for blocks j0 .. j0 + 3 of the stage
        auto compute_half = [&](auto full, const uint32_t(&v)[kMmaHalfBlocks * kMmaNPG], int j0, int nb,
                                const uint8_t *st) {
            constexpr bool FULL = decltype(full)::value;
            const uint64_t nmagic = pack_u32x2(0xCB400000u, 0xCB400000u);  // -1.5 * 2^23
#pragma unroll
            for (int jj = 0; jj < kMmaHalfBlocks; ++jj) {
                const int j = j0 + jj;
                if (!FULL && j >= nb) break;
                const float dw = __half2float(*reinterpret_cast<const __half *>(
                    st + kMmaDOff + (g * kMmaSB + j) * 16 + r * 2));
                const float4 *tab = reinterpret_cast<const float4 *>(st + kMmaTabOff + j * kMmaN * 8);
                const uint64_t dw2 = pack_u32x2(__float_as_uint(dw), __float_as_uint(dw));
                const uint32_t *vb = v + jj * kMmaNPG;
#pragma unroll
                for (int p = 0; p < kMmaNPG / 4; ++p) {
                    const float4 dx4 = tab[n0 / 4 + p];
                    const float4 kc4 = tab[kMmaN / 4 + n0 / 4 + p];
                    const int n = 4 * p;
                    const uint64_t f01 = add_f32x2(pack_u32x2(vb[n] + __float_as_uint(kc4.x),
                                                              vb[n + 1] + __float_as_uint(kc4.y)), nmagic);
                    const uint64_t f23 = add_f32x2(pack_u32x2(vb[n + 2] + __float_as_uint(kc4.z),
                                                              vb[n + 3] + __float_as_uint(kc4.w)), nmagic);
                    const uint64_t s01 = mul_f32x2(dw2, pack_u32x2(__float_as_uint(dx4.x), __float_as_uint(dx4.y)));
                    const uint64_t s23 = mul_f32x2(dw2, pack_u32x2(__float_as_uint(dx4.z), __float_as_uint(dx4.w)));
                    acc2[2 * p] = fma_f32x2(f01, s01, acc2[2 * p]);
                    acc2[2 * p + 1] = fma_f32x2(f23, s23, acc2[2 * p + 1]);
                }
            }
        };
        int it = 0, slot = 0, phase = 0;  // ring position of iteration `it`, carried along
        int ts = 0, tph = 0;              // TMEM slot of the next half and its phase
        for (int tl = 0; tl < n_tiles; ++tl) {
#pragma unroll
            for (int p = 0; p < kMmaNPG / 2; ++p) acc2[p] = 0ull;
            for (int ks = 0; ks < ksteps;
                 ++ks, ++it, slot = slot + 1 == a.stages ? 0 : slot + 1, phase ^= slot == 0 ? 1 : 0) {
                uint8_t *st = smem + (size_t)slot * kMmaStageBytes;
                bool ok = mbar_wait_warp(full0 + 8 * slot, phase, abort_flag);
                const float dx_cur = dx_next;
                dx_next = dx_load(it + 1, ks + 1 == ksteps ? 0 : ks + 1);  // one stage ahead: it has a stage to land
                if (ok && tab_thread) {
                    // table entry (jt, nt): d_x and the int bits that fold the
                    // 128 * sum(xq) correction into the float conversion
                    const uint4 *xs = reinterpret_cast<const uint4 *>(st + kMmaXOff);
                    const int sx = byte_sum_s8(xs[(2 * jt + 1) * kMmaN + nt], byte_sum_s8(xs[2 * jt * kMmaN + nt], 0));
                    float *tab = reinterpret_cast<float *>(st + kMmaTabOff + jt * kMmaN * 8);
                    tab[nt] = dx_cur;
                    tab[kMmaN + nt] = __int_as_float(0x4B400000 - 128 * sx);
                }
                named_barrier(1, kMmaEpiThreads);
                const int nb = min(kMmaSB, nblk - ks * kMmaSB);
                // The TMEM loads of half h + 1 are issued before half h is
                // computed, so their latency hides behind the arithmetic
                // (tcgen05.wait::ld waits for every earlier load of the thread,
                // so one batch is in flight at a time).
                uint32_t va[kMmaHalfBlocks * kMmaNPG], vb[kMmaHalfBlocks * kMmaNPG];
                // wait for half h's slot and issue its loads (no wait)
                auto fetch = [&](int h, uint32_t(&v)[kMmaHalfBlocks * kMmaNPG]) -> bool {
                    const bool okh = mbar_wait_warp(tfull0 + 8 * ts, tph, abort_flag);
                    if (okh && h * kMmaHalfBlocks < nb) {
                        tc_fence_after();
#pragma unroll
                        for (int jj = 0; jj < kMmaHalfBlocks; ++jj) {
                            const uint32_t ta = taddr + ts * kMmaSlotCols + jj * kMmaN;
                            if constexpr (kMmaNPG == 8)
                                tmem_ld8_async(ta, v + jj * kMmaNPG);
                            else
                                tmem_ld4_async(ta, v + jj * kMmaNPG);
                        }
                    }
                    return okh;
                };
                // wait for the loads in flight, then hand the slot back to the MMAs
                auto land = [&](int h, uint32_t(&v)[kMmaHalfBlocks * kMmaNPG]) {
                    if (h * kMmaHalfBlocks < nb) {
#pragma unroll
                        for (int i = 0; i < kMmaHalfBlocks * kMmaNPG; i += 8) tmem_wait_ld8(v + i);
                        tc_fence_before();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty0 + 8 * ts);
                    if (++ts == kMmaTSlots) { ts = 0; tph ^= 1; }
                };
                auto compute = [&](int h, const uint32_t(&v)[kMmaHalfBlocks * kMmaNPG]) {
                    // a full stage takes the branch-free path, so the four
                    // blocks' loads and arithmetic can interleave
                    if (nb == kMmaSB)
                        compute_half(std::true_type{}, v, h * kMmaHalfBlocks, nb, st);
                    else
                        compute_half(std::false_type{}, v, h * kMmaHalfBlocks, nb, st);
                };
                static_assert(kMmaHalves % 2 == 0, "halves go in pairs through va, vb");
                if (ok) {
                    ok = fetch(0, va);
                    if (ok) land(0, va);
                }
#pragma unroll
                for (int h = 0; h < kMmaHalves && ok; h += 2) {
                    // va holds half h; vb takes half h + 1
                    ok = fetch(h + 1, vb);
                    if (!ok) break;
                    compute(h, va);
                    land(h + 1, vb);
                    if (h + 2 < kMmaHalves) {
                        ok = fetch(h + 2, va);
                        if (!ok) break;
                    }
                    compute(h + 1, vb);
                    if (h + 2 < kMmaHalves) land(h + 2, va);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty0 + 8 * slot);
            }
            // ---- tile done: K-split partials meet in the leader, rank order ----
            float acc[kMmaNPG];
#pragma unroll
            for (int p = 0; p < kMmaNPG / 2; ++p) {
                const float2 f = unpack_f32x2(acc2[p]);
                acc[2 * p] = f.x;
                acc[2 * p + 1] = f.y;
            }
            const int grow = (t0 + tl) * 128 + row;
            bool store = true;
            if (S > 1) {
                if (rank != 0) {
                    store = false;
                    if (tl == 0 || mbar_wait_cluster(redfree, (tl - 1) & 1, abort_flag)) {
#pragma unroll
                        for (int n = 0; n < kMmaNPG; ++n) red[(n0 + n) * 128 + row] = acc[n];
                    }
                    mbar_arrive_cluster(map_to_rank(redfull, 0));
                } else {
                    if (mbar_wait_cluster(redfull, tl & 1, abort_flag)) {
                        for (int p = 1; p < S; ++p) {
                            const uint32_t base = map_to_rank(smem_u32(red), (uint32_t)p);
#pragma unroll
                            for (int n = 0; n < kMmaNPG; ++n)
                                acc[n] += ld_cluster_f32(base + ((n0 + n) * 128 + row) * 4);
                        }
                    } else {
                        store = false;
                    }
                    for (int p = 1; p < S; ++p) mbar_arrive_cluster(map_to_rank(redfree, (uint32_t)p));
                }
            }
            if (store && grow < a.M) {
#pragma unroll
                for (int n = 0; n < kMmaNPG; ++n)
                    if (n0 + n < a.N) a.y[(size_t)(n0 + n) * a.M + grow] = acc[n];
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kMmaTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag) {
        const int n_issued = *issued;
        for (int i = n_issued > a.stages ? n_issued - a.stages : 0; i < n_issued; ++i)
            mbar_drain(full0 + 8 * (i % a.stages), (i / a.stages) & 1);
    }
    __syncwarp();
    // no CTA leaves while a peer may still read its partials
    if (S > 1) cluster_sync_all();
}

}  // namespace q8
