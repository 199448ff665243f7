// kquant.cuh -- the K-quant decode GEMV: Q4_K and Q6_K weights (GGUF
// super-blocks of 256 weights, read in their raw layout) times 1..4 fp32
// activation rows, on the CUDA cores.  These are the formats of the Q4_K /
// Q6_K GEMV probes of the "skuznetsov/cogni-ml" README ("Build Qwen CLIs"),
// which also run over the raw GGUF blocks.
//
// Block layouts (the GGUF packing; include/q8.h states them in full):
//   Q4_K, 144 B: d | dmin (binary16) | scales[12] (6-bit scale and min of 8
//   sub-blocks of 32) | qs[128] (nibbles; bytes 32t..32t+31 hold sub-block
//   2t in the low and 2t+1 in the high nibbles).  w = d*sc*q - dmin*m.
//   Q6_K, 210 B: ql[128] | qh[64] | scales[16] (int8, per 16 weights) | d.
//   w = d*scale*(q - 32), q = 4 low bits from ql, 2 high bits from qh.
//
// Q6_K on raw blocks (q8_q6k_gemv): one warp per output row (grid-stride);
// lane l takes the 32-weight chunks l, l + 32, ... of the row, decodes the
// chunk's two scales once, forms each weight d*scale*(q-32) exactly in fp32
// and multiplies it into every activation row.  Lanes' partial sums meet in a
// fixed shuffle tree, so results are bit-identical from run to run.  Raw
// blocks start on 2-byte boundaries, so this kernel reads bytes; the packed
// units below serve the tile kernel.
#pragma once

#include "q8_device.cuh"

namespace q8 {

constexpr int kKqThreads = 256;

// acc[n] += sum over 8 weights w[0..7] of w * x[n][k0 .. k0 + 7]
template <int NMAX>
__device__ __forceinline__ void kq_dot8(const float (&w)[8], const float *__restrict__ x, int K, int N,
                                        int64_t k0, float (&acc)[NMAX]) {
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        if (n < N) {
            const float4 *xs = reinterpret_cast<const float4 *>(x + (size_t)n * K + k0);
            const float4 a = __ldg(xs), b = __ldg(xs + 1);
            float s = acc[n];
            s = fmaf(w[0], a.x, s);
            s = fmaf(w[1], a.y, s);
            s = fmaf(w[2], a.z, s);
            s = fmaf(w[3], a.w, s);
            s = fmaf(w[4], b.x, s);
            s = fmaf(w[5], b.y, s);
            s = fmaf(w[6], b.z, s);
            s = fmaf(w[7], b.w, s);
            acc[n] = s;
        }
    }
}

template <int NMAX>
__global__ void __launch_bounds__(kKqThreads) q6k_row_kernel(const uint8_t *__restrict__ W,
                                                             const float *__restrict__ x,
                                                             float *__restrict__ y, int M, int K, int N) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int BYTES = 210;
    const int lane = threadIdx.x & 31;
    const int SB = K / 256, chunks = K / 32;
    const int warps = (int)(gridDim.x * (kKqThreads / 32));
    for (int row = (int)(blockIdx.x * (kKqThreads / 32) + (threadIdx.x >> 5)); row < M; row += warps) {
        float acc[NMAX];
#pragma unroll
        for (int n = 0; n < NMAX; ++n) acc[n] = 0.f;
        for (int c = lane; c < chunks; c += 32) {
            const uint8_t *blk = W + ((size_t)row * SB + (c >> 3)) * BYTES;
            const int cc = c & 7;
            const int64_t k0 = (int64_t)c * 32;
            const int hh = cc >> 2, c4 = cc & 3;
            const uint8_t *ql = blk + 64 * hh + 32 * (c4 & 1);
            const uint8_t *qh = blk + 128 + 32 * hh;
            const int8_t *scl = reinterpret_cast<const int8_t *>(blk + 192 + 8 * hh + 2 * c4);
            const float d = __half2float(__ushort_as_half(
                (unsigned short)(blk[208] | ((unsigned)blk[209] << 8))));
            const float a0 = d * (float)scl[0], a1 = d * (float)scl[1];  // exact in fp32
            const int lshift = 4 * (c4 >> 1), hshift = 2 * c4;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                float w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int l = 8 * p + i;
                    const int q = (int)(((ql[l] >> lshift) & 15) | (((qh[l] >> hshift) & 3) << 4)) - 32;
                    w[i] = (l < 16 ? a0 : a1) * (float)q;  // exact: 11 x 8 x 6 significant bits
                }
                kq_dot8<NMAX>(w, x, K, N, k0 + 8 * p, acc);
            }
        }
#pragma unroll
        for (int n = 0; n < NMAX; ++n)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[n] += __shfl_xor_sync(0xffffffffu, acc[n], o);
        if (lane == 0) {
#pragma unroll
            for (int n = 0; n < NMAX; ++n)
                if (n < N) y[(size_t)n * M + row] = acc[n];
        }
    }
}

// ---------------------------------------------------------------------------
// Tile kernel (N <= 2): Q4_K on its raw blocks, Q6_K on the packed layout
// ---------------------------------------------------------------------------
// The kernel above re-reads x for every row, and holds one row's loads at a
// time.  Here a CTA of 8 warps takes tiles of kKqRows = 32 output rows; within
// a tile, warp w takes super-blocks b = w', w' + 8, ... (w' = w rotated by
// i * SB for the CTA's i-th tile, so that over a few consecutive tiles every
// warp gets the same share when SB is not a multiple of 8; rotating by the
// global tile index would not, since a CTA's tiles are a grid apart).  A
// warp's (tile, block) steps stream through its own ring of shared-memory
// stages, each holding one block of the tile's 32 rows and filled by one copy
// that lane 0 issues on the stage's mbarrier:
//   * Q4_K: the raw rows are 144 * SB bytes, so a 3-D TMA box {144 B, 1 block,
//     32 rows} lands the stage as [32 rows][144 B] (rows past M read as zero);
//   * Q6_K: raw 210-byte blocks start on 2-byte boundaries, out of reach of
//     TMA and of 16-byte async copies, so the weights are first packed
//     (q8_q6k_pack_weights) into 6720-byte units, one per (tile, block):
//     [32 rows][ql 128 | qh 64 | scales 16] then the 32 binary16 d's.  One
//     bulk copy brings a unit.
// Lane (r, u) = (lane >> 3, lane & 7) takes piece u (a 16-byte run of the
// block's value bytes) of rows r, r + 4, ..., r + 28 of the stage, and loads
// the 32 activations that piece multiplies once per step, reusing them over
// the 8 rows.  The 8 lanes of a row read 128 contiguous bytes: no bank
// conflicts.
//   * Q4_K piece u = 2t + h: weights 64t + 16h + i (low nibbles, sub-block 2t)
//     and 64t + 32 + 16h + i (high nibbles, sub-block 2t + 1), i < 16.  Each
//     weight is fma(d*sc, q, -dmin*m) (d*sc and dmin*m exact in fp32), one
//     rounding relative to itself: factoring the sub-block's terms out of
//     the sum would be cheaper, but its rounding would scale with
//     d*sc*sum q x and dmin*m*sum x, not with sum |w x|, and the two cancel
//     when the weights are near zero.  Each lane decodes one sub-block's
//     6-bit scale and min; the lanes of a row exchange them by shuffles.
//   * Q6_K piece u = 4hh + 2a + j: ql bytes 64hh + 32a + 16j + i (i < 16) give
//     weights 128hh + 32a + 16j + i (low nibble, 2 high bits from qh byte
//     32hh + 16j + i at bit 2a, scale 8hh + 2a + j) and 128hh + 64 + 32a + 16j
//     + i (high nibble, qh bits 2a + 4, scale 8hh + 4 + 2a + j).  q - 32 is
//     exact in fp32, so each 16-weight run is dotted as sum (q - 32) x and
//     scaled once by d * scale (exact): the rounding is relative to
//     sum |w x| all the same, since w = d * scale * (q - 32) has no offset
//     term that could cancel.
// A 4- or 6-bit value becomes a float without a conversion: placed in the low
// mantissa bits of 2^23 by a byte permute it gives 2^23 + q exactly, and one
// paired subtract removes the bias.  Dots use packed f32x2 FMAs.
// Row sums: the 8 lanes of a row by a shuffle tree, then the 8 warps'
// partials in warp order by one reducer warp per tile (warp i % 8 for the
// CTA's i-th tile), so results are bit-identical from run to run (the
// rotation depends on the grid, so they may differ between GPUs with
// different SM counts).  The partials go through RB shared buffers (4 at
// N = 1, 2 at N = 2; tile i uses buffer i % RB) under named barriers: a warp
// arrives on the buffer's "full" barrier and moves on; only the reducer waits
// there.  Before writing tile i's partials a warp waits on the buffer's
// "free" barrier, on which the reducer of tile i - RB arrives once it has
// read them.  So no computing warp waits for a slower one, except across RB
// tiles.
constexpr int kKqWarps = 8;
constexpr int kKqTileThreads = kKqWarps * 32;
constexpr int kKqRows = 32;                      // rows per tile (8 per lane)
constexpr int kQ4StageBytes = kKqRows * 144;     // 4608
constexpr int kQ6RowBytes = 208;                 // ql | qh | scales of one row
constexpr int kQ6UnitBytes = kKqRows * kQ6RowBytes + kKqRows * 2;  // 6720
constexpr int kQ6DOff = kKqRows * kQ6RowBytes;   // 6656
// partial-sum buffers (tiles in flight): 4 at N = 1, 2 at N = 2 (so that two
// CTAs fit on an SM)
template <int NMAX>
__host__ __device__ constexpr int kq_red_bufs() { return NMAX == 1 ? 4 : 2; }

template <int FMT>
__host__ __device__ constexpr int kq_stage_bytes() { return FMT == 4 ? kQ4StageBytes : kQ6UnitBytes; }
// Shared memory: rings [warp][stage] | partials [RB][warp][NMAX][32] | barriers [warp][stage] | abort flag
template <int FMT, int NMAX, int STAGES>
__host__ __device__ constexpr int kq_red_off() { return kKqWarps * STAGES * kq_stage_bytes<FMT>(); }
template <int FMT, int NMAX, int STAGES>
__host__ __device__ constexpr int kq_bar_off() {
    return kq_red_off<FMT, NMAX, STAGES>() + kq_red_bufs<NMAX>() * kKqWarps * NMAX * kKqRows * 4;
}
template <int FMT, int NMAX, int STAGES>
__host__ __device__ constexpr int kq_smem_bytes() { return kq_bar_off<FMT, NMAX, STAGES>() + kKqWarps * STAGES * 8 + 16; }

// Named barriers of the partial-sum exchange (0 is __syncthreads').
constexpr int kKqBarFull = 1;  // + buffer
constexpr int kKqBarFree = 5;  // + buffer
__device__ __forceinline__ void named_arrive(int id, int threads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Bulk (non-tensor) copy global -> shared completing on an mbarrier; both
// addresses 16-byte aligned, size a multiple of 16 (no multicast).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// The 32 weights of a 16-byte Q4_K nibble piece v as fp32 pairs: lo[k] the low
// nibbles (sub-block 2t, scale a0 = d*sc, offset b0 = dmin*m), hi[k] the high
// ones (sub-block 2t + 1: a1, b1); element 2k, 2k + 1 of a run are bytes
// 2k, 2k + 1 of v.  Each weight is fma(a, q, -b): one rounding of the exact
// d*sc*q - dmin*m.
__device__ __forceinline__ void q4_weights(const uint4 v, uint64_t a0, uint64_t nb0, uint64_t a1, uint64_t nb1,
                                           uint64_t (&lo)[8], uint64_t (&hi)[8]) {
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
    const uint32_t nm = __float_as_uint(-8388608.0f);
    const uint64_t neg = pack_u32x2(nm, nm);  // 2^23 + q - 2^23 = q, exact
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t l = words[i] & 0x0F0F0F0Fu, h = (words[i] >> 4) & 0x0F0F0F0Fu;
        const uint64_t l0 = add_f32x2(pack_u32x2(__byte_perm(l, 0x4B000000u, 0x7540u), __byte_perm(l, 0x4B000000u, 0x7541u)), neg);
        const uint64_t l1 = add_f32x2(pack_u32x2(__byte_perm(l, 0x4B000000u, 0x7542u), __byte_perm(l, 0x4B000000u, 0x7543u)), neg);
        const uint64_t h0 = add_f32x2(pack_u32x2(__byte_perm(h, 0x4B000000u, 0x7540u), __byte_perm(h, 0x4B000000u, 0x7541u)), neg);
        const uint64_t h1 = add_f32x2(pack_u32x2(__byte_perm(h, 0x4B000000u, 0x7542u), __byte_perm(h, 0x4B000000u, 0x7543u)), neg);
        lo[2 * i] = fma_f32x2(a0, l0, nb0);
        lo[2 * i + 1] = fma_f32x2(a0, l1, nb0);
        hi[2 * i] = fma_f32x2(a1, h0, nb1);
        hi[2 * i + 1] = fma_f32x2(a1, h1, nb1);
    }
}

// Sub-block j's 6-bit scale (bits 0..5) and min (bits 16..21) from the 12
// scale bytes held in s1 (bytes 0-3), s2 (4-7), s3 (8-11), without a branch
// on j: j < 4 takes the low 6 bits of bytes j and j + 4; j >= 4 takes the
// nibbles of byte j + 4 and the top 2 bits of bytes j - 4 and j.
__device__ __forceinline__ uint32_t q4_sc_m_packed(uint32_t s1, uint32_t s2, uint32_t s3, int j) {
    const uint32_t sel = 0x4440u | (uint32_t)(j & 3);  // byte j % 4 into byte 0, zeros above
    const uint32_t c1 = __byte_perm(s1, 0u, sel), c2 = __byte_perm(s2, 0u, sel), c3 = __byte_perm(s3, 0u, sel);
    const uint32_t sc = j < 4 ? (c1 & 63u) : ((c3 & 15u) | ((c1 >> 2) & 0x30u));
    const uint32_t m = j < 4 ? (c2 & 63u) : ((c3 >> 4) | ((c2 >> 2) & 0x30u));
    return sc | (m << 16);
}

// q - 32 of the 16 Q6_K values of one run as fp32 pairs: 4 low bits per byte
// of `ql4` (already shifted down), 2 high bits per byte at bits 4..5 of `qh4`.
__device__ __forceinline__ void q6_values(const uint32_t (&ql4)[4], const uint32_t (&qh4)[4], uint64_t (&w)[8]) {
    const uint32_t nb = __float_as_uint(-8388640.0f);  // -(2^23 + 32)
    const uint64_t neg = pack_u32x2(nb, nb);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t q = (ql4[i] & 0x0F0F0F0Fu) | (qh4[i] & 0x30303030u);
        w[2 * i] = add_f32x2(pack_u32x2(__byte_perm(q, 0x4B000000u, 0x7540u), __byte_perm(q, 0x4B000000u, 0x7541u)), neg);
        w[2 * i + 1] = add_f32x2(pack_u32x2(__byte_perm(q, 0x4B000000u, 0x7542u), __byte_perm(q, 0x4B000000u, 0x7543u)), neg);
    }
}

// sum over 16 weights (8 pairs) of w * x, in a fixed order
__device__ __forceinline__ float dot16_pairs(const uint64_t (&w)[8], const uint64_t (&x)[8]) {
    uint64_t p0 = mul_f32x2(w[0], x[0]), p1 = mul_f32x2(w[1], x[1]);
#pragma unroll
    for (int k = 2; k < 8; k += 2) {
        p0 = fma_f32x2(w[k], x[k], p0);
        p1 = fma_f32x2(w[k + 1], x[k + 1], p1);
    }
    const float2 s = unpack_f32x2(add_f32x2(p0, p1));
    return s.x + s.y;
}

// FMT 4: Q4_K raw blocks through `tmap` ({144, SB, M} bytes); FMT 6: Q6_K
// packed units at W.  MINB CTAs per SM.
template <int FMT, int NMAX, int STAGES, int MINB>
__global__ void __launch_bounds__(kKqTileThreads, MINB)
    kq_tile_kernel(const __grid_constant__ CUtensorMap tmap, const uint8_t *__restrict__ W,
                   const float *__restrict__ x, float *__restrict__ y, int M, int K, int N) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int SBYTES = kq_stage_bytes<FMT>();
    constexpr int IT = kKqRows / 4;  // rows per lane per tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 3, u = lane & 7;
    uint8_t *ring = smem + warp * STAGES * SBYTES;
    float *red = reinterpret_cast<float *>(smem + kq_red_off<FMT, NMAX, STAGES>());  // [2][warp][n][row]
    const uint32_t bar0 = smem_u32(smem + kq_bar_off<FMT, NMAX, STAGES>()) + warp * STAGES * 8;
    volatile int *abort_flag =
        reinterpret_cast<volatile int *>(smem + kq_bar_off<FMT, NMAX, STAGES>() + kKqWarps * STAGES * 8);
    const int SB = K >> 8;
    const int tiles = (M + kKqRows - 1) / kKqRows;
    const int my_tiles = tiles > (int)blockIdx.x ? (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    {
        uint32_t dyn;
        asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if (dyn < (uint32_t)kq_smem_bytes<FMT, NMAX, STAGES>() || blockDim.x != kKqTileThreads) {
            if (threadIdx.x == 0) record_error(kErrLaunchConfig);
            return;
        }
    }
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
        if (warp == 0) *abort_flag = 0;
        fence_mbar_init();
    }
    if (FMT == 4 && threadIdx.x == 0) prefetch_tensormap(&tmap);
    __syncthreads();
    // warp w's first block in tile t: blocks rotate by t * SB (mod 8)
    const int sb8 = SB & 7;
    auto first_block = [&](int ti) { return (warp - (ti & 7) * sb8) & 7; };
    auto blocks_of = [&](int ti) {
        const int b0 = first_block(ti);
        return b0 < SB ? (SB - b0 + kKqWarps - 1) / kKqWarps : 0;
    };
    // producer iterator (lane 0): the (tile, block) of step `issued`
    int p_ti = 0, p_bi = 0, p_nb = my_tiles > 0 ? blocks_of(0) : 0;
    int p_slot = 0, issued = 0;
    const uint64_t pw = policy_evict_first();
    bool broken = false;
    auto issue_next = [&]() {
        // advance past tiles where this warp has no block
        while (p_ti < my_tiles && p_bi >= p_nb) {
            ++p_ti;
            p_bi = 0;
            p_nb = p_ti < my_tiles ? blocks_of(p_ti) : 0;
        }
        if (p_ti >= my_tiles || broken) return;
        const int tile = (int)blockIdx.x + p_ti * (int)gridDim.x;
        const int b = first_block(p_ti) + p_bi * kKqWarps;
        if (lane == 0) {
            const uint32_t bar = bar0 + 8 * p_slot;
            const uint32_t dst = smem_u32(ring + p_slot * SBYTES);
            mbar_arrive_expect_tx(bar, SBYTES);
            if (FMT == 4)
                tma_load_3d(dst, &tmap, bar, 0, b, tile * kKqRows, pw);
            else
                bulk_load(dst, W + ((size_t)tile * SB + b) * kQ6UnitBytes, SBYTES, bar, pw);
        }
        ++p_bi;
        ++issued;
        p_slot = p_slot + 1 == STAGES ? 0 : p_slot + 1;
    };
    // weights do not depend on the previous grid: start the first copies now
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) issue_next();
    pdl_wait();
    pdl_launch_dependents();
    int c_slot = 0, c_phase = 0, consumed = 0;
    for (int ti = 0; ti < my_tiles; ++ti) {
        const int tile = (int)blockIdx.x + ti * (int)gridDim.x;
        const int row0 = tile * kKqRows;
        const int nb = blocks_of(ti), bfirst = first_block(ti);
        float acc[IT][NMAX];
#pragma unroll
        for (int i = 0; i < IT; ++i)
#pragma unroll
            for (int n = 0; n < NMAX; ++n) acc[i][n] = 0.f;
        for (int bi = 0; bi < nb; ++bi) {
            issue_next();
            const int b = bfirst + bi * kKqWarps;
            // this lane's 32 activations per column: two runs of 16 (L1/L2)
            int k_lo, k_hi;
            if (FMT == 4) {
                k_lo = 256 * b + 64 * (u >> 1) + 16 * (u & 1);
                k_hi = k_lo + 32;
            } else {
                k_lo = 256 * b + 16 * (u + 4 * (u >> 2));
                k_hi = k_lo + 64;
            }
            uint64_t xlo[NMAX][8], xhi[NMAX][8];
#pragma unroll
            for (int n = 0; n < NMAX; ++n) {
                const float *xn = x + (size_t)(n < N ? n : 0) * K;
                const ulonglong2 *pl = reinterpret_cast<const ulonglong2 *>(xn + k_lo);
                const ulonglong2 *ph = reinterpret_cast<const ulonglong2 *>(xn + k_hi);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const ulonglong2 va = __ldg(pl + i), vc = __ldg(ph + i);
                    xlo[n][2 * i] = va.x;
                    xlo[n][2 * i + 1] = va.y;
                    xhi[n][2 * i] = vc.x;
                    xhi[n][2 * i + 1] = vc.y;
                }
            }
            const bool ok = !broken && mbar_wait(bar0 + 8 * c_slot, c_phase, abort_flag);
            if (!ok) broken = true;
            if (ok) {
                const uint8_t *st = ring + c_slot * SBYTES;
#pragma unroll
                for (int i = 0; i < IT; ++i) {
                    const int rr = r + 4 * i;
                    if (FMT == 4) {
                        const uint8_t *blk = st + rr * 144;
                        const uint4 hd = *reinterpret_cast<const uint4 *>(blk);                // d, dmin, scales
                        const uint4 qv = *reinterpret_cast<const uint4 *>(blk + 16 + 16 * u);  // piece u
                        const float d = __half2float(__ushort_as_half((unsigned short)(hd.x & 0xFFFFu)));
                        const float dmin = __half2float(__ushort_as_half((unsigned short)(hd.x >> 16)));
                        // lane u decodes sub-block u's scale and min; this lane's
                        // sub-blocks 2t, 2t + 1 come from lanes 2t, 2t + 1 of its row
                        const uint32_t scm = q4_sc_m_packed(hd.y, hd.z, hd.w, u);
                        const int t = u >> 1, base = lane & ~7;
                        const uint32_t p0 = __shfl_sync(0xffffffffu, scm, base + 2 * t);
                        const uint32_t p1 = __shfl_sync(0xffffffffu, scm, base + 2 * t + 1);
                        // d*sc and dmin*m are exact in fp32 (11 x 6 significant bits):
                        // d * (2^23 + sc) - d * 2^23 in one fma
                        const float d23 = d * 8388608.0f, dm23 = dmin * 8388608.0f;
                        const uint32_t a0 = __float_as_uint(fmaf(d, __uint_as_float(0x4B000000u | (p0 & 63u)), -d23));
                        const uint32_t b0 = __float_as_uint(fmaf(-dmin, __uint_as_float(0x4B000000u | (p0 >> 16)), dm23));
                        const uint32_t a1 = __float_as_uint(fmaf(d, __uint_as_float(0x4B000000u | (p1 & 63u)), -d23));
                        const uint32_t b1 = __float_as_uint(fmaf(-dmin, __uint_as_float(0x4B000000u | (p1 >> 16)), dm23));
                        uint64_t wl[8], wh[8];
                        q4_weights(qv, pack_u32x2(a0, a0), pack_u32x2(b0, b0), pack_u32x2(a1, a1), pack_u32x2(b1, b1),
                                   wl, wh);
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) {
                            uint64_t p0 = mul_f32x2(wl[0], xlo[n][0]), p1 = mul_f32x2(wh[0], xhi[n][0]);
#pragma unroll
                            for (int k = 1; k < 8; ++k) {
                                p0 = fma_f32x2(wl[k], xlo[n][k], p0);
                                p1 = fma_f32x2(wh[k], xhi[n][k], p1);
                            }
                            const float2 sm = unpack_f32x2(add_f32x2(p0, p1));
                            acc[i][n] += sm.x + sm.y;
                        }
                    } else {
                        const uint8_t *row = st + rr * kQ6RowBytes;
                        const int hh = u >> 2, a = (u >> 1) & 1, j = u & 1;
                        const uint4 lv = *reinterpret_cast<const uint4 *>(row + 16 * u);
                        const uint4 hv = *reinterpret_cast<const uint4 *>(row + 128 + 16 * (2 * hh + j));
                        const uint2 sv = *reinterpret_cast<const uint2 *>(row + 192 + 8 * hh);
                        const float d = __half2float(*reinterpret_cast<const __half *>(st + kQ6DOff + 2 * rr));
                        // scales 8hh + 2a + j (low run) and + 4 (high run): bytes of sv
                        const int sel = 2 * a + j;
                        const int s_lo = (int)(int8_t)(uint8_t)(sv.x >> (8 * sel));
                        const int s_hi = (int)(int8_t)(uint8_t)(sv.y >> (8 * sel));
                        const float alo = d * (float)s_lo, ahi = d * (float)s_hi;  // exact: 11 x 8 bits
                        const uint32_t lw[4] = {lv.x, lv.y, lv.z, lv.w}, hw[4] = {hv.x, hv.y, hv.z, hv.w};
                        uint32_t ql4[4], qh4[4];
                        uint64_t w[8];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            ql4[k] = lw[k];
                            qh4[k] = hw[k] << (4 - 2 * a);  // bits 2a, 2a+1 -> 4, 5
                        }
                        q6_values(ql4, qh4, w);
                        float slo[NMAX];
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) slo[n] = dot16_pairs(w, xlo[n]);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            ql4[k] = lw[k] >> 4;
                            qh4[k] = hw[k] >> (2 * a);  // bits 2a+4, 2a+5 -> 4, 5
                        }
                        q6_values(ql4, qh4, w);
#pragma unroll
                        for (int n = 0; n < NMAX; ++n) {
                            const float shi = dot16_pairs(w, xhi[n]);
                            acc[i][n] = fmaf(ahi, shi, fmaf(alo, slo[n], acc[i][n]));
                        }
                    }
                }
            }
            __syncwarp();  // every lane has read the stage before a later copy refills it
            if (ok) {  // a broken pipeline stops here: its copies in flight are drained at the end
                ++consumed;
                c_slot = c_slot + 1 == STAGES ? 0 : c_slot + 1;
                c_phase ^= c_slot == 0 ? 1 : 0;
            }
        }
        // ---- partial sums: the 8 lanes of a row, then the warps in order ----
        constexpr int RB = kq_red_bufs<NMAX>();
        const int p = ti & (RB - 1);
        const int reducer = ti & 7;
        if (ti >= RB && warp != ((ti - RB) & 7)) named_barrier(kKqBarFree + p, kKqTileThreads);
        float *rp = red + (size_t)p * kKqWarps * NMAX * kKqRows;  // [warp][n][row] of buffer p
#pragma unroll
        for (int i = 0; i < IT; ++i)
#pragma unroll
            for (int n = 0; n < NMAX; ++n) {
                float v = acc[i][n];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                if (u == 0) rp[(warp * NMAX + n) * kKqRows + r + 4 * i] = v;
            }
        if (warp == reducer) {
            named_barrier(kKqBarFull + p, kKqTileThreads);
#pragma unroll
            for (int n = 0; n < NMAX; ++n) {
                const int row = row0 + lane;
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kKqWarps; ++w) sum += rp[(w * NMAX + n) * kKqRows + lane];
                if (n < N && row < M && !broken) y[(size_t)n * M + row] = sum;
            }
            __syncwarp();
            if (ti + RB < my_tiles) named_arrive(kKqBarFree + p, kKqTileThreads);
        } else {
            named_arrive(kKqBarFull + p, kKqTileThreads);
        }
    }
    // a broken pipeline: wait (bounded) for this warp's copies still in flight
    if (lane == 0) {
        for (; consumed < issued; ++consumed) {
            mbar_drain(bar0 + 8 * c_slot, c_phase);
            c_slot = c_slot + 1 == STAGES ? 0 : c_slot + 1;
            c_phase ^= c_slot == 0 ? 1 : 0;
        }
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Q6_K packing: raw GGUF blocks <-> the tile kernel's units
// ---------------------------------------------------------------------------
// Packed unit (tile t, block b), 6720 bytes at (t * SB + b) * 6720: row i of
// the tile (matrix row 32t + i) at byte 208 i holds bytes 0..207 of its raw
// block b (ql | qh | scales); bytes 6656 + 2i, 6657 + 2i hold its d.  Rows
// past M are zero.  One thread per output 16-byte piece, written whole.
__global__ void q6k_pack_kernel(const uint8_t *__restrict__ raw, uint8_t *__restrict__ packed, int M, int SB,
                                long long pieces) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int kPieces = kQ6UnitBytes / 16;  // 420
    for (long long pc = blockIdx.x * (long long)blockDim.x + threadIdx.x; pc < pieces;
         pc += (long long)gridDim.x * blockDim.x) {
        const long long unit = pc / kPieces;
        const int o0 = (int)(pc - unit * kPieces) * 16;
        const int tile = (int)(unit / SB), b = (int)(unit - (long long)tile * SB);
        uint32_t wv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t word = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int o = o0 + 4 * q + k;
                int i, src;
                if (o < kQ6DOff) {
                    i = o / kQ6RowBytes;
                    src = o - i * kQ6RowBytes;
                } else {
                    i = (o - kQ6DOff) >> 1;
                    src = 208 + ((o - kQ6DOff) & 1);
                }
                const int row = tile * kKqRows + i;
                const uint32_t byte = row < M ? raw[((size_t)row * SB + b) * 210 + src] : 0u;
                word |= byte << (8 * k);
            }
            wv[q] = word;
        }
        *reinterpret_cast<uint4 *>(packed + pc * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
}

// The inverse, one thread per raw byte.
__global__ void q6k_unpack_kernel(const uint8_t *__restrict__ packed, uint8_t *__restrict__ raw, int M, int SB,
                                  long long bytes) {
    pdl_wait();
    pdl_launch_dependents();
    for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < bytes;
         o += (long long)gridDim.x * blockDim.x) {
        const long long blk = o / 210;
        const int src = (int)(o - blk * 210);
        const int row = (int)(blk / SB), b = (int)(blk - (long long)row * SB);
        const int tile = row / kKqRows, i = row - tile * kKqRows;
        const size_t unit = ((size_t)tile * SB + b) * kQ6UnitBytes;
        raw[o] = src < kQ6RowBytes ? packed[unit + (size_t)i * kQ6RowBytes + src]
                                   : packed[unit + kQ6DOff + 2 * i + (src - kQ6RowBytes)];
    }
}

}  // namespace q8
