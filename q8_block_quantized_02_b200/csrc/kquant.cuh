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
// The first kernel (every Q6_K product, and Q4_K at N = 3, 4): one warp per
// output row (grid-stride); lane l takes the 32-weight chunks
// l, l + 32, ... of the row: it decodes its chunk's scale (and min) once,
// forms each weight with one fp32 FMA (Q4_K: d*sc*q - dmin*m; Q6_K:
// d*scale*(q-32), exact), and multiplies it into every activation row.
// Lanes' partial sums meet in a fixed shuffle tree, so results are
// bit-identical from run to run.
#pragma once

#include "q8_device.cuh"

namespace q8 {

constexpr int kKqThreads = 256;

// Sub-block j's 6-bit scale and min from the 12 packed bytes of a Q4_K block.
__device__ __forceinline__ void q4k_scale_min(const uint8_t *s, int j, int &sc, int &m) {
    if (j < 4) {
        sc = s[j] & 63;
        m = s[j + 4] & 63;
    } else {
        sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
        m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
}

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

// FMT 4: Q4_K; FMT 6: Q6_K.
template <int NMAX, int FMT>
__global__ void __launch_bounds__(kKqThreads) kquant_gemv_kernel(const uint8_t *__restrict__ W,
                                                                 const float *__restrict__ x,
                                                                 float *__restrict__ y, int M, int K, int N) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int BYTES = FMT == 4 ? 144 : 210;
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
            if (FMT == 4) {
                const uint32_t dw = *reinterpret_cast<const uint32_t *>(blk);
                const float d = __half2float(__ushort_as_half((unsigned short)(dw & 0xFFFFu)));
                const float dmin = __half2float(__ushort_as_half((unsigned short)(dw >> 16)));
                int sc, m;
                q4k_scale_min(blk + 4, cc, sc, m);
                const float a = d * (float)sc, b = dmin * (float)m;  // both exact in fp32
                const uint4 *qs = reinterpret_cast<const uint4 *>(blk + 16 + 32 * (cc >> 1));
                const int shift = 4 * (cc & 1);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 v = qs[h];
                    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        float w[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint32_t byte = (words[2 * p + (i >> 2)] >> (8 * (i & 3))) & 0xFFu;
                            w[i] = fmaf(a, (float)((byte >> shift) & 15u), -b);
                        }
                        kq_dot8<NMAX>(w, x, K, N, k0 + 16 * h + 8 * p, acc);
                    }
                }
            } else {
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
// Q4_K at N <= 2: activations held in registers across rows
// ---------------------------------------------------------------------------
// The kernel above re-reads x for every row, and holds one row's loads at a
// time.  Here a CTA takes a tile of
// kQ4Rows rows at a time and its warps split the row's super-blocks between
// them (warp w: blocks w, w + warps, ...).  Within a warp, lane (r, u) =
// (lane >> 3, lane & 7) takes the 16-byte piece u of the block's 128 nibble
// bytes for rows r, r + 4, ..., r + kQ4Rows - 4 of the tile: piece u = 2t + h
// holds weights 64t + 16h + i (low nibbles, sub-block 2t) and 64t + 32 + 16h
// + i (high nibbles, sub-block 2t + 1), i < 16.  So the lane loads those 32
// activations once per (tile, block) and reuses them for kQ4Rows / 4 rows;
// the 8 lanes of a row read its block's 128 bytes contiguously.  A nibble
// becomes a float without a conversion: masked into a byte and permuted
// into the low mantissa of 2^23 it gives 2^23 + q exactly, and one paired
// subtract leaves q; each weight is then one fma(d*sc, q, -dmin*m) (d*sc and
// dmin*m exact in fp32), so it carries one rounding, relative to itself, as
// in the kernel above (factoring the sub-block's terms out of the sum would
// be cheaper, but its rounding would scale with d*sc*sum q x and dmin*m*sum x,
// not with sum |w x|, which cancel when the weights are near zero).  The 32
// weights are dotted with packed f32x2 FMAs.  The weight bytes reach the warp
// through a per-warp ring in shared memory (below): cp.async copies of the
// next blocks' 32 rows are in flight while it computes, so HBM sees many
// requests per SM without holding them in registers.  Row sums: the 8 lanes
// of a row by a shuffle tree, then the warps' partials in warp order (fixed
// order, so results are bit-identical from run to run).
constexpr int kQ4Warps = 8;
constexpr int kQ4Threads = kQ4Warps * 32;
constexpr int kQ4Rows = 32;  // rows per tile (8 per lane)

// The 32 weights of a 16-byte nibble piece v as fp32 pairs: lo[k] the low
// nibbles (sub-block 2t, scale a0 = d*sc, offset b0 = dmin*m), hi[k] the high
// ones (sub-block 2t + 1: a1, b1); element 2k, 2k + 1 of a run are bytes
// 2k, 2k + 1 of v.  Each weight is fma(a, q, -b): one rounding of the exact
// d*sc*q - dmin*m, as in the row-per-warp kernel.
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

// The 6-bit scale and min of sub-block j from the 12 scale bytes held in the
// words s1 (bytes 0-3), s2 (4-7), s3 (8-11), as small exact floats.
__device__ __forceinline__ void q4_sc_m(uint32_t s1, uint32_t s2, uint32_t s3, int j, float &sc, float &m) {
    uint32_t a, b;
    if (j < 4) {
        a = (s1 >> (8 * j)) & 63u;
        b = (s2 >> (8 * j)) & 63u;
    } else {
        const int k = 8 * (j - 4);
        a = ((s3 >> k) & 15u) | (((s1 >> k) >> 6 & 3u) << 4);
        b = ((s3 >> k) >> 4 & 15u) | (((s2 >> k) >> 6 & 3u) << 4);
    }
    sc = __uint_as_float(0x4B000000u | a) - 8388608.0f;
    m = __uint_as_float(0x4B000000u | b) - 8388608.0f;
}

// 16-byte asynchronous copy global -> shared (L2 only), and its group fences.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int PENDING>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(PENDING) : "memory");
}

// Per warp, a ring of kQ4Stages stages of one block of the tile's rows: the
// raw bytes [kQ4Rows rows][144 B], copied by the warp's lanes (9 pieces of
// 16 B per row) while the warp computes an earlier stage.
constexpr int kQ4Stages = 3;
constexpr int kQ4StageBytes = kQ4Rows * 144;
constexpr int kQ4SmemBytes = kQ4Warps * kQ4Stages * kQ4StageBytes + kQ4Warps * 2 * kQ4Rows * 4;

// N = 1: two CTAs per SM (128 registers a thread, 2 x 112 KB of shared
// memory), twice the warps to hide the dequantise-and-dot latencies.
template <int NMAX>
__global__ void __launch_bounds__(kQ4Threads, NMAX == 1 ? 2 : 1)
    q4k_tile_kernel(const uint8_t *__restrict__ W, const float *__restrict__ x, float *__restrict__ y, int M, int K,
                    int N) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = smem + warp * kQ4Stages * kQ4StageBytes;
    float *red = reinterpret_cast<float *>(smem + kQ4Warps * kQ4Stages * kQ4StageBytes);  // [warp][n][row]
    const int r = lane >> 3, u = lane & 7, t = u >> 1, h = u & 1;
    const int SB = K >> 8;
    const size_t row_bytes = (size_t)SB * 144;
    const int tiles = (M + kQ4Rows - 1) / kQ4Rows;
    constexpr int IT = kQ4Rows / 4;  // rows per lane per tile
    pdl_wait();
    pdl_launch_dependents();
    // this warp's (tile, block) steps, in order: tiles of the CTA, blocks
    // warp, warp + kQ4Warps, ... of each
    const int nb = SB > warp ? (SB - warp + kQ4Warps - 1) / kQ4Warps : 0;  // blocks per tile for this warp
    const int my_tiles = tiles > (int)blockIdx.x ? (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const int steps = nb * my_tiles;
    // copy step s into its stage: 32 rows x 9 pieces, 9 pieces per lane
    auto issue = [&](int s) {
        if (s < steps) {
            const int tile = (int)blockIdx.x + (s / nb) * (int)gridDim.x;
            const int b = warp + (s % nb) * kQ4Warps;
            const uint32_t st = smem_u32(ring + (s % kQ4Stages) * kQ4StageBytes);
#pragma unroll
            for (int k = 0; k < 9; ++k) {
                const int p = lane + 32 * k, rr = p / 9, c = p - 9 * rr;
                const int row = min(tile * kQ4Rows + rr, M - 1);  // rows past M: the last row again, never stored
                cp_async16(st + rr * 144 + c * 16, W + (size_t)row * row_bytes + (size_t)b * 144 + c * 16);
            }
        }
        cp_async_commit();  // an empty group past the end keeps the count uniform
    };
#pragma unroll
    for (int s = 0; s < kQ4Stages - 1; ++s) issue(s);
    int s = 0;
    for (int ti = 0; ti < my_tiles; ++ti) {
        const int row0 = ((int)blockIdx.x + ti * (int)gridDim.x) * kQ4Rows;
        float acc[IT][NMAX];
#pragma unroll
        for (int i = 0; i < IT; ++i)
#pragma unroll
            for (int n = 0; n < NMAX; ++n) acc[i][n] = 0.f;
        for (int bi = 0; bi < nb; ++bi, ++s) {
            issue(s + kQ4Stages - 1);
            const int b = warp + bi * kQ4Warps;
            // this lane's 32 activations per column: two runs of 16 (L1/L2)
            const int k_lo = 256 * b + 64 * t + 16 * h, k_hi = k_lo + 32;
            uint64_t xlo[NMAX][8], xhi[NMAX][8];
#pragma unroll
            for (int n = 0; n < NMAX; ++n) {
                const ulonglong2 *pl = reinterpret_cast<const ulonglong2 *>(x + (size_t)(n < N ? n : 0) * K + k_lo);
                const ulonglong2 *ph = reinterpret_cast<const ulonglong2 *>(x + (size_t)(n < N ? n : 0) * K + k_hi);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const ulonglong2 a = __ldg(pl + i), c = __ldg(ph + i);
                    xlo[n][2 * i] = a.x;
                    xlo[n][2 * i + 1] = a.y;
                    xhi[n][2 * i] = c.x;
                    xhi[n][2 * i + 1] = c.y;
                }
            }
            cp_async_wait<kQ4Stages - 1>();  // this lane's copies of step s have landed
            __syncwarp();                    // ... and every other lane's
            const uint8_t *st = ring + (s % kQ4Stages) * kQ4StageBytes;
#pragma unroll
            for (int i = 0; i < IT; ++i) {
                const uint8_t *blk = st + (r + 4 * i) * 144;
                const uint4 hd = *reinterpret_cast<const uint4 *>(blk);           // d, dmin, scales
                const uint4 qv = *reinterpret_cast<const uint4 *>(blk + 16 + 16 * u);  // piece u
                const float d = __half2float(__ushort_as_half((unsigned short)(hd.x & 0xFFFFu)));
                const float dmin = __half2float(__ushort_as_half((unsigned short)(hd.x >> 16)));
                float sc0, m0, sc1, m1;
                q4_sc_m(hd.y, hd.z, hd.w, 2 * t, sc0, m0);
                q4_sc_m(hd.y, hd.z, hd.w, 2 * t + 1, sc1, m1);
                // d*sc and dmin*m are exact in fp32 (11 x 6 significant bits)
                const uint32_t a0 = __float_as_uint(d * sc0), b0 = __float_as_uint(-(dmin * m0));
                const uint32_t a1 = __float_as_uint(d * sc1), b1 = __float_as_uint(-(dmin * m1));
                uint64_t wl[8], wh[8];
                q4_weights(qv, pack_u32x2(a0, a0), pack_u32x2(b0, b0), pack_u32x2(a1, a1), pack_u32x2(b1, b1), wl, wh);
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
            }
            __syncwarp();  // the stage is read before a later issue() overwrites it
        }
        // the 8 lanes of a row, then the warps in order (a warp with no block
        // of this row leaves zeros)
#pragma unroll
        for (int i = 0; i < IT; ++i)
#pragma unroll
            for (int n = 0; n < NMAX; ++n) {
                float v = acc[i][n];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                if (u == 0) red[(warp * NMAX + n) * kQ4Rows + r + 4 * i] = v;
            }
        __syncthreads();
        if (threadIdx.x < NMAX * kQ4Rows) {
            const int n = threadIdx.x / kQ4Rows, rr = threadIdx.x % kQ4Rows;
            const int row = row0 + rr;
            if (n < N && row < M) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kQ4Warps; ++w) sum += red[(w * NMAX + n) * kQ4Rows + rr];
                y[(size_t)n * M + row] = sum;
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();  // nothing may still land after the CTA exits
}

}  // namespace q8
