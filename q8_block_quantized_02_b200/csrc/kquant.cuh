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
// One warp per output row (grid-stride); lane l takes the 32-weight chunks
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

}  // namespace q8
