// q8q8.cuh -- S7: activation quantisation to Q8_0, and the bit-exact int32
// block-dot test aid of S8.  (The Q8 x Q8 products themselves run in the tile
// kernel's kModeQ8Q8 and in the tensor-core kernel.)
#pragma once

#include "q8_device.cuh"

namespace q8 {

// Per (row n, block b), one warp: amax over the block, d32 = amax / 127,
// q = roundf(x / d32) clamped to +-127 (roundf rounds half away from zero),
// stored scale = binary16 RN of d32.  Divisions are IEEE round-to-nearest
// (__fdiv_rn) so the result is bit-exact with any IEEE implementation of the
// same steps.
__global__ void quantize_act_kernel(const float *__restrict__ x, int8_t *__restrict__ xq,
                                    uint16_t *__restrict__ xd, int64_t N, int64_t K) {
    // one warp per 32-block, lane i takes element i (the loads of a warp are
    // one coalesced 128-byte line; the block's max by a shuffle tree, exact)
    pdl_wait();
    pdl_launch_dependents();
    const int64_t B = K / 32;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < N * B; i += warps) {
        const float v = x[i * 32 + lane];
        float amax = fabsf(v);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float d32 = __fdiv_rn(amax, 127.0f);
        int q = 0;
        if (d32 != 0.0f) {
            float r = roundf(__fdiv_rn(v, d32));
            r = fminf(fmaxf(r, -127.0f), 127.0f);
            q = (int)r;
        }
        xq[i * 32 + lane] = (int8_t)q;
        if (lane == 0) xd[i] = __half_as_ushort(__float2half_rn(d32));
    }
}

// r = 1 / sqrt(sum / K + eps), correctly rounded; xhat = (x * r) * gamma, two
// fp32 roundings in that order (the "augur" README's Triton RMSNorm, section
// "Kernels", sums in fp32 and keeps its reference's order of conversions);
// then each 32-block of xhat is quantised by the rule of quantize_act_kernel,
// one warp per block (lane i takes element i).
constexpr int kRmsThreads = 256;

__global__ void __launch_bounds__(kRmsThreads) rmsnorm_quantize_kernel(
    const float *__restrict__ x, const float *__restrict__ gamma, float eps, int8_t *__restrict__ xq,
    uint16_t *__restrict__ xd, float *__restrict__ rinv, int64_t K) {
    __shared__ float part[kRmsThreads / 32];
    __shared__ float r_s;
    pdl_wait();
    pdl_launch_dependents();
    const int64_t n = blockIdx.x;
    const float *xr = x + n * K;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    float ss = 0.0f;
    for (int64_t i = t; i < K / 4; i += kRmsThreads) {
        const float4 v = reinterpret_cast<const float4 *>(xr)[i];
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) part[warp] = ss;
    __syncthreads();
    if (t == 0) {
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < kRmsThreads / 32; ++w) sum += part[w];
        const float r = __frsqrt_rn(__fadd_rn(__fdiv_rn(sum, (float)K), eps));
        r_s = r;
        if (rinv) rinv[n] = r;
    }
    __syncthreads();
    const float r = r_s;
    const int64_t B = K / 32;
    for (int64_t b = warp; b < B; b += kRmsThreads / 32) {
        const float xh = __fmul_rn(__fmul_rn(xr[32 * b + lane], r), gamma[32 * b + lane]);
        float amax = fabsf(xh);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float d32 = __fdiv_rn(amax, 127.0f);
        int q = 0;
        if (d32 != 0.0f) {
            float rq = roundf(__fdiv_rn(xh, d32));
            rq = fminf(fmaxf(rq, -127.0f), 127.0f);
            q = (int)rq;
        }
        xq[n * K + 32 * b + lane] = (int8_t)q;
        if (lane == 0) xd[n * B + b] = __half_as_ushort(__float2half_rn(d32));
    }
}

// Test aid: dots[n][m][b] = sum_i q_w[m][32b+i] * xq[n][32b+i], one thread per
// output, straight from the packed layout.
__global__ void block_dots_kernel(const uint8_t *__restrict__ W, const int8_t *__restrict__ xq,
                                  int32_t *__restrict__ dots, int64_t M, int64_t K, int64_t N) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t B = K / 32;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N * M * B;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = i % B, m = (i / B) % M, n = i / (B * M);
        const uint8_t *grp = W + (m / kGroupRows) * kGroupBytesPerBlock * B;
        const int r = (int)(m % kGroupRows);
        const uint4 lo = *reinterpret_cast<const uint4 *>(grp + (2 * b) * kColBytes + r * 16);
        const uint4 hi = *reinterpret_cast<const uint4 *>(grp + (2 * b + 1) * kColBytes + r * 16);
        const uint4 xa = *reinterpret_cast<const uint4 *>(xq + n * K + 32 * b);
        const uint4 xb = *reinterpret_cast<const uint4 *>(xq + n * K + 32 * b + 16);
        const uint32_t wq[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        const uint32_t xx[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        int dot = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            int d;
            asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(wq[k] ^ 0x80808080u), "r"(xx[k]), "r"(dot));
            dot = d;
        }
        dots[i] = dot;
    }
}

}  // namespace q8
