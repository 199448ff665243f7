// route.cuh -- S5: MoE router.  One warp per token: softmax over the E gate
// logits and top-k selection by logit value (softmax is monotone), ties to
// the lowest expert index, picks in descending order.
#pragma once

#include "q8_device.cuh"

namespace q8 {

constexpr int kRouteMaxE = 256;  // 8 experts per lane
constexpr int kRouteMaxK = 8;

__global__ void route_kernel(const float *__restrict__ logits, int T, int E, int top_k,
                             int renormalize, int32_t *__restrict__ idx, float *__restrict__ w) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *l = logits + (size_t)t * E;
    float v[kRouteMaxE / 32];
#pragma unroll
    for (int i = 0; i < kRouteMaxE / 32; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? l[e] : -INFINITY;
    }
    unsigned taken = 0;  // bit i: expert lane + 32 i already picked
    int pick_e[kRouteMaxK];
    float pick_v[kRouteMaxK];
    for (int s = 0; s < top_k; ++s) {
        // lane-local best among unpicked experts (lowest index on ties)
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kRouteMaxE / 32; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
                bv = v[i];
                be = e;
            }
        }
        // warp argmax, lowest index on ties
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        pick_e[s] = be;
        pick_v[s] = bv;
        if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
    }
    // softmax denominator over all E experts, relative to the largest logit
    const float mx = pick_v[0];
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < kRouteMaxE / 32; ++i)
        if (lane + 32 * i < E) z += expf(v[i] - mx);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane == 0) {
        float p[kRouteMaxK], sp = 0.f;
        for (int s = 0; s < top_k; ++s) {
            p[s] = expf(pick_v[s] - mx) / z;
            sp += p[s];
        }
        for (int s = 0; s < top_k; ++s) {
            idx[(size_t)t * top_k + s] = pick_e[s];
            w[(size_t)t * top_k + s] = renormalize ? p[s] / sp : p[s];
        }
    }
}

}  // namespace q8
