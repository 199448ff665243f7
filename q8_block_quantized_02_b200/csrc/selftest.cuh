// selftest.cuh -- a test aid for the failure-detection protocol: a kernel whose
// warps wait, through the same bounded-wait routine as the pipelines, on a
// shared-memory barrier that nothing ever completes.  The first wait to run
// past its (short) limit records kErrWaitTimeout in the sticky device error
// word and raises the CTA's abort flag; every other warp sees the flag and
// leaves its wait; the kernel returns normally.  No fault, trap or endless
// loop is involved, so the context stays usable.
#pragma once

#include "q8_device.cuh"

namespace q8 {

constexpr int kSelftestThreads = 128;

__global__ void __launch_bounds__(kSelftestThreads, 1) wait_timeout_kernel(uint64_t limit_ns, int *out) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    __shared__ int ok_warps;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);  // one arrival completes it; none ever comes
        abort_flag = 0;
        ok_warps = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait_and_trigger();
    const bool ok = mbar_wait_warp(smem_u32(&bar), 0, &abort_flag, limit_ns);
    if ((threadIdx.x & 31) == 0 && ok) atomicAdd(&ok_warps, 1);
    __syncthreads();
    // [0]: warps whose wait succeeded (0 expected), [1]: the abort flag
    if (threadIdx.x == 0) {
        out[0] = ok_warps;
        out[1] = abort_flag;
    }
}

}  // namespace q8
