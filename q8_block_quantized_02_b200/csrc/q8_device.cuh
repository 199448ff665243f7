// q8_device.cuh -- device-side building blocks shared by the libq8 kernels:
// shared-memory barriers, TMA tile loads, programmatic dependent launch, the
// bounded-wait protocol and the Q8_0 dequantisation of the packed layout.
// All inline PTX is written from the PTX ISA for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace q8 {

// ---------------------------------------------------------------------------
// Packed layout constants (see include/q8.h)
// ---------------------------------------------------------------------------
constexpr int kGroupRows = 8;          // rows per packed group
constexpr int kColBytes = 128;         // one 16-byte column of a group: 8 rows x 16 B
constexpr int kGroupBytesPerBlock = 272;  // per 32-weight block of a group: 256 q + 16 d

// ---------------------------------------------------------------------------
// Sticky device error word (read and cleared by q8_read_device_error)
// ---------------------------------------------------------------------------
enum : unsigned int {
    kErrWaitTimeout = 1u << 0,   // a pipeline barrier wait ran past its limit
    kErrDrainTimeout = 1u << 1,  // waiting for in-flight copies at exit ran out
    kErrBadExpert = 1u << 2,     // an expert index outside [0, E) was seen
    kErrLaunchConfig = 1u << 3,  // shared memory, cluster or tensor memory differ from the plan
};

__device__ unsigned int g_q8_error;

__device__ __forceinline__ void record_error(unsigned int bits) { atomicOr(&g_q8_error, bits); }

// A barrier wait gives up after this long (ns of %globaltimer).  Healthy waits
// in these kernels finish within microseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---------------------------------------------------------------------------
// Small PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may suspend the thread for up to `hint_ns` while the phase is
// incomplete, so a waiting thread takes no issue slots from working warps.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Suspend-time hint of the waiting loops: far below the wait limit, so the
// limit and the abort flag are still checked often.
constexpr uint32_t kWaitHintNs = 20000;

// Wait for the phase with the given parity to complete.  Returns false (and
// raises *abort) when the wait runs past kWaitLimitNs; returns false at once
// when *abort is already raised, so that every thread of a CTA leaves a broken
// pipeline quickly and still reaches the CTA's remaining barriers.
// (`limit_ns` is the wait limit; only the wait self-test passes a shorter one.)
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, kWaitHintNs)) return true;
        if (abort && *abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_error(kErrWaitTimeout);
            if (abort) *abort = 1;
            return false;
        }
    }
}

// mbar_wait for a whole warp: lane 0 alone polls the barrier (32 lanes polling
// one barrier serialise in the shared-memory pipe), then __syncwarp orders its
// acquire before every lane's reads of the guarded data.  Warp-uniform result.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int *abort,
                                               uint64_t limit_ns = kWaitLimitNs) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, limit_ns) ? 1 : 0;
    __syncwarp();
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Bounded wait used while draining in-flight copies before a CTA exits.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(kErrDrainTimeout);
            return;
        }
    }
}

// L2 policies: weights are streamed once (evict first); activations are
// re-read by every CTA (evict last).
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 3-D tiled TMA load global -> shared, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}

// 3-D tiled TMA prefetch of a box into L2 (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Programmatic dependent launch: wait for the grids this one depends on
// (no-op when launched without the attribute), and let the next grid on the
// stream start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// The kernels trigger their dependents only once their own wait has returned
// (every thread, after its wait): then at most the next kernel on the stream
// is resident early, prefetching its weights, and the block scheduler keeps
// free SMs, so two CTAs of one kernel seldom share an SM.
__device__ __forceinline__ void pdl_wait_and_trigger() {
    pdl_wait();
    pdl_launch_dependents();
}

// Named barrier over `threads` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------------------
// Q8_0 dequantisation of a packed 16-byte piece
// ---------------------------------------------------------------------------
// The packed layout stores each int8 q as the byte q + 128.  Placing that byte
// in the low mantissa bits of 2^23 gives the float 2^23 + 128 + q exactly;
// subtracting 2^23 + 128 leaves q exactly.  One byte permute + one add per
// weight, and no int->float conversion instruction.
__device__ __forceinline__ float biased_byte_to_float(uint32_t word, uint32_t sel) {
    return __uint_as_float(__byte_perm(word, 0x4B000000u, sel)) - 8388736.0f;
}

__device__ __forceinline__ void dequant16(const uint4 v, float (&w)[16]) {
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w[4 * i + 0] = biased_byte_to_float(words[i], 0x7540u);
        w[4 * i + 1] = biased_byte_to_float(words[i], 0x7541u);
        w[4 * i + 2] = biased_byte_to_float(words[i], 0x7542u);
        w[4 * i + 3] = biased_byte_to_float(words[i], 0x7543u);
    }
}

// Packed fp32 pairs (sm_100 f32x2 instructions: two IEEE fp32 operations per
// instruction, each rounded as the scalar one would be).
__device__ __forceinline__ uint64_t pack_u32x2(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ float2 unpack_f32x2(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return make_float2(lo, hi);
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Dequantise 16 packed bytes into 8 fp32 pairs (q0,q1), (q2,q3), ...: a byte
// permute per weight, then one paired subtraction of 2^23 + 128 per two.
__device__ __forceinline__ void dequant16_x2(const uint4 v, uint64_t (&w)[8]) {
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
    const uint32_t nb = __float_as_uint(-8388736.0f);
    const uint64_t neg_bias = pack_u32x2(nb, nb);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t b0 = __byte_perm(words[i], 0x4B000000u, 0x7540u);
        const uint32_t b1 = __byte_perm(words[i], 0x4B000000u, 0x7541u);
        const uint32_t b2 = __byte_perm(words[i], 0x4B000000u, 0x7542u);
        const uint32_t b3 = __byte_perm(words[i], 0x4B000000u, 0x7543u);
        w[2 * i] = add_f32x2(pack_u32x2(b0, b1), neg_bias);
        w[2 * i + 1] = add_f32x2(pack_u32x2(b2, b3), neg_bias);
    }
}

// sum_i w_i x_i over 16 values held as 8 pairs each (two interleaved chains).
__device__ __forceinline__ float dot16_x2(const uint64_t (&w)[8], const ulonglong2 x0,
                                          const ulonglong2 x1, const ulonglong2 x2,
                                          const ulonglong2 x3) {
    uint64_t a = mul_f32x2(w[0], x0.x), b = mul_f32x2(w[1], x0.y);
    a = fma_f32x2(w[2], x1.x, a);
    b = fma_f32x2(w[3], x1.y, b);
    a = fma_f32x2(w[4], x2.x, a);
    b = fma_f32x2(w[5], x2.y, b);
    a = fma_f32x2(w[6], x3.x, a);
    b = fma_f32x2(w[7], x3.y, b);
    const float2 s = unpack_f32x2(add_f32x2(a, b));
    return s.x + s.y;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

}  // namespace q8
