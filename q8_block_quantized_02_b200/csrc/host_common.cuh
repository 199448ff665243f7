// host_common.cuh -- host-side helpers for the libq8 entry points: status and
// error text, argument checks, device properties, TMA tensor-map encoding and
// kernel launches with programmatic dependent launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/q8.h"

namespace q8 {

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
inline char *last_error_buf() {
    static thread_local char buf[256] = "no error";
    return buf;
}

inline q8_status cuda_fail(cudaError_t e, const char *what) {
    snprintf(last_error_buf(), 256, "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
    return Q8_ERR_CUDA;
}

#define Q8_CUDA_TRY(expr)                                        \
    do {                                                         \
        cudaError_t e_ = (expr);                                 \
        if (e_ != cudaSuccess) return ::q8::cuda_fail(e_, #expr); \
    } while (0)

// ---------------------------------------------------------------------------
// per-device state
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sms = 0;
    int max_smem_optin = 0;
    bool ready = false;
};

inline DeviceInfo g_devices[kMaxDevices];
inline std::mutex g_device_mutex;

// Kernels that need more than 48 KB of dynamic shared memory register a hook
// here; it runs once per device, on the first library call on that device.
using DeviceSetupFn = cudaError_t (*)(int max_smem);
constexpr int kMaxSetupFns = 32;
inline DeviceSetupFn g_setup_fns[kMaxSetupFns];
inline int g_n_setup_fns = 0;

struct RegisterSetup {
    explicit RegisterSetup(DeviceSetupFn f) { g_setup_fns[g_n_setup_fns++] = f; }
};

inline q8_status device_info(const DeviceInfo **out) {
    int dev = 0;
    Q8_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice, "device index");
    DeviceInfo &d = g_devices[dev];
    if (!d.ready) {
        std::lock_guard<std::mutex> lock(g_device_mutex);
        if (!d.ready) {
            Q8_CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
            Q8_CUDA_TRY(cudaDeviceGetAttribute(&d.max_smem_optin,
                                               cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
            for (int i = 0; i < g_n_setup_fns; ++i) Q8_CUDA_TRY(g_setup_fns[i](d.max_smem_optin));
            d.ready = true;
        }
    }
    *out = &d;
    return Q8_OK;
}

// ---------------------------------------------------------------------------
// argument checks
// ---------------------------------------------------------------------------
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device memory of the current device (or managed memory).
inline q8_status check_device_ptr(const void *p, bool need_align = true) {
    if (!p) return Q8_ERR_INVALID;
    if (need_align && !aligned16(p)) return Q8_ERR_ALIGN;
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_NOT_DEVICE;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return Q8_ERR_NOT_DEVICE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || attr.device != dev) return Q8_ERR_NOT_DEVICE;
    return Q8_OK;
}

#define Q8_CHECK(expr)                       \
    do {                                     \
        q8_status s_ = (expr);               \
        if (s_ != Q8_OK) return s_;          \
    } while (0)

// ---------------------------------------------------------------------------
// TMA tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Encoded maps are kept in a small per-thread cache keyed by every encoding
// input: decode loops call the same matrices with the same buffers again and
// again, and encoding costs microseconds of host time.
struct MapKey {
    const void *base;
    uint64_t d0, d1, d2, s1, s2;
    uint32_t b0, b1, b2;
    int dtype;
    int stream_l2;
    int device;
    bool operator==(const MapKey &o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};

struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool valid;
};

constexpr int kMapCacheSize = 256;

inline q8_status encode_map_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                               uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
                               uint32_t b0, uint32_t b1, uint32_t b2, bool stream_l2);

// A 3-D tensor map over `base` with the given extents, byte strides of dims 1
// and 2, and box; zero fill outside the tensor, no swizzle.
inline q8_status make_map_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                             uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
                             uint32_t b0, uint32_t b1, uint32_t b2, bool stream_l2) {
    static thread_local MapEntry cache[kMapCacheSize];
    MapKey key;
    std::memset(&key, 0, sizeof(key));
    key.base = base;
    key.d0 = d0; key.d1 = d1; key.d2 = d2; key.s1 = s1; key.s2 = s2;
    key.b0 = b0; key.b1 = b1; key.b2 = b2;
    key.dtype = (int)dtype;
    key.stream_l2 = stream_l2 ? 1 : 0;
    int dev = 0;
    cudaGetDevice(&dev);
    key.device = dev;
    uint64_t h = reinterpret_cast<uintptr_t>(base) * 0x9E3779B97F4A7C15ull;
    h ^= (d1 * 31 + d2) * 0xC2B2AE3D27D4EB4Full ^ (b1 * 131 + b2 * 7 + (uint64_t)dtype);
    MapEntry &e = cache[(h >> 32) % kMapCacheSize];
    if (e.valid && e.key == key) {
        *map = e.map;
        return Q8_OK;
    }
    q8_status st = encode_map_3d(map, dtype, base, d0, d1, d2, s1, s2, b0, b1, b2, stream_l2);
    if (st == Q8_OK) {
        e.key = key;
        e.map = *map;
        e.valid = true;
    }
    return st;
}

inline q8_status encode_map_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                               uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
                               uint32_t b0, uint32_t b1, uint32_t b2, bool stream_l2) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) {
        snprintf(last_error_buf(), 256, "cuTensorMapEncodeTiled unavailable");
        return Q8_ERR_CUDA;
    }
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, dtype, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    stream_l2 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(last_error_buf(), 256, "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return Q8_ERR_CUDA;
    }
    return Q8_OK;
}

// ---------------------------------------------------------------------------
// launches (programmatic dependent launch on the given stream)
// ---------------------------------------------------------------------------
// `cluster_x` > 1 groups consecutive CTAs along x into thread-block clusters.
template <typename... KArgs, typename... Args>
inline q8_status launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, const char *name, unsigned cluster_x,
                                    Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster_x;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return Q8_OK;
}

template <typename... KArgs, typename... Args>
inline q8_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t stream, const char *name, Args &&...args) {
    return launch_pdl_cluster(kernel, grid, block, smem, stream, name, 1u, std::forward<Args>(args)...);
}

// How many clusters of `cluster_x` CTAs of `kernel` (threads, dynamic shared
// memory) the current device runs at once; cached per (device, kernel,
// threads, smem, cluster size).  Clusters are placed within one GPC, so with
// one CTA per SM a cluster size that does not divide a GPC's SMs leaves SMs
// idle: 28 clusters of 5 do not fit at once on a 148-SM part (26 do), and the
// last ones would run as a second wave.  0 when the query fails.
inline int max_active_clusters(const void *kernel, int threads, size_t smem, int cluster_x) {
    struct Entry {
        int dev;
        const void *k;
        int threads;
        size_t smem;
        int cx;
        int n;
    };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev && cache[i].k == kernel && cache[i].threads == threads && cache[i].smem == smem &&
            cache[i].cx == cluster_x)
            return cache[i].n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cluster_x);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();  // not sticky; clear it
        return 0;
    }
    if (used < 64) cache[used++] = Entry{dev, kernel, threads, smem, cluster_x, n};
    return n;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

}  // namespace q8
