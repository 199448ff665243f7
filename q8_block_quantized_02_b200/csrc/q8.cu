// q8.cu -- libq8: the C ABI declared in include/q8.h.
//
// One translation unit: the kernels live in the included .cuh files, so the
// sticky device error word is a single symbol.  Every entry point validates
// its arguments on the host, picks a launch shape, and enqueues its kernels on
// the caller's stream with programmatic dependent launch; nothing here
// allocates, frees or synchronises (q8_read_device_error excepted).
#include "host_common.cuh"
#include "pack.cuh"
#include "q8q8.cuh"
#include "route.cuh"
#include "tile_gemm.cuh"

namespace q8 {

// ---------------------------------------------------------------------------
// tile GEMM (S2 / S3 / S4)
// ---------------------------------------------------------------------------
using TileKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, TileArgs);

template <int MODE>
static TileKernel tile_kernel_mode(int nmax) {
    switch (nmax) {
        case 1: return &tile_gemm_kernel<1, MODE>;
        case 2: return &tile_gemm_kernel<2, MODE>;
        case 4: return &tile_gemm_kernel<4, MODE>;
        case 8: return &tile_gemm_kernel<8, MODE>;
        default: return &tile_gemm_kernel<16, MODE>;
    }
}

static TileKernel tile_kernel_for(int nmax, int mode) {
    return mode == kModeF32 ? tile_kernel_mode<kModeF32>(nmax)
           : mode == kModeSwiGLU ? tile_kernel_mode<kModeSwiGLU>(nmax)
                                 : tile_kernel_mode<kModeQ8Q8>(nmax);
}

static cudaError_t setup_tile_kernels(int max_smem) {
    const int nm[5] = {1, 2, 4, 8, 16};
    for (int i = 0; i < 5; ++i)
        for (int mode = 0; mode < 3; ++mode) {
            cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void *>(tile_kernel_for(nm[i], mode)),
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}
static RegisterSetup g_reg_tile(setup_tile_kernels);

static int nmax_for(int64_t N) { return N <= 1 ? 1 : N <= 2 ? 2 : N <= 4 ? 4 : N <= 8 ? 8 : 16; }

struct TilePlan {
    TileArgs a;
    int grid;
    size_t smem;
};

static int64_t pow2_ceil(int64_t v) {
    int64_t p = 1;
    while (p < v) p <<= 1;
    return p;
}

// Launch shape for `units` row groups of C 16-byte columns.  The grid is one
// CTA per SM (or one per unit when there are fewer units); each CTA owns a
// contiguous unit range, taken in tiles of TG units.  A stage holds about
// 32 KB of weights (16 KB for each half of a SwiGLU tile) and at most 16 KB of
// activations.
static TilePlan plan_tile(int64_t units, int64_t C, int64_t N, int mode, int sms) {
    const bool swiglu = mode == kModeSwiGLU;
    const int64_t grid = units < sms ? units : sms;
    const int64_t upc = ceil_div(units, grid);
    const int64_t tg_max = swiglu ? 8 : 16;
    const int64_t tg = std::min<int64_t>(tg_max, pow2_ceil(upc));
    const int64_t pairs = swiglu ? 128 : 256;
    const int64_t eff = std::min<int64_t>(upc, tg);
    const int64_t x_col_bytes = mode == kModeQ8Q8 ? 16 : 64;  // per column per activation row
    const int nb = nmax_for(N);
    int64_t cs = std::max<int64_t>(8, (pairs / eff) / 8 * 8);
    cs = std::min<int64_t>(cs, round_up(C, 8));
    while (cs > 8 && nb * cs * x_col_bytes > 16384) cs -= 8;
    TilePlan p;
    TileArgs &a = p.a;
    a = TileArgs{};
    a.N = (int)N;
    a.C = (int)C;
    a.B = (int)(C / 2);
    a.units = (int)units;
    a.TG = (int)tg;
    a.CS = (int)cs;
    a.ksteps = (int)ceil_div(C, cs);
    a.NQ = (int)ceil_div(C, 4);
    const uint32_t halves = swiglu ? 2 : 1;
    a.q_box = (uint32_t)(cs * kColBytes);
    a.d_box = (uint32_t)(cs * 8);
    a.d_slot = (uint32_t)round_up(a.d_box, 128);
    a.x_box = (uint32_t)(N * cs * x_col_bytes);
    a.q_half = (uint32_t)tg * a.q_box;
    a.d_off = halves * a.q_half;
    a.d_half = (uint32_t)tg * a.d_slot;
    a.x_off = a.d_off + halves * a.d_half;
    a.stage_bytes = (uint32_t)round_up(a.x_off + a.x_box, 128);
    int stages = (int)(112 * 1024 / a.stage_bytes);
    a.stages = stages < 2 ? 2 : stages > 8 ? 8 : stages;
    p.grid = (int)grid;
    const int sets = swiglu ? 4 : 2;
    p.smem = (size_t)a.stages * a.stage_bytes + 16 * a.stages + tile_red_floats(nb, sets) * 4 + 16;
    return p;
}

static q8_status run_tile(const void *W, const void *x, const uint16_t *xd, float *y,
                          int64_t rows_out, int64_t K, int64_t N, int mode, cudaStream_t stream) {
    const bool swiglu = mode == kModeSwiGLU;
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int64_t B = K / 32, C = K / 16;
    const int64_t units = ceil_div(rows_out, kGroupRows);
    const int64_t total_groups = swiglu ? 2 * units : units;
    TilePlan p = plan_tile(units, C, N, mode, dev->sms);
    TileArgs &a = p.a;
    a.y = y;
    a.xd = xd;
    a.M_out = (int)rows_out;
    a.up_group0 = swiglu ? (int)units : 0;
    if (p.smem > (size_t)dev->max_smem_optin) return Q8_ERR_UNSUPPORTED;
    const uint64_t gstride = (uint64_t)kGroupBytesPerBlock * B;
    CUtensorMap tq, td, tx;
    Q8_CHECK(make_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, kColBytes, C, total_groups,
                         kColBytes, gstride, kColBytes, a.CS, 1, true));
    Q8_CHECK(make_map_3d(&td, CU_TENSOR_MAP_DATA_TYPE_UINT16,
                         static_cast<const uint8_t *>(W) + 256 * B, 8, B, total_groups, 16, gstride,
                         8, a.CS / 2, 1, true));
    if (mode == kModeQ8Q8)
        Q8_CHECK(make_map_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, x, 16, C, N, 16, (uint64_t)K, 16,
                             a.CS, (uint32_t)N, false));
    else
        Q8_CHECK(make_map_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, x, 16, C, N, 64,
                             (uint64_t)K * 4, 16, a.CS, (uint32_t)N, false));
    TileKernel k = tile_kernel_for(nmax_for(N), mode);
    const char *name = mode == kModeF32      ? "q8_gemv launch"
                       : mode == kModeSwiGLU ? "q8_gate_up_swiglu launch"
                                             : "q8q8_gemv launch";
    return launch_pdl(k, dim3(p.grid), dim3(kTileThreads), p.smem, stream, name, tq, td, tx, a);
}

}  // namespace q8

using namespace q8;

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char *q8_status_string(int status) {
    switch (status) {
        case Q8_OK: return "ok";
        case Q8_ERR_INVALID: return "invalid argument (null pointer or bad flag)";
        case Q8_ERR_SHAPE: return "invalid shape";
        case Q8_ERR_ALIGN: return "pointer not 16-byte aligned";
        case Q8_ERR_NOT_DEVICE: return "pointer is not device memory of the current device";
        case Q8_ERR_UNSUPPORTED: return "unsupported size (outside what the kernels serve)";
        case Q8_ERR_CUDA: return "CUDA error";
        case Q8_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
        default: return "unknown status";
    }
}

const char *q8_last_cuda_error(void) { return last_error_buf(); }

int q8_version(void) { return 100; }

q8_status q8_read_device_error(uint32_t *detail) {
    Q8_CUDA_TRY(cudaDeviceSynchronize());
    unsigned int word = 0, zero = 0;
    Q8_CUDA_TRY(cudaMemcpyFromSymbol(&word, g_q8_error, sizeof(word)));
    Q8_CUDA_TRY(cudaMemcpyToSymbol(g_q8_error, &zero, sizeof(zero)));
    if (detail) *detail = word;
    return word ? Q8_ERR_DEVICE_TIMEOUT : Q8_OK;
}

size_t q8_packed_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0 || K % 32) return 0;
    return (size_t)ceil_div(M, kGroupRows) * kGroupBytesPerBlock * (size_t)(K / 32);
}

q8_status q8_pack_weights(const void *gguf_blocks, int64_t M, int64_t K, void *packed,
                          q8_stream_t stream) {
    if (M <= 0 || K <= 0 || K % 32) return Q8_ERR_SHAPE;
    Q8_CHECK(check_device_ptr(gguf_blocks, false));
    Q8_CHECK(check_device_ptr(packed));
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int64_t B = K / 32;
    const int64_t total = ceil_div(M, kGroupRows) * kGroupRows * B;
    const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), (int64_t)dev->sms * 16);
    return launch_pdl(pack_kernel, dim3((unsigned)blocks), dim3(256), 0, (cudaStream_t)stream,
                      "q8_pack_weights launch", static_cast<const uint8_t *>(gguf_blocks),
                      static_cast<uint8_t *>(packed), M, B);
}

q8_status q8_unpack_weights(const void *packed, int64_t M, int64_t K, void *gguf_blocks,
                            q8_stream_t stream) {
    if (M <= 0 || K <= 0 || K % 32) return Q8_ERR_SHAPE;
    Q8_CHECK(check_device_ptr(packed));
    Q8_CHECK(check_device_ptr(gguf_blocks, false));
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int64_t B = K / 32;
    const int64_t blocks = std::min<int64_t>(ceil_div(M * B, 256), (int64_t)dev->sms * 16);
    return launch_pdl(unpack_kernel, dim3((unsigned)blocks), dim3(256), 0, (cudaStream_t)stream,
                      "q8_unpack_weights launch", static_cast<const uint8_t *>(packed),
                      static_cast<uint8_t *>(gguf_blocks), M, B);
}

q8_status q8_gemv(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                  q8_stream_t stream) {
    if (M <= 0 || K <= 0 || N <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > 16 || M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(y));
    return run_tile(W, x, nullptr, y, M, K, N, kModeF32, (cudaStream_t)stream);
}

q8_status q8_gate_up_swiglu(const void *W, const float *x, float *h, int64_t I, int64_t K,
                            int64_t N, q8_stream_t stream) {
    if (I <= 0 || K <= 0 || N <= 0 || K % 32 || I % 8) return Q8_ERR_SHAPE;
    if (N > 16 || I > (int64_t)1 << 29 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(h));
    return run_tile(W, x, nullptr, h, I, K, N, kModeSwiGLU, (cudaStream_t)stream);
}

q8_status q8_quantize_act(const float *x, int8_t *xq, uint16_t *xd, int64_t N, int64_t K,
                          q8_stream_t stream) {
    if (N <= 0 || K <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > (int64_t)1 << 20 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(xq));
    Q8_CHECK(check_device_ptr(xd, false));
    if (reinterpret_cast<uintptr_t>(xd) & 1u) return Q8_ERR_ALIGN;
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int64_t blocks = std::min<int64_t>(ceil_div(N * (K / 32), 128), (int64_t)dev->sms * 8);
    return launch_pdl(quantize_act_kernel, dim3((unsigned)blocks), dim3(128), 0,
                      (cudaStream_t)stream, "q8_quantize_act launch", x, xq, xd, N, K);
}

q8_status q8q8_gemv(const void *W, const int8_t *xq, const uint16_t *xd, float *y, int64_t M,
                    int64_t K, int64_t N, q8_stream_t stream) {
    if (M <= 0 || K <= 0 || N <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > 16 || M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(xq));
    Q8_CHECK(check_device_ptr(xd, false));
    if (reinterpret_cast<uintptr_t>(xd) & 1u) return Q8_ERR_ALIGN;
    Q8_CHECK(check_device_ptr(y));
    return run_tile(W, xq, xd, y, M, K, N, kModeQ8Q8, (cudaStream_t)stream);
}

q8_status q8q8_block_dots(const void *W, const int8_t *xq, int32_t *dots, int64_t M, int64_t K,
                          int64_t N, q8_stream_t stream) {
    if (M <= 0 || K <= 0 || N <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > 16 || M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(xq));
    Q8_CHECK(check_device_ptr(dots));
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int64_t blocks = std::min<int64_t>(ceil_div(N * M * (K / 32), 256), (int64_t)dev->sms * 16);
    return launch_pdl(block_dots_kernel, dim3((unsigned)blocks), dim3(256), 0,
                      (cudaStream_t)stream, "q8q8_block_dots launch",
                      static_cast<const uint8_t *>(W), xq, dots, M, K, N);
}

q8_status q8_moe_route(const float *logits, int64_t T, int64_t E, int64_t top_k,
                       int renormalize, int32_t *idx, float *w, q8_stream_t stream) {
    if (T <= 0 || E <= 0 || top_k <= 0 || top_k > E) return Q8_ERR_SHAPE;
    if (T > 16 || E > kRouteMaxE || top_k > kRouteMaxK) return Q8_ERR_UNSUPPORTED;
    if (renormalize != 0 && renormalize != 1) return Q8_ERR_INVALID;
    Q8_CHECK(check_device_ptr(logits, false));
    Q8_CHECK(check_device_ptr(idx, false));
    Q8_CHECK(check_device_ptr(w, false));
    if ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(idx) |
         reinterpret_cast<uintptr_t>(w)) & 3u)
        return Q8_ERR_ALIGN;
    const int warps = 4;
    return launch_pdl(route_kernel, dim3((unsigned)ceil_div(T, warps)), dim3(32 * warps), 0,
                      (cudaStream_t)stream, "q8_moe_route launch", logits, (int)T, (int)E,
                      (int)top_k, renormalize, idx, w);
}

size_t q8_moe_workspace_bytes(int64_t T, int64_t E, int64_t top_k, int64_t H, int64_t I,
                              int64_t I_shared) {
    (void)T; (void)E; (void)top_k; (void)H; (void)I; (void)I_shared;
    return 0;
}

q8_status q8_moe_gemv(const void *gate_up_experts, const void *down_experts,
                      const void *shared_gate_up, const void *shared_down,
                      const int32_t *idx, const float *w, const float *x, float *y, int64_t T,
                      int64_t E, int64_t top_k, int64_t H, int64_t I, int64_t I_shared,
                      void *workspace, size_t workspace_bytes, q8_stream_t stream) {
    (void)gate_up_experts; (void)down_experts; (void)shared_gate_up; (void)shared_down;
    (void)idx; (void)w; (void)x; (void)y; (void)T; (void)E; (void)top_k; (void)H; (void)I;
    (void)I_shared; (void)workspace; (void)workspace_bytes; (void)stream;
    return Q8_ERR_UNSUPPORTED;
}

}  // extern "C"
