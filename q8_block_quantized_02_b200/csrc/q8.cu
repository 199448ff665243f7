// q8.cu -- libq8: the C ABI declared in include/q8.h.
//
// One translation unit: the kernels live in the included .cuh files, so the
// sticky device error word is a single symbol.  Every entry point validates
// its arguments on the host, picks a launch shape, and enqueues its kernels on
// the caller's stream with programmatic dependent launch; nothing here
// allocates, frees or synchronises (q8_read_device_error excepted).
#include <atomic>

#include "host_common.cuh"
#include "pack.cuh"
#include "q8q8.cuh"
#include "q8q8_mma.cuh"
#include "f32_mma.cuh"
#include "route.cuh"
#include "tile_gemm.cuh"
#include "resident.cuh"
#include "moe.cuh"
#include "kquant.cuh"
#include "selftest.cuh"

namespace q8 {

// ---------------------------------------------------------------------------
// tile GEMM (S2 / S3 / S4)
// ---------------------------------------------------------------------------
using TileKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                           TileArgs);

// `wide` selects, at N = 1, the 16-consumer-warp column kernel (more warps
// per SM for matrices with much work per CTA; the 8-warp kernels leave room
// for the next kernel on the stream to become resident early), and for N > 4
// the group-owner build that runs two CTAs per SM.
template <int MODE>
static TileKernel tile_kernel_mode(int nmax, bool wide) {
    switch (nmax) {
        case 1: return wide ? &cols_kernel<1, MODE, 16> : &cols_kernel<1, MODE, 8>;
        case 2: return &cols_kernel<2, MODE, 8>;
        case 4: return &cols_kernel<4, MODE, 8>;
        case 8: return wide ? &tile_gemm_kernel<8, MODE, 2> : &tile_gemm_kernel<8, MODE, 1>;
        default:
            return wide && tile_two_ctas_ok(16, MODE) ? &tile_gemm_kernel<16, MODE, 2> : &tile_gemm_kernel<16, MODE, 1>;
    }
}

static TileKernel tile_kernel_for(int nmax, int mode, bool wide = false) {
    return mode == kModeF32 ? tile_kernel_mode<kModeF32>(nmax, wide)
           : mode == kModeSwiGLU ? tile_kernel_mode<kModeSwiGLU>(nmax, wide)
                                 : tile_kernel_mode<kModeQ8Q8>(nmax, wide);
}

// Launch geometry of the kernel serving (nmax, mode): threads per CTA, the
// column-owner kernel's units per tile (0 for the group-owner kernel) and the
// floats of its partial-sum area.
struct KernelShape {
    int threads, tgm, red_floats;
};

template <int NMAX, int MODE, int CW>
static KernelShape cols_shape() {
    using C = ColsCfg<NMAX, MODE, CW>;
    return {C::THREADS, C::TGM, C::RED_FLOATS};
}

static KernelShape kernel_shape(int nmax, int mode, bool wide = false) {
    if (nmax <= 4) {
        switch (mode * 8 + nmax) {
            case kModeF32 * 8 + 1: return wide ? cols_shape<1, kModeF32, 16>() : cols_shape<1, kModeF32, 8>();
            case kModeF32 * 8 + 2: return cols_shape<2, kModeF32, 8>();
            case kModeF32 * 8 + 4: return cols_shape<4, kModeF32, 8>();
            case kModeSwiGLU * 8 + 1:
                return wide ? cols_shape<1, kModeSwiGLU, 16>() : cols_shape<1, kModeSwiGLU, 8>();
            case kModeSwiGLU * 8 + 2: return cols_shape<2, kModeSwiGLU, 8>();
            case kModeSwiGLU * 8 + 4: return cols_shape<4, kModeSwiGLU, 8>();
            case kModeQ8Q8 * 8 + 1: return wide ? cols_shape<1, kModeQ8Q8, 16>() : cols_shape<1, kModeQ8Q8, 8>();
            case kModeQ8Q8 * 8 + 2: return cols_shape<2, kModeQ8Q8, 8>();
            default: return cols_shape<4, kModeQ8Q8, 8>();
        }
    }
    const int sets = mode == kModeSwiGLU ? 4 : 2;
    return {kTileThreads, 0, tile_red_floats(nmax, sets)};
}

static cudaError_t setup_tile_kernels(int max_smem) {
    const int nm[5] = {1, 2, 4, 8, 16};
    for (int i = 0; i < 8; ++i)
        for (int mode = 0; mode < 3; ++mode) {
            const void *k = reinterpret_cast<const void *>(
                i < 5 ? tile_kernel_for(nm[i], mode) : tile_kernel_for(i == 5 ? 1 : i == 6 ? 8 : 16, mode, true));
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
            if (e != cudaSuccess) return e;
            // every tile kernel asks for the largest shared-memory carveout, so
            // consecutive kernels keep one SM configuration and can co-reside
            e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}
static RegisterSetup g_reg_tile(setup_tile_kernels);

static int nmax_for(int64_t N) { return N <= 1 ? 1 : N <= 2 ? 2 : N <= 4 ? 4 : N <= 8 ? 8 : 16; }

struct TilePlan {
    TileArgs a;
    int grid;
    int threads;
    bool wide;
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
    const int nb = nmax_for(N);
    const bool cols_path = nb <= 4;  // column-owner kernel (see tile_gemm.cuh)
    // the group-owner kernel (N > 4) is bound by its FP32 issue: two CTAs per
    // SM (each within half of it) double the warps that hide the FMA latency,
    // when there are units enough for whole tiles of 8 per CTA
    const bool dual = !cols_path && tile_two_ctas_ok(nb, mode) && units >= 16 * sms;
    const int64_t ctas = dual ? 2 * sms : sms;
    const int64_t grid = units < ctas ? units : ctas;
    const int64_t upc = ceil_div(units, grid);
    // much work per CTA (many row groups, or few very long ones): take the
    // 16-warp kernel (it fills the SM on its own); otherwise stay within half
    // an SM so the next kernel can co-reside
    const int64_t cta_bytes = upc * (swiglu ? 2 : 1) * C * (kColBytes + 8);
    const bool wide = (nb == 1 && (upc >= 32 || cta_bytes >= 256 * 1024)) || dual;
    const KernelShape ks = kernel_shape(nb, mode, wide);
    int64_t tg = cols_path ? ks.tgm : std::min<int64_t>(swiglu ? 8 : 16, pow2_ceil(upc));
    tg = std::min<int64_t>(tg, upc);  // a stage never holds more units than a CTA owns
    // weight (unit x column) pairs per stage: ~32 KB of packed weights
    const int64_t pairs = swiglu ? 128 : 256;
    const int64_t eff = std::min<int64_t>(upc, tg);
    const int64_t x_col_bytes = mode == kModeQ8Q8 ? 16 : 64;  // per column per activation row
    // CS is a multiple of 16, so every scale box is a multiple of 128 bytes and
    // a tile box lands in shared memory exactly as TG unit boxes would
    int64_t cs = std::max<int64_t>(16, (pairs / eff) / 16 * 16);
    cs = std::min<int64_t>(cs, round_up(C, 16));
    while (cs > 16 && nb * cs * x_col_bytes > 16384) cs -= 16;
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
    a.d_slot = a.d_box;
    a.x_box = (uint32_t)(N * cs * x_col_bytes);
    a.q_half = (uint32_t)tg * a.q_box;
    a.d_off = halves * a.q_half;
    a.d_half = (uint32_t)tg * a.d_slot;
    a.x_off = a.d_off + halves * a.d_half;
    a.stage_bytes = (uint32_t)round_up(a.x_off + a.x_box, 128);
    const int64_t fixed = (cols_path ? 32 : 0) + (int64_t)ks.red_floats * 4 + 16;
    const int64_t budget = (wide ? 124 * 1024 : 100 * 1024) - fixed;
    int64_t stages = budget / a.stage_bytes;
    stages = stages < 2 ? 2 : stages > 8 ? 8 : stages;
    // no more buffers than a CTA ever fills: small kernels then leave room for
    // the next kernel on the stream to become resident early
    stages = std::min<int64_t>(stages, ceil_div(upc, tg) * a.ksteps);
    a.stages = (int)stages;
    p.grid = (int)grid;
    p.threads = ks.threads;
    p.wide = wide;
    // must match the kernels' shared-memory carve-up (tile_gemm.cuh)
    p.smem = (size_t)a.stages * a.stage_bytes + 16 * a.stages + (cols_path ? 32 : 0) +
             (size_t)ks.red_floats * 4 + 16;
    return p;
}

// ---------------------------------------------------------------------------
// resident kernel: small matrices whose CTA-share of weights fits in shared
// memory (see tile_gemm.cuh)
// ---------------------------------------------------------------------------
using ResidentKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, const float *, TileArgs);

// N = 1 only.  One instance per row-group count, so the column step needs no
// per-group branch.
template <int MODE>
static ResidentKernel resident_kernel_mode(int tgm) {
    switch (tgm) {
        case 1: return &resident_kernel<1, MODE, 1>;
        case 2: return &resident_kernel<1, MODE, 2>;
        case 3: return &resident_kernel<1, MODE, 3>;
        case 4: return &resident_kernel<1, MODE, 4>;
        case 5: return &resident_kernel<1, MODE, 5>;
        case 6: return &resident_kernel<1, MODE, 6>;
        case 7: return &resident_kernel<1, MODE, 7>;
        default: return &resident_kernel<1, MODE, 8>;
    }
}
static ResidentKernel resident_kernel_for(int mode, int tgm) {
    return mode == kModeSwiGLU ? resident_kernel_mode<kModeSwiGLU>(tgm) : resident_kernel_mode<kModeF32>(tgm);
}
template <int MODE>
static int resident_red_floats_mode(int tgm) {
    switch (tgm) {
        case 1: return res_red_floats<1, MODE, 1>();
        case 2: return res_red_floats<1, MODE, 2>();
        case 3: return res_red_floats<1, MODE, 3>();
        case 4: return res_red_floats<1, MODE, 4>();
        case 5: return res_red_floats<1, MODE, 5>();
        case 6: return res_red_floats<1, MODE, 6>();
        case 7: return res_red_floats<1, MODE, 7>();
        default: return res_red_floats<1, MODE, 8>();
    }
}
static int resident_red_floats(int mode, int tgm) {
    return mode == kModeSwiGLU ? resident_red_floats_mode<kModeSwiGLU>(tgm) : resident_red_floats_mode<kModeF32>(tgm);
}
static int resident_threads(int mode, int tgm) {
    return 32 * (mode == kModeF32 && tgm == 1 ? res_warps<kModeF32, 1>() : res_warps<kModeSwiGLU, 2>());
}

static cudaError_t setup_resident_kernels(int max_smem) {
    for (int i = 0; i < 2 * kResTGM; ++i) {
        const void *k = reinterpret_cast<const void *>(resident_kernel_for(i / kResTGM, 1 + i % kResTGM));
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
static RegisterSetup g_reg_resident(setup_resident_kernels);

// Shared memory a resident launch may take: room is left on the SM for the
// next kernel on the stream to become resident early.
constexpr int64_t kResidentSmemBudget = 100 * 1024;

// Plan for the resident kernel, or false when the matrix is too large for it
// (more than kResTGM row groups per CTA, or the weights do not fit).
static bool plan_resident(int64_t units, int64_t C, int64_t N, int mode, int sms, TilePlan *out) {
    if (mode != kModeF32 && mode != kModeSwiGLU) return false;
    if (N != 1) return false;
    const int64_t grid = units < sms ? units : sms;
    const int64_t upc = ceil_div(units, grid);
    if (upc > kResTGM) return false;
    const int64_t halves = mode == kModeSwiGLU ? 2 : 1;
    // weight boxes of at most 256 columns, as even as multiples of 16 allow
    const int64_t nchunks = ceil_div(C, 256);
    const int64_t cb = round_up(ceil_div(C, nchunks), 16);
    const int64_t cs = nchunks * cb;
    TilePlan p;
    TileArgs &a = p.a;
    a = TileArgs{};
    a.N = (int)N;
    a.C = (int)C;
    a.B = (int)(C / 2);
    a.units = (int)units;
    a.TG = (int)upc;
    a.CS = (int)cs;
    a.ksteps = 1;
    a.NQ = (int)ceil_div(C, 4);
    a.stages = 1;
    a.CB = (int)cb;
    a.nchunks = (int)nchunks;
    a.q_box = (uint32_t)(cs * kColBytes);
    a.d_box = (uint32_t)(cs * 8);
    a.d_slot = a.d_box;
    a.x_box = (uint32_t)(N * cs * 64);
    a.q_half = (uint32_t)(upc * a.q_box);
    a.d_off = (uint32_t)(halves * a.q_half);
    a.d_half = (uint32_t)(upc * a.d_box);
    a.x_off = a.d_off + (uint32_t)(halves * a.d_half);
    a.stage_bytes = (uint32_t)round_up(a.x_off + a.x_box, 128);
    const int64_t smem = (int64_t)a.stage_bytes + (int64_t)resident_red_floats(mode, (int)upc) * 4 + 16;
    if (smem > kResidentSmemBudget) return false;
    if (halves * upc * (int64_t)(a.q_box + a.d_box) >= (1 << 20)) return false;  // mbarrier tx count
    p.grid = (int)grid;
    p.threads = resident_threads(mode, (int)upc);
    p.wide = false;
    p.smem = (size_t)smem;
    *out = p;
    return true;
}

static q8_status run_resident(const TilePlan &plan, const void *W, const float *x, float *y,
                              int64_t rows_out, int64_t K, int64_t N, int mode, cudaStream_t stream,
                              const float *res) {
    TilePlan p = plan;
    TileArgs &a = p.a;
    const bool swiglu = mode == kModeSwiGLU;
    const int64_t B = K / 32, C = K / 16;
    const int64_t total_groups = swiglu ? 2 * (int64_t)a.units : a.units;
    a.y = y;
    a.res = res;
    a.M_out = (int)rows_out;
    a.up_group0 = swiglu ? a.units : 0;
    const uint64_t gstride = (uint64_t)kGroupBytesPerBlock * B;
    const uint8_t *dbase = static_cast<const uint8_t *>(W) + 256 * B;
    // one chunk: maps whose box depth is the CTA's row-group count (TG, or
    // TG - 1 on the CTAs holding one fewer); several chunks: depth 1
    const uint32_t depth = a.nchunks == 1 ? (uint32_t)a.TG : 1u;
    const uint32_t depth1 = a.nchunks == 1 && a.TG > 1 ? (uint32_t)a.TG - 1 : depth;
    CUtensorMap tq, td, tq1, td1;
    Q8_CHECK(make_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, kColBytes, C, total_groups, kColBytes,
                         gstride, kColBytes, a.CB, depth, true));
    Q8_CHECK(make_map_3d(&td, CU_TENSOR_MAP_DATA_TYPE_UINT16, dbase, 8, B, total_groups, 16, gstride, 8,
                         a.CB / 2, depth, true));
    Q8_CHECK(make_map_3d(&tq1, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, kColBytes, C, total_groups, kColBytes,
                         gstride, kColBytes, a.CB, depth1, true));
    Q8_CHECK(make_map_3d(&td1, CU_TENSOR_MAP_DATA_TYPE_UINT16, dbase, 8, B, total_groups, 16, gstride, 8,
                         a.CB / 2, depth1, true));
    return launch_pdl(resident_kernel_for(mode, a.TG), dim3(p.grid), dim3(p.threads), p.smem, stream,
                      swiglu ? "q8_gate_up_swiglu launch" : "q8_gemv launch", tq, td, tq1, td1, x, a);
}

static q8_status run_fm(const void *W, const float *x, float *y, int64_t rows_out, int64_t K,
                        int64_t N, bool swiglu, cudaStream_t stream, const float *res);

constexpr int64_t kFmMinN = 5;       // smallest N the split entry points always send to the tensor cores
constexpr int64_t kFmMinNLarge = 3;  // ... and for matrices with a 128-row tile per SM or more

// The split entry points (q8_gemv_split, q8_gate_up_swiglu_split) send fp32
// activations to the tensor-core kernel from N = 5, and from N = 3 when the
// matrix has at least one output tile per SM (no K split): measured on the
// 7B-class shapes, 37888x3584 SwiGLU at N = 3 / 4 takes 46 / 49 us there
// against 69 / 77 us on the CUDA cores, 152064x3584 186 / 197 us against
// 259 / 291 us; the 3584x18944 down projection (28 tiles, K split over
// clusters) stays faster on the CUDA cores below N = 5 (42 / 48 us against
// 54 / 58 us).  The default entry points keep every N on the CUDA cores, whose
// error bound is relative to sum |w x| for every input.
static bool fm_serves(int64_t rows_out, int64_t N, bool swiglu, int sms) {
    if (N >= kFmMinN) return true;
    const int64_t tiles = ceil_div(rows_out, swiglu ? 64 : 128);
    return N >= kFmMinNLarge && tiles >= sms;
}

// `best` (fp32 GEMV, N <= 4 only): also leave the arg-max key of every
// column there (q8_gemv_argmax); the column-owner kernel serves it.
// `res` (fp32 GEMV): added to every output (q8_gemv_residual).
// `split` (fp32 modes): the tensor-core kernel with the three-term int8 split
// of x may serve the call where it is faster (fm_serves).
static q8_status run_tile(const void *W, const void *x, const uint16_t *xd, float *y,
                          int64_t rows_out, int64_t K, int64_t N, int mode, cudaStream_t stream,
                          unsigned long long *best = nullptr, const float *res = nullptr, bool split = false) {
    const bool swiglu = mode == kModeSwiGLU;
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    if (split && mode != kModeQ8Q8 && !best && fm_serves(rows_out, N, swiglu, dev->sms))
        return run_fm(W, static_cast<const float *>(x), y, rows_out, K, N, swiglu, stream, res);
    const int64_t B = K / 32, C = K / 16;
    const int64_t units = ceil_div(rows_out, kGroupRows);
    const int64_t total_groups = swiglu ? 2 * units : units;
    {
        TilePlan rp;
        if (!best && plan_resident(units, C, N, mode, dev->sms, &rp) && rp.smem <= (size_t)dev->max_smem_optin &&
            (uint64_t)units * (uint64_t)rp.grid < (1ull << 31))
            return run_resident(rp, W, static_cast<const float *>(x), y, rows_out, K, N, mode, stream, res);
    }
    TilePlan p = plan_tile(units, C, N, mode, dev->sms);
    TileArgs &a = p.a;
    a.y = y;
    a.best = best;
    a.res = res;
    a.xd = xd;
    a.M_out = (int)rows_out;
    a.up_group0 = swiglu ? (int)units : 0;
    if (p.smem > (size_t)dev->max_smem_optin) return Q8_ERR_UNSUPPORTED;
    const uint64_t gstride = (uint64_t)kGroupBytesPerBlock * B;
    if ((uint64_t)units * (uint64_t)p.grid >= (1ull << 31)) return Q8_ERR_UNSUPPORTED;
    CUtensorMap tq, td, tq1, td1, tx;
    const uint8_t *dbase = static_cast<const uint8_t *>(W) + 256 * B;
    Q8_CHECK(make_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, kColBytes, C, total_groups,
                         kColBytes, gstride, kColBytes, a.CS, a.TG, true));
    Q8_CHECK(make_map_3d(&td, CU_TENSOR_MAP_DATA_TYPE_UINT16, dbase, 8, B, total_groups, 16,
                         gstride, 8, a.CS / 2, a.TG, true));
    Q8_CHECK(make_map_3d(&tq1, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, kColBytes, C, total_groups,
                         kColBytes, gstride, kColBytes, a.CS, 1, true));
    Q8_CHECK(make_map_3d(&td1, CU_TENSOR_MAP_DATA_TYPE_UINT16, dbase, 8, B, total_groups, 16,
                         gstride, 8, a.CS / 2, 1, true));
    if (mode == kModeQ8Q8)
        Q8_CHECK(make_map_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, x, 16, C, N, 16, (uint64_t)K, 16,
                             a.CS, (uint32_t)N, false));
    else
        Q8_CHECK(make_map_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, x, 16, C, N, 64,
                             (uint64_t)K * 4, 16, a.CS, (uint32_t)N, false));
    TileKernel k = tile_kernel_for(nmax_for(N), mode, p.wide);
    const char *name = mode == kModeF32      ? "q8_gemv launch"
                       : mode == kModeSwiGLU ? "q8_gate_up_swiglu launch"
                                             : "q8q8_gemv launch";
    return launch_pdl(k, dim3(p.grid), dim3(p.threads), p.smem, stream, name, tq, td, tq1, td1,
                      tx, a);
}

// ---------------------------------------------------------------------------
// Q8 x Q8 on the tensor cores (S8, 9..16 activation columns)
// ---------------------------------------------------------------------------
#ifndef Q8_MMA_MIN_N
#define Q8_MMA_MIN_N 5
#endif
constexpr int64_t kMmaMinN = Q8_MMA_MIN_N;  // smallest N sent to the tcgen05 kernel
constexpr int kMmaMaxStages = 2;  // 78 KB stages: 32 columns (4 KB per group) keep HBM bursts long

static cudaError_t setup_mma_kernel(int max_smem) {
    const void *k = reinterpret_cast<const void *>(&q8q8_mma_kernel);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared);
}
static RegisterSetup g_reg_mma(setup_mma_kernel);

struct MmaPlan {
    MmaArgs a;
    int grid;     // CTAs (a multiple of a.split)
    size_t smem;
};

// One CTA per SM.  With at least as many 128-row tiles as SMs each cluster is
// one CTA walking a contiguous tile range; with fewer, every tile gets a
// cluster of up to 8 CTAs that split K between them: the largest split whose
// clusters all run at once (max_active_clusters), else none.
static MmaPlan plan_mma(int64_t M, int64_t K, int64_t N, int sms) {
    MmaPlan p;
    MmaArgs &a = p.a;
    a = MmaArgs{};
    const int64_t B = K / 32;
    const int64_t tiles = ceil_div(ceil_div(M, kGroupRows), kMmaTileGroups);
    a.M = (int)M;
    a.N = (int)N;
    a.B = (int)B;
    a.tiles = (int)tiles;
    auto finish = [&](int64_t split) {
        const int64_t clusters = tiles < sms ? tiles : sms;
        const int64_t blocks = ceil_div(B, split);
        const int64_t per_cta = ceil_div(tiles, clusters) * ceil_div(blocks, kMmaSB);
        a.split = (int)split;
        a.stages = (int)std::max<int64_t>(1, std::min<int64_t>(kMmaMaxStages, per_cta));
        p.grid = (int)(clusters * split);
        p.smem = mma_smem_bytes(a.stages, split > 1);
    };
    int64_t split = 1;
    if (tiles < sms) {
        split = std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(kMmaMaxSplit, sms / tiles), B));
        for (; split > 1; --split) {
            finish(split);
            if (max_active_clusters(reinterpret_cast<const void *>(&q8q8_mma_kernel), kMmaThreads, p.smem,
                                    (int)split) >= tiles)
                break;
        }
    }
    finish(split);
    return p;
}

static q8_status run_mma(const void *W, const int8_t *xq, const uint16_t *xd, float *y, int64_t M,
                         int64_t K, int64_t N, cudaStream_t stream) {
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int64_t B = K / 32, C = K / 16;
    const int64_t groups = ceil_div(M, kGroupRows);
    MmaPlan p = plan_mma(M, K, N, dev->sms);
    if (p.smem > (size_t)dev->max_smem_optin) return Q8_ERR_UNSUPPORTED;
    p.a.y = y;
    p.a.xd = xd;
    const uint64_t gstride = (uint64_t)kGroupBytesPerBlock * B;
    const uint8_t *dbase = static_cast<const uint8_t *>(W) + 256 * B;
    CUtensorMap tq, td, tx;
    // weights: [group][16-byte column][8 rows x 16 B], 16 groups x kMmaCS columns a box
    Q8_CHECK(make_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, kColBytes, C, groups, kColBytes,
                         gstride, kColBytes, kMmaCS, kMmaTileGroups, true));
    // scales: [group][block][8 rows] fp16
    Q8_CHECK(make_map_3d(&td, CU_TENSOR_MAP_DATA_TYPE_UINT16, dbase, 8, B, groups, 16, gstride, 8,
                         kMmaSB, kMmaTileGroups, true));
    // activations: [16-byte column][row][16 B]; rows past N read as zero
    Q8_CHECK(make_map_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, 16, N, C, (uint64_t)K, 16, 16,
                         kMmaN, kMmaCS, false));
    return launch_pdl_cluster(q8q8_mma_kernel, dim3(p.grid), dim3(kMmaThreads), p.smem, stream,
                              "q8q8_gemv (tensor cores) launch", (unsigned)p.a.split, tq, td, tx, p.a);
}

// ---------------------------------------------------------------------------
// fp32 activations on the tensor cores (S3 / S4, 5..16 activation columns)
// ---------------------------------------------------------------------------
static cudaError_t setup_fm_kernels(int max_smem) {
    const void *ks[6] = {reinterpret_cast<const void *>(&f32_mma_kernel<false, 1>),
                         reinterpret_cast<const void *>(&f32_mma_kernel<false, 2>),
                         reinterpret_cast<const void *>(&f32_mma_kernel<false, 4>),
                         reinterpret_cast<const void *>(&f32_mma_kernel<true, 1>),
                         reinterpret_cast<const void *>(&f32_mma_kernel<true, 2>),
                         reinterpret_cast<const void *>(&f32_mma_kernel<true, 4>)};
    for (const void *k : ks) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
static RegisterSetup g_reg_fm(setup_fm_kernels);

struct FmPlan {
    FmArgs a;
    int grid;  // CTAs (a multiple of a.split)
    size_t smem;
};

// One CTA per SM.  A tile is 128 output rows (SwiGLU: 64 outputs, their gate
// and up rows).  With at least as many tiles as SMs each cluster is one CTA
// walking a contiguous tile range; with fewer, every tile gets a cluster of up
// to 8 CTAs that split K between them: the largest split whose clusters all
// run at once (max_active_clusters of `kern`), else none.
static FmPlan plan_fm(int64_t rows_out, int64_t K, int64_t N, bool swiglu, int sms, const void *kern) {
    FmPlan p;
    FmArgs &a = p.a;
    a = FmArgs{};
    const int64_t B = K / 32;
    const int64_t tiles = ceil_div(rows_out, swiglu ? 64 : 128);
    a.M_out = (int)rows_out;
    a.N = (int)N;
    a.B = (int)B;
    a.tiles = (int)tiles;
    a.up_group0 = swiglu ? (int)(rows_out / kGroupRows) : 0;
    auto finish = [&](int64_t split) {
        const int64_t clusters = tiles < sms ? tiles : sms;
        const int64_t blocks = ceil_div(B, split);
        const int64_t per_cta = ceil_div(tiles, clusters) * ceil_div(blocks, kFmSB);
        a.split = (int)split;
        a.stages = (int)std::max<int64_t>(1, std::min<int64_t>(kFmMaxStages, per_cta));
        p.grid = (int)(clusters * split);
        p.smem = fm_smem_bytes(a.stages);
    };
    int64_t split = 1;
    if (tiles < sms) {
        split = std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(kFmMaxSplit, sms / tiles), B));
        for (; split > 1; --split) {
            finish(split);
            if (max_active_clusters(kern, kFmThreads, p.smem, (int)split) >= tiles) break;
        }
    }
    finish(split);
    return p;
}

static q8_status run_fm(const void *W, const float *x, float *y, int64_t rows_out, int64_t K,
                        int64_t N, bool swiglu, cudaStream_t stream, const float *res) {
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int64_t B = K / 32, C = K / 16;
    const int64_t units = ceil_div(rows_out, kGroupRows);
    const int64_t groups = swiglu ? 2 * units : units;
    using FmKernel = void (*)(CUtensorMap, CUtensorMap, const float *, FmArgs);
    // each epilogue warp takes 1 activation row up to N = 4, 2 up to N = 8, else 4
    const FmKernel k = swiglu ? (N <= 4 ? &f32_mma_kernel<true, 1> : N <= 8 ? &f32_mma_kernel<true, 2> : &f32_mma_kernel<true, 4>)
                              : (N <= 4 ? &f32_mma_kernel<false, 1> : N <= 8 ? &f32_mma_kernel<false, 2> : &f32_mma_kernel<false, 4>);
    FmPlan p = plan_fm(rows_out, K, N, swiglu, dev->sms, reinterpret_cast<const void *>(k));
    if (p.smem > (size_t)dev->max_smem_optin) return Q8_ERR_UNSUPPORTED;
    p.a.y = y;
    p.a.res = swiglu ? nullptr : res;
    const uint64_t gstride = (uint64_t)kGroupBytesPerBlock * B;
    const uint8_t *dbase = static_cast<const uint8_t *>(W) + 256 * B;
    CUtensorMap tq, td;
    // weights: [group][16-byte column][8 rows x 16 B], 8 groups x kFmCS columns a box
    Q8_CHECK(make_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, kColBytes, C, groups, kColBytes,
                         gstride, kColBytes, kFmCS, 8, true));
    // scales: [group][block][8 rows] fp16, 8 groups x kFmSB blocks a box
    Q8_CHECK(make_map_3d(&td, CU_TENSOR_MAP_DATA_TYPE_UINT16, dbase, 8, B, groups, 16, gstride, 8,
                         kFmSB, 8, true));
    // the activations are read by the kernel's splitter warps with plain loads
    return launch_pdl_cluster(k, dim3(p.grid), dim3(kFmThreads), p.smem, stream,
                              swiglu ? "q8_gate_up_swiglu (tensor cores) launch" : "q8_gemv (tensor cores) launch",
                              (unsigned)p.a.split, tq, td, x, p.a);
}

// ---------------------------------------------------------------------------
// grouped MoE (S6)
// ---------------------------------------------------------------------------
using MoeKernel = void (*)(MoeMaps, MoeArgs);

static MoeKernel moe_kernel_for(int nmax) {
    switch (nmax) {
        case 1: return &moe_fused_kernel<1>;
        case 2: return &moe_fused_kernel<2>;
        case 4: return &moe_fused_kernel<4>;
        case 8: return &moe_fused_kernel<8>;
        default: return &moe_fused_kernel<16>;
    }
}

static cudaError_t setup_moe_kernels(int max_smem) {
    const int nm[5] = {1, 2, 4, 8, 16};
    for (int i = 0; i < 5; ++i) {
        const void *k = reinterpret_cast<const void *>(moe_kernel_for(nm[i]));
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
static RegisterSetup g_reg_moe(setup_moe_kernels);

// K-quant tile kernel variants: (format, N, stages, CTAs per SM).  Two CTAs
// per SM (twice the warps to hide the dequantise-and-dot latency) wherever
// there are tiles for them; at N = 2 that leaves room for two-stage rings
// only, so matrices with fewer than two tiles per SM take one CTA per SM with
// deeper rings (measured: 152064x3584 N = 2 Q4_K 161 against 180 us, Q6_K 151
// against 179; 3584x18944 the other way round, 25.7 against 29.5).
#define Q8_KQ_VARIANTS(X) X(4, 1, 3, 2) X(4, 2, 4, 1) X(4, 2, 2, 2) X(6, 1, 2, 2) X(6, 2, 3, 1) X(6, 2, 2, 2)
static cudaError_t setup_q4k_kernels(int max_smem) {
    (void)max_smem;
#define Q8_KQ_SETUP(F, NM, ST, MB)                                                                             \
    {                                                                                                        \
        const void *k = reinterpret_cast<const void *>(&kq_tile_kernel<F, NM, ST, MB>);                      \
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,                 \
                                             kq_smem_bytes<F, NM, ST>());                                    \
        if (e != cudaSuccess) return e;                                                                      \
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,                          \
                                 cudaSharedmemCarveoutMaxShared);                                            \
        if (e != cudaSuccess) return e;                                                                      \
    }
    Q8_KQ_VARIANTS(Q8_KQ_SETUP)
#undef Q8_KQ_SETUP
    return cudaSuccess;
}
static RegisterSetup g_reg_q4k(setup_q4k_kernels);

struct MoePlan {
    MoeArgs a;
    size_t smem;
};

// Ring slots of the largest stage any tile of this token bucket has; as many
// as fit next to the barriers, the partial-sum buffers and the table.
static bool plan_moe(int64_t T, int max_smem, MoePlan &p) {
    MoeArgs &a = p.a;
    a = MoeArgs{};
    const int nmax = nmax_for(T);
    uint32_t slot = 0;
    int red_a = 0;
    for (int nx = 1; nx <= nmax; nx *= 2)
        for (int ph = 1; ph <= 2; ++ph) {
            slot = std::max(slot, moe_stage_bytes(ph, nx));
            red_a = std::max(red_a, moe_halves(ph) * moe_tg(ph, nx) * nx);
        }
    a.slot_bytes = (uint32_t)round_up(slot, 128);
    a.red_a = red_a;
    const size_t fixed = kMoeBarBytes + (size_t)kMoeRedBufs * 8 * red_a * 8 * 4 + sizeof(MoeTable) + 16;
    const int64_t stages = ((int64_t)max_smem - (int64_t)fixed) / a.slot_bytes;
    if (stages < 2) return false;
    a.stages = (int)std::min<int64_t>(stages, kMoeMaxStages);
    p.smem = (size_t)a.stages * a.slot_bytes + fixed;
    return true;
}

// workspace: counters | routed h | shared h | partial outputs
static size_t moe_ctr_bytes(int64_t H) { return (size_t)round_up((kCtrGroups + H / 8) * 4, 256); }
static size_t moe_hbuf_bytes(int64_t T, int64_t k, int64_t I) { return (size_t)round_up(T * k * I * 4, 256); }
static size_t moe_hsh_bytes(int64_t T, int64_t Is) { return (size_t)round_up(T * Is * 4, 256); }
// K chunks of the shared expert's down projection: about as long as a routed
// expert's K (at most kMoeMaxSplit chunks), an even number of 16-byte columns
// each (whole Q8_0 blocks)
static void moe_shared_chunks(int64_t I, int64_t Is, int &nsplit, int &cc) {
    if (Is <= 0) {
        nsplit = 0;
        cc = 0;
        return;
    }
    const int64_t C = Is / 16, n0 = std::min<int64_t>(ceil_div(Is, I), kMoeMaxSplit);
    cc = (int)round_up(ceil_div(C, n0), 2);
    nsplit = (int)ceil_div(C, cc);
}
// partial outputs: one row per (token, slot) pair, then one per (shared chunk, token)
static size_t moe_part_bytes(int64_t T, int64_t k, int64_t H, int64_t I, int64_t Is) {
    int nsplit, cc;
    moe_shared_chunks(I, Is, nsplit, cc);
    return (size_t)round_up((T * k + nsplit * T) * H * 4, 256);
}

// ---------------------------------------------------------------------------
// scratch for q8_moe_gemv_noalloc: a fixed array in the library's own device
// memory, so that call needs no buffer from the caller.  Each device that
// loads the library holds these bytes until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_moe_noalloc_scratch[kNoAllocScratchBytes];

// device address of the array, per device; written once under the mutex
// (release) and read without it (acquire)
static std::atomic<void *> g_moe_noalloc_addr[kMaxDevices];
static std::mutex g_moe_noalloc_mutex;

// The array's name is only a host-side stand-in; the address a kernel can use
// comes from cudaGetSymbolAddress, looked up once per device with that device
// current (the first call on each device does this).
static q8_status moe_noalloc_scratch(void **out) {
    int dev = 0;
    Q8_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice, "device index");
    void *p = g_moe_noalloc_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_moe_noalloc_mutex);
        p = g_moe_noalloc_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            cudaError_t e = cudaGetSymbolAddress(&p, g_moe_noalloc_scratch);
            if (e != cudaSuccess || p == nullptr)
                return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                                 "cudaGetSymbolAddress(moe scratch)");
            g_moe_noalloc_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return Q8_OK;
}

// Host-side checks of q8_moe_gemv's arguments other than its workspace, and
// its launch plan; nothing is enqueued.
static q8_status moe_check_args(const void *gate_up_experts, const void *down_experts,
                                const void *shared_gate_up, const void *shared_down, const int32_t *idx,
                                const float *w, const float *x, float *y, int64_t T, int64_t E, int64_t top_k,
                                int64_t H, int64_t I, int64_t I_shared, MoePlan &p) {
    if (T <= 0 || E <= 0 || top_k <= 0 || top_k > E || H <= 0 || I <= 0 || I_shared < 0)
        return Q8_ERR_SHAPE;
    if (H % 32 || I % 32 || I_shared % 32) return Q8_ERR_SHAPE;
    if (T > kMoeMaxT || top_k > kMoeMaxK || E > kMoeMaxE || H > 65536 || I > 65536 ||
        I_shared > 65536)
        return Q8_ERR_UNSUPPORTED;
    const bool has_shared = shared_gate_up != nullptr || shared_down != nullptr;
    if (has_shared != (I_shared > 0) || (has_shared && (!shared_gate_up || !shared_down)))
        return Q8_ERR_INVALID;
    Q8_CHECK(check_device_ptr(gate_up_experts));
    Q8_CHECK(check_device_ptr(down_experts));
    if (has_shared) {
        Q8_CHECK(check_device_ptr(shared_gate_up));
        Q8_CHECK(check_device_ptr(shared_down));
    }
    Q8_CHECK(check_device_ptr(idx, false));
    Q8_CHECK(check_device_ptr(w, false));
    if ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(w)) & 3u) return Q8_ERR_ALIGN;
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(y));
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    if (!plan_moe(T, dev->max_smem_optin, p)) return Q8_ERR_UNSUPPORTED;
    return Q8_OK;
}

// Encodes the tensor maps and launches the MoE kernel (arguments checked).
static q8_status moe_launch(MoePlan &p, const void *gate_up_experts, const void *down_experts,
                            const void *shared_gate_up, const void *shared_down, const int32_t *idx,
                            const float *w, const float *x, float *y, int64_t T, int64_t E, int64_t top_k,
                            int64_t H, int64_t I, int64_t I_shared, void *workspace, cudaStream_t stream) {
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const bool has_shared = shared_gate_up != nullptr;
    MoeArgs &a = p.a;
    const int64_t Ish = has_shared ? I_shared : 0;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    a.T = (int)T; a.E = (int)E; a.k = (int)top_k; a.H = (int)H; a.I = (int)I; a.Is = (int)Ish;
    moe_shared_chunks(I, Ish, a.nsplit, a.cc);
    a.idx = idx;
    a.w = w;
    a.y = y;
    a.ctr = reinterpret_cast<unsigned *>(ws);
    a.hbuf = reinterpret_cast<float *>(ws + moe_ctr_bytes(H));
    a.hsh = reinterpret_cast<float *>(ws + moe_ctr_bytes(H) + moe_hbuf_bytes(T, top_k, I));
    a.part = reinterpret_cast<float *>(ws + moe_ctr_bytes(H) + moe_hbuf_bytes(T, top_k, I) +
                                       moe_hsh_bytes(T, I_shared));

    // Weight maps: [16-byte column][8 rows x 16 B] q boxes and [block][8 rows]
    // fp16 scale boxes of 1, 2, 4 or 8 consecutive packed groups (the tile
    // kernels' layout).  Activation maps: [row][column][16 fp32], one row per
    // box, or all T rows for the shared expert's segment.
    MoeMaps m;
    const uint8_t *gu = static_cast<const uint8_t *>(gate_up_experts);
    const uint8_t *dn = static_cast<const uint8_t *>(down_experts);
    // weight maps of every box depth (see moe.cuh): [phase][routed|shared][q|scales][depth]
    auto weight_maps = [&](CUtensorMap(&w)[2][kMoeDepths], const uint8_t *base, int64_t K, int64_t groups)
        -> q8_status {
        const uint64_t gs = (uint64_t)kGroupBytesPerBlock * (K / 32);
        for (int d = 0; d < kMoeDepths; ++d) {
            Q8_CHECK(make_map_3d(&w[0][d], CU_TENSOR_MAP_DATA_TYPE_UINT8, base, kColBytes, K / 16, groups,
                                 kColBytes, gs, kColBytes, kMoeCS, 1u << d, true));
            Q8_CHECK(make_map_3d(&w[1][d], CU_TENSOR_MAP_DATA_TYPE_UINT16, base + 256 * (K / 32), 8, K / 32,
                                 groups, 16, gs, 8, kMoeCS / 2, 1u << d, true));
        }
        return Q8_OK;
    };
    Q8_CHECK(weight_maps(m.w[0][0], gu, H, E * (2 * I / 8)));
    Q8_CHECK(weight_maps(m.w[1][0], dn, I, E * (H / 8)));
    Q8_CHECK(make_map_3d(&m.x1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, x, 16, H / 16, T, 64, (uint64_t)H * 4, 16, kMoeCS,
                         1, false));
    Q8_CHECK(make_map_3d(&m.x1s, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, x, 16, H / 16, T, 64, (uint64_t)H * 4, 16, kMoeCS,
                         (uint32_t)T, false));
    Q8_CHECK(make_map_3d(&m.h2r, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.hbuf, 16, I / 16, T * top_k, 64,
                         (uint64_t)I * 4, 16, kMoeCS, 1, false));
    if (has_shared) {
        const uint8_t *sgu = static_cast<const uint8_t *>(shared_gate_up);
        const uint8_t *sdn = static_cast<const uint8_t *>(shared_down);
        Q8_CHECK(weight_maps(m.w[0][1], sgu, H, 2 * Ish / 8));
        Q8_CHECK(weight_maps(m.w[1][1], sdn, Ish, H / 8));
        Q8_CHECK(make_map_3d(&m.h2s, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.hsh, 16, Ish / 16, T, 64,
                             (uint64_t)Ish * 4, 16, kMoeCS, (uint32_t)T, false));
    } else {
        for (int ph = 0; ph < 2; ++ph)
            for (int qd = 0; qd < 2; ++qd)
                for (int d = 0; d < kMoeDepths; ++d) m.w[ph][1][qd][d] = m.w[ph][0][qd][d];
        m.h2s = m.h2r;
    }
    return launch_pdl(moe_kernel_for(nmax_for(T)), dim3((unsigned)dev->sms), dim3(moe_threads(nmax_for(T))), p.smem,
                      stream, "q8_moe_gemv launch", m, a);
}

// One launch of the K-quant tile kernel (kquant.cuh) for N <= 2: a CTA per
// 32-row tile, at most MINB per SM.
template <int FMT, int NM, int ST, int MB>
static q8_status launch_kq_tile(const CUtensorMap &map, const uint8_t *w8, const float *x, float *y, int64_t M,
                                int64_t K, int N, int sms, cudaStream_t stream, const char *name) {
    const int64_t tiles = ceil_div(M, kKqRows);
    const unsigned g = (unsigned)std::min<int64_t>(tiles, (int64_t)sms * MB);
    return launch_pdl(kq_tile_kernel<FMT, NM, ST, MB>, dim3(g), dim3(kKqTileThreads),
                      (size_t)kq_smem_bytes<FMT, NM, ST>(), stream, name, map, w8, x, y, (int)M, (int)K, N);
}

// K-quant argument checks shared by the entry points.
static q8_status kquant_check(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                              bool w_aligned) {
    if (M <= 0 || K <= 0 || N <= 0 || K % 256) return Q8_ERR_SHAPE;
    if (N > 4 || M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W, w_aligned));
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(y, false));
    if (reinterpret_cast<uintptr_t>(y) & 3u) return Q8_ERR_ALIGN;
    return Q8_OK;
}

template <int FMT>
// K-quant GEMV on raw blocks: argument checks, then the tile kernel (Q4_K)
// or one warp per row (Q6_K on raw blocks).
static q8_status run_kquant(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                            cudaStream_t stream, const char *name) {
    Q8_CHECK(kquant_check(W, x, y, M, K, N, FMT == 4));  // Q4_K blocks are read as aligned words / TMA boxes
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const int nm = (int)N;
    const uint8_t *w8 = static_cast<const uint8_t *>(W);
    if constexpr (FMT == 4) {
        // raw rows of 144 * SB bytes: boxes of {one 144-byte block, 32 rows};
        // activation rows two per launch
        const int64_t SB = K / 256;
        CUtensorMap map;
        const q8_status ms =
            make_map_3d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, 144, SB, M, 144, 144 * SB, 144, 1, kKqRows, true);
        if (ms != Q8_OK) return ms;
        const bool many = ceil_div(M, kKqRows) >= 2 * (int64_t)dev->sms;
        for (int64_t n0 = 0; n0 < N; n0 += 2) {
            const int nn = (int)std::min<int64_t>(2, N - n0);
            const float *xn = x + n0 * K;
            float *yn = y + n0 * M;
            const q8_status st =
                nn == 1 ? launch_kq_tile<4, 1, 3, 2>(map, w8, xn, yn, M, K, 1, dev->sms, stream, name)
                : many  ? launch_kq_tile<4, 2, 2, 2>(map, w8, xn, yn, M, K, 2, dev->sms, stream, name)
                        : launch_kq_tile<4, 2, 4, 1>(map, w8, xn, yn, M, K, 2, dev->sms, stream, name);
            if (st != Q8_OK) return st;
        }
        return Q8_OK;
    } else {
        const int64_t warps = std::min<int64_t>(M, (int64_t)dev->sms * 64);
        const unsigned grid = (unsigned)ceil_div(warps, kKqThreads / 32);
        switch (nmax_for(N)) {
            case 1: return launch_pdl(q6k_row_kernel<1>, dim3(grid), dim3(kKqThreads), 0, stream, name, w8, x, y, (int)M, (int)K, nm);
            case 2: return launch_pdl(q6k_row_kernel<2>, dim3(grid), dim3(kKqThreads), 0, stream, name, w8, x, y, (int)M, (int)K, nm);
            default: return launch_pdl(q6k_row_kernel<4>, dim3(grid), dim3(kKqThreads), 0, stream, name, w8, x, y, (int)M, (int)K, nm);
        }
    }
}

// Q6_K on the packed units: the tile kernel, activation rows two at a time.
static q8_status run_q6k_packed(const void *P, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                                cudaStream_t stream) {
    Q8_CHECK(kquant_check(P, x, y, M, K, N, true));
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const char *name = "q8_q6k_gemv_packed launch";
    const uint8_t *w8 = static_cast<const uint8_t *>(P);
    CUtensorMap unused;
    std::memset(&unused, 0, sizeof(unused));
    const bool many = ceil_div(M, kKqRows) >= 2 * (int64_t)dev->sms;
    for (int64_t n0 = 0; n0 < N; n0 += 2) {
        const int nm = (int)std::min<int64_t>(2, N - n0);
        const float *xn = x + n0 * K;
        float *yn = y + n0 * M;
        const q8_status st = nm == 1 ? launch_kq_tile<6, 1, 2, 2>(unused, w8, xn, yn, M, K, 1, dev->sms, stream, name)
                             : many  ? launch_kq_tile<6, 2, 2, 2>(unused, w8, xn, yn, M, K, 2, dev->sms, stream, name)
                                     : launch_kq_tile<6, 2, 3, 1>(unused, w8, xn, yn, M, K, 2, dev->sms, stream, name);
        if (st != Q8_OK) return st;
    }
    return Q8_OK;
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

q8_status q8_gemv_split(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                        q8_stream_t stream) {
    if (M <= 0 || K <= 0 || N <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > 16 || M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(y));
    return run_tile(W, x, nullptr, y, M, K, N, kModeF32, (cudaStream_t)stream, nullptr, nullptr, true);
}

q8_status q8_q4k_gemv(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                      q8_stream_t stream) {
    return run_kquant<4>(W, x, y, M, K, N, (cudaStream_t)stream, "q8_q4k_gemv launch");
}

q8_status q8_q6k_gemv(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                      q8_stream_t stream) {
    return run_kquant<6>(W, x, y, M, K, N, (cudaStream_t)stream, "q8_q6k_gemv launch");
}

size_t q8_q6k_packed_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0 || K % 256) return 0;
    return (size_t)ceil_div(M, kKqRows) * (size_t)(K / 256) * kQ6UnitBytes;
}

q8_status q8_q6k_pack_weights(const void *raw, int64_t M, int64_t K, void *packed, q8_stream_t stream) {
    if (M <= 0 || K <= 0 || K % 256) return Q8_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(raw, false));
    Q8_CHECK(check_device_ptr(packed));
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const long long pieces = (long long)(q8_q6k_packed_bytes(M, K) / 16);
    const unsigned grid = (unsigned)std::min<long long>((pieces + 255) / 256, (long long)dev->sms * 16);
    return launch_pdl(q6k_pack_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, "q8_q6k_pack_weights launch",
                      static_cast<const uint8_t *>(raw), static_cast<uint8_t *>(packed), (int)M, (int)(K / 256),
                      pieces);
}

q8_status q8_q6k_unpack_weights(const void *packed, int64_t M, int64_t K, void *raw, q8_stream_t stream) {
    if (M <= 0 || K <= 0 || K % 256) return Q8_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(packed));
    Q8_CHECK(check_device_ptr(raw, false));
    const DeviceInfo *dev = nullptr;
    Q8_CHECK(device_info(&dev));
    const long long bytes = (long long)M * (K / 256) * 210;
    const unsigned grid = (unsigned)std::min<long long>((bytes + 255) / 256, (long long)dev->sms * 16);
    return launch_pdl(q6k_unpack_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream,
                      "q8_q6k_unpack_weights launch", static_cast<const uint8_t *>(packed),
                      static_cast<uint8_t *>(raw), (int)M, (int)(K / 256), bytes);
}

q8_status q8_q6k_gemv_packed(const void *packed, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                             q8_stream_t stream) {
    return run_q6k_packed(packed, x, y, M, K, N, (cudaStream_t)stream);
}

q8_status q8_gemv_residual(const void *W, const float *x, const float *residual, float *y, int64_t M,
                           int64_t K, int64_t N, q8_stream_t stream) {
    if (M <= 0 || K <= 0 || N <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > 16 || M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(y));
    Q8_CHECK(check_device_ptr(residual, false));
    if (reinterpret_cast<uintptr_t>(residual) & 3u) return Q8_ERR_ALIGN;
    // residual == y is the in-place update; any other overlap is undefined
    return run_tile(W, x, nullptr, y, M, K, N, kModeF32, (cudaStream_t)stream, nullptr, residual);
}

q8_status q8_gemv_argmax(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                         uint64_t *best, q8_stream_t stream) {
    if (M <= 0 || K <= 0 || N <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > 4 || M > (int64_t)1 << 30 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(x));
    if (y) Q8_CHECK(check_device_ptr(y));
    Q8_CHECK(check_device_ptr(best, false));
    if (reinterpret_cast<uintptr_t>(best) & 7u) return Q8_ERR_ALIGN;
    // the GEMV's CTAs combine their keys with atomicMax, starting from zero
    Q8_CHECK(launch_pdl(clear_keys_kernel, dim3(1), dim3(32), 0, (cudaStream_t)stream,
                        "q8_gemv_argmax clear launch", reinterpret_cast<unsigned long long *>(best),
                        (int)N));
    return run_tile(W, x, nullptr, y, M, K, N, kModeF32, (cudaStream_t)stream,
                    reinterpret_cast<unsigned long long *>(best));
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

q8_status q8_gate_up_swiglu_split(const void *W, const float *x, float *h, int64_t I, int64_t K,
                                  int64_t N, q8_stream_t stream) {
    if (I <= 0 || K <= 0 || N <= 0 || K % 32 || I % 8) return Q8_ERR_SHAPE;
    if (N > 16 || I > (int64_t)1 << 29 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(W));
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(h));
    return run_tile(W, x, nullptr, h, I, K, N, kModeSwiGLU, (cudaStream_t)stream, nullptr, nullptr, true);
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
    // a warp per 32-block, 8 warps a CTA
    const int64_t blocks = std::min<int64_t>(ceil_div(N * (K / 32), 8), (int64_t)dev->sms * 8);
    return launch_pdl(quantize_act_kernel, dim3((unsigned)blocks), dim3(256), 0,
                      (cudaStream_t)stream, "q8_quantize_act launch", x, xq, xd, N, K);
}

q8_status q8_rmsnorm_quantize_act(const float *x, const float *gamma, float eps, int8_t *xq,
                                  uint16_t *xd, float *rinv, int64_t N, int64_t K, q8_stream_t stream) {
    if (N <= 0 || K <= 0 || K % 32) return Q8_ERR_SHAPE;
    if (N > (int64_t)1 << 20 || K > (int64_t)1 << 24) return Q8_ERR_UNSUPPORTED;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return Q8_ERR_INVALID;  // negative, NaN or infinite
    Q8_CHECK(check_device_ptr(x));
    Q8_CHECK(check_device_ptr(gamma, false));
    Q8_CHECK(check_device_ptr(xq, false));
    Q8_CHECK(check_device_ptr(xd, false));
    if ((reinterpret_cast<uintptr_t>(gamma) & 3u) || (reinterpret_cast<uintptr_t>(xd) & 1u))
        return Q8_ERR_ALIGN;
    if (rinv) {
        Q8_CHECK(check_device_ptr(rinv, false));
        if (reinterpret_cast<uintptr_t>(rinv) & 3u) return Q8_ERR_ALIGN;
    }
    return launch_pdl(rmsnorm_quantize_kernel, dim3((unsigned)N), dim3(kRmsThreads), 0,
                      (cudaStream_t)stream, "q8_rmsnorm_quantize_act launch", x, gamma, eps, xq, xd,
                      rinv, K);
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
    if (N >= kMmaMinN) return run_mma(W, xq, xd, y, M, K, N, (cudaStream_t)stream);
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
    if (T <= 0 || E <= 0 || top_k <= 0 || H <= 0 || I <= 0 || I_shared < 0) return 0;
    return moe_ctr_bytes(H) + moe_hbuf_bytes(T, top_k, I) + moe_hsh_bytes(T, I_shared) +
           moe_part_bytes(T, top_k, H, I, I_shared);
}

q8_status q8_moe_workspace_init(void *workspace, size_t workspace_bytes, q8_stream_t stream) {
    if (workspace_bytes == 0) return Q8_ERR_SHAPE;
    Q8_CHECK(check_device_ptr(workspace));
    Q8_CUDA_TRY(cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream));
    return Q8_OK;
}

q8_status q8_moe_gemv(const void *gate_up_experts, const void *down_experts,
                      const void *shared_gate_up, const void *shared_down,
                      const int32_t *idx, const float *w, const float *x, float *y, int64_t T,
                      int64_t E, int64_t top_k, int64_t H, int64_t I, int64_t I_shared,
                      void *workspace, size_t workspace_bytes, q8_stream_t stream) {
    MoePlan p;
    Q8_CHECK(moe_check_args(gate_up_experts, down_experts, shared_gate_up, shared_down, idx, w, x, y, T, E,
                            top_k, H, I, I_shared, p));
    Q8_CHECK(check_device_ptr(workspace));
    if (workspace_bytes < q8_moe_workspace_bytes(T, E, top_k, H, I, I_shared)) return Q8_ERR_SHAPE;
    return moe_launch(p, gate_up_experts, down_experts, shared_gate_up, shared_down, idx, w, x, y, T, E, top_k,
                      H, I, I_shared, workspace, (cudaStream_t)stream);
}

q8_status q8_moe_gemv_noalloc(const void *gate_up_experts, const void *down_experts,
                              const void *shared_gate_up, const void *shared_down,
                              const int32_t *idx, const float *w, const float *x, float *y,
                              int64_t T, int64_t E, int64_t top_k, int64_t H, int64_t I,
                              int64_t I_shared, q8_stream_t stream) {
    const size_t need = q8_moe_workspace_bytes(T, E, top_k, H, I, I_shared);
    if (need == 0) return Q8_ERR_SHAPE;
    if (need > kNoAllocScratchBytes) {
        snprintf(last_error_buf(), 256,
                 "q8_moe_gemv_noalloc: these sizes need %zu bytes of scratch; the built-in "
                 "scratch holds %zu",
                 need, kNoAllocScratchBytes);
        return Q8_ERR_UNSUPPORTED;
    }
    // every argument is checked before anything is enqueued
    MoePlan p;
    Q8_CHECK(moe_check_args(gate_up_experts, down_experts, shared_gate_up, shared_down, idx, w, x, y, T, E,
                            top_k, H, I, I_shared, p));
    void *scratch = nullptr;
    Q8_CHECK(moe_noalloc_scratch(&scratch));
    // The array keeps whatever the previous call left in it; the MoE kernel
    // needs its counters at zero when its dependency wait returns.  A one-warp
    // kernel of the dependent-launch chain clears them (a memset node there
    // would stop the MoE kernel from starting early and prefetching weights).
    const int words = (int)(moe_ctr_bytes(H) / 4);
    Q8_CHECK(launch_pdl(clear_words_kernel, dim3(1), dim3(32), 0, (cudaStream_t)stream,
                        "q8_moe_gemv_noalloc clear launch", static_cast<unsigned *>(scratch), words));
    return moe_launch(p, gate_up_experts, down_experts, shared_gate_up, shared_down, idx, w, x, y, T, E, top_k,
                      H, I, I_shared, scratch, (cudaStream_t)stream);
}

q8_status q8_test_wait_timeout(uint32_t limit_us, int32_t *out, q8_stream_t stream) {
    if (limit_us == 0 || limit_us > 1000000u) return Q8_ERR_UNSUPPORTED;
    Q8_CHECK(check_device_ptr(out, false));
    if (reinterpret_cast<uintptr_t>(out) & 3u) return Q8_ERR_ALIGN;
    return launch_pdl(wait_timeout_kernel, dim3(1), dim3(kSelftestThreads), 0, (cudaStream_t)stream,
                      "q8_test_wait_timeout launch", (uint64_t)limit_us * 1000ull, reinterpret_cast<int *>(out));
}

}  // extern "C"
