// f32_mma.cuh -- S3 / S4 on the tensor cores: Q8_0 weights times fp32
// activations for 5..16 activation columns (small-batch GEMM and the fused
// gate_up + SwiGLU), where the CUDA cores' FMA issue, not HBM, would bound the
// product.
//
// The packed weight bytes are the A operand of tcgen05.mma kind::i8 exactly as
// they land from TMA (the layout is the MMA's K-major core-matrix order, see
// q8q8_mma.cuh).  The fp32 activations are made integer in shared memory: per
// activation row n and 32-block b, with amax the block's largest |x| and s the
// power of two with amax / s in [32, 64) (read off amax's exponent),
//     v0 = x / s (exact),  q0 = rint(v0),  v1 = (v0 - q0) * 254,  q1 = rint(v1),
//     v2 = (v1 - q1) * 254,  q2 = rint(v2),
// so x = s * (q0 + q1 / 254 + q2 / 254^2) up to s * (0.5 / 254^2 + 2^-25),
// below 2.5e-7 of amax.  |q0| <= 64 and |q1|, |q2| <= 127: every piece is an
// int8.  A power-of-two s keeps the split exact under scaling: x -> 2x gives
// the same pieces and twice s, and unit-scale one-hot inputs come out exactly.
// The three pieces are stacked along the MMA's N
// (rows 16 k + n of the B operand), so one kind::i8 MMA per Q8_0 block gives
// the three exact int32 dots D_k = sum_i q_w,i * q_k,i of all activation rows
// at once, and the epilogue adds
//     d_w * s * (D_0 + D_1 / 254 + D_2 / 254^2)
// into fp32 accumulators.  Each Q8_0 block needs its own weight scale d_w, so
// one MMA per block, as in the integer path.  (The weights are the raw GGUF
// Q8_0 blocks of the "skuznetsov/cogni-ml" README's Q8_0 GEMV probe, "Build
// Qwen CLIs", w = d * q per 32-block; the per-block int8 dot followed by the
// scales is the activation-quantised dot of "Add Qwen1.5-MoE Q8_0 ... - #144",
// "Key implementation notes", here with an exact three-term split of x in
// place of the one-term Q8_0 rounding, so the result keeps fp32 accuracy.)
//
// Activation blocks whose largest magnitude is below 2^-121 are scaled as if
// it were 2^-121 and lose relative accuracy (fp32 subnormal territory).
// Non-finite activations give undefined outputs.
//
// Operands and tensor memory:
//   * A = 128 weight rows (16 packed groups) x 32 bytes per block: two TMA
//     boxes of 8 groups per stage.  For the fused SwiGLU a tile is 64 gate
//     rows (groups 8t ..) and the matching 64 up rows (groups I/8 + 8t ..), so
//     TMEM lanes 0..63 hold g and lanes 64..127 hold u of the same outputs;
//   * B = 48 rows (3 pieces x 16 activation rows, rows past N never read) x
//     32 bytes per block, [column][48 rows][16 B] with a column stride of
//     784 B (768 + 16: the splitters' 8-byte stores then spread over all
//     banks);
//   * D = 128 lanes x 48 int32 columns per block, block j at TMEM column
//     64 j (512 columns for a stage of 8 blocks); the MMA fills one half
//     stage (4 blocks) while the epilogue reads the other.
// The stored bytes are q + 128 (A read as unsigned), so D_k carries
// 128 * sum_i q_k,i; the epilogue removes it exactly inside its int -> float
// conversion (add the correction to the bits of 1.5 * 2^23, subtract
// 1.5 * 2^23 as a float: exact for |D| < 2^22; |D_k| <= 32 * 255 * 127).
//
// Pipeline: the TMA ring carries weights only (q and d, 34 KB a stage, up to
// 5 stages), so HBM sees up to 170 KB in flight per SM.  Eight splitter warps
// read the activations from L2 straight into registers (one stage ahead),
// split them and write the int8 pieces and the table into a ring of three
// activation buffers, running ahead of the MMAs.  Warps: 0 issues TMA (weight
// boxes of the first stages before griddepcontrol.wait), 1 owns tensor memory
// and issues the MMAs, 2..9 split (warp 2 + i takes activation rows i and
// i + 8), 10..25 are the epilogue: warp w reads TMEM lanes 32 * (w % 4) .. and
// TOK activation rows from TOK * ((w - 10) / 4) (TOK = 1 for N <= 4, 2 for
// N <= 8, else 4),
// so the epilogue's work spreads over 16 warps at any N, and no epilogue warp
// waits for a split.  With fewer 128-row tiles than
// SMs, K is split over a cluster of up to 8 CTAs and the partial sums meet in
// the leader in rank order (bit-identical results from run to run).
// Every wait is bounded; a stalled pipeline records an error, waits for its
// copies and MMAs in flight, frees its tensor memory and exits.
#pragma once

#include "q8q8_mma.cuh"

namespace q8 {

constexpr int kFmN = 16;                          // activation rows per piece (N <= 16)
constexpr int kFmPieces = 3;                      // int8 terms per activation
constexpr int kFmMmaN = kFmPieces * kFmN;         // MMA N = 48
constexpr int kFmCS = 16;                         // 16-byte columns per stage
constexpr int kFmSB = kFmCS / 2;                  // blocks per stage (8)
constexpr int kFmHalfBlocks = 4;                  // blocks per TMEM half
constexpr int kFmHalves = kFmSB / kFmHalfBlocks;  // 2
constexpr uint32_t kFmBlockCols = 64;             // TMEM columns per block (48 used)
constexpr uint32_t kFmTmemCols = kFmSB * kFmBlockCols;  // 512
constexpr int kFmSplitWarps = 8;
constexpr int kFmEpiWarps = 16;
constexpr int kFmEpiThreads = kFmEpiWarps * 32;
constexpr int kFmThreads = 64 + 32 * kFmSplitWarps + kFmEpiThreads;  // producer, MMA, splitters, epilogue
constexpr int kFmNB = 3;                          // activation buffers (pieces + table)
constexpr int kFmMaxSplit = 8;

constexpr uint32_t kFmXbColStride = kFmMmaN * 16 + 16;           // 784 B
constexpr uint32_t kFmQBytes = 16 * kFmCS * kColBytes;           // 32 KB (two 8-group boxes)
constexpr uint32_t kFmQBox = 8 * kFmCS * kColBytes;              // 16 KB
constexpr uint32_t kFmDBytes = 16 * kFmSB * 16;                  // 2 KB
constexpr uint32_t kFmDBox = 8 * kFmSB * 16;                     // 1 KB
constexpr uint32_t kFmDOff = kFmQBytes;
constexpr uint32_t kFmStageBytes = kFmQBytes + kFmDBytes;        // weight ring stage, 34 KB
constexpr uint32_t kFmXbBytes = kFmCS * kFmXbColStride;          // 12544 B of int8 pieces
constexpr uint32_t kFmTabBytes = kFmSB * kFmN * 16;              // 2 KB
constexpr uint32_t kFmTabOff = (kFmXbBytes + 127) / 128 * 128;   // within an activation buffer
constexpr uint32_t kFmActBytes = (kFmTabOff + kFmTabBytes + 127) / 128 * 128;
constexpr uint32_t kFmRedBytes = kFmN * 128 * 4;                 // one tile's partials
constexpr int kFmMaxStages = 5;

static_assert(kFmStageBytes % 128 == 0 && kFmActBytes % 128 == 0, "stage layout");

// Shared memory: weight stages | kFmNB activation buffers | barriers | partials | misc.
__host__ __device__ constexpr uint32_t fm_act_off(int stages) { return stages * kFmStageBytes; }
__host__ __device__ constexpr uint32_t fm_bar_off(int stages) { return fm_act_off(stages) + kFmNB * kFmActBytes; }
__host__ __device__ constexpr uint32_t fm_nbars(int stages) { return 2 * stages + 2 * kFmNB + 2 * kFmHalves + 3; }
__host__ __device__ constexpr uint32_t fm_red_off(int stages) {
    return (fm_bar_off(stages) + 8 * fm_nbars(stages) + 127) / 128 * 128;
}
__host__ __device__ constexpr uint32_t fm_misc_off(int stages) { return fm_red_off(stages) + kFmRedBytes; }
__host__ __device__ constexpr uint32_t fm_smem_bytes(int stages) { return fm_misc_off(stages) + 16; }

// Instruction descriptor: D s32, A unsigned 8-bit, B signed 8-bit, both
// K-major, N = 48, M = 128 (PTX ISA, tcgen05 instruction descriptor table).
constexpr uint32_t kFmIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kFmMmaN >> 3) << 17) |
                              ((uint32_t)(128 >> 4) << 24);

struct FmArgs {
    float *y;       // [N][M_out]
    int M_out;      // output rows (GEMV: M; SwiGLU: I)
    int N, B;       // activation rows, blocks per row
    int tiles;      // GEMV: ceil(groups / 16); SwiGLU: ceil(I / 64)
    int split;      // CTAs per cluster (K split)
    int stages;
    int up_group0;  // SwiGLU: packed group of the first up row (I / 8)
    const float *res;  // GEMV: [N][M_out] added to the outputs (q8_gemv_residual; may be y), or null
};

// The low byte of four words, in order, as one word.
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

// Activations of one stage for lane l of the splitter warp of row n: values
// 8 (l & 3) .. + 7 of block l >> 2, read from global memory (L2) into
// registers; zeros past the end of the CTA's K range (nb blocks in the stage)
// or past N.
__device__ __forceinline__ void fm_load_x(const float *__restrict__ x, int K, int n, int N, int b0, int nb,
                                          int lane, uint4 (&xr)[2]) {
    const int j = lane >> 2, qq = lane & 3;
    xr[0] = make_uint4(0, 0, 0, 0);
    xr[1] = make_uint4(0, 0, 0, 0);
    if (n < N && j < nb) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)n * K + 32 * (b0 + j) + 8 * qq);
        xr[0] = __ldg(src);
        xr[1] = __ldg(src + 1);
    }
}

// Split activation row n of one stage (its values in xr, see fm_load_x) into
// its three int8 pieces (the B operand) and the table entry (s, corrections)
// of each block, in activation buffer ab.  The four lanes of a block meet in
// shuffles.  Blocks past the end of the CTA's K range (j >= nb) are skipped.
__device__ __forceinline__ void fm_split_row(uint8_t *ab, const uint4 (&xr)[2], int n, int lane, int nb) {
    const int j = lane >> 2, qq = lane & 3;
    const uint64_t xv[4] = {pack_u32x2(xr[0].x, xr[0].y), pack_u32x2(xr[0].z, xr[0].w),
                            pack_u32x2(xr[1].x, xr[1].y), pack_u32x2(xr[1].z, xr[1].w)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = unpack_f32x2(xv[i]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    // amax in [2^(e-127), 2^(e-126)) for its biased exponent e: inv = 2^(132-e)
    // puts |x| * inv below 64, s = 1 / inv; e >= 6 keeps both normal
    const uint32_t e = max((__float_as_uint(amax) >> 23) & 0xFFu, 6u);
    const float s = __uint_as_float((e - 5u) << 23);
    const uint32_t ui = (259u - e) << 23, um = __float_as_uint(12582912.0f);  // inv; 1.5 * 2^23
    const uint64_t inv2 = pack_u32x2(ui, ui), m2 = pack_u32x2(um, um);
    const uint32_t un = __float_as_uint(-12582912.0f), u254 = __float_as_uint(254.0f);
    const uint64_t nm2 = pack_u32x2(un, un), r2 = pack_u32x2(u254, u254);
    uint32_t tb[3][8];  // float bits of v_k + 1.5 * 2^23: the low byte is rint(v_k)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint64_t v = mul_f32x2(xv[i], inv2);
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const uint64_t t = add_f32x2(v, m2);
            const float2 tf = unpack_f32x2(t);
            tb[k][2 * i] = __float_as_uint(tf.x);
            tb[k][2 * i + 1] = __float_as_uint(tf.y);
            if (k < 2) {
                const uint64_t qf = add_f32x2(t, nm2);                          // rint(v), exact
                const uint64_t rem = add_f32x2(v, qf ^ 0x8000000080000000ull);  // v - rint(v), exact
                v = mul_f32x2(rem, r2);
            }
        }
    }
    int sum[3];
    uint2 words[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        words[k].x = low_bytes4(tb[k][0], tb[k][1], tb[k][2], tb[k][3]);
        words[k].y = low_bytes4(tb[k][4], tb[k][5], tb[k][6], tb[k][7]);
        int sk = 0;
        asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(sk) : "r"(words[k].x), "r"(0x01010101));
        asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(sk) : "r"(words[k].y), "r"(0x01010101));
        sk += __shfl_xor_sync(0xffffffffu, sk, 1);
        sk += __shfl_xor_sync(0xffffffffu, sk, 2);
        sum[k] = sk;
    }
    if (j < nb) {
        uint8_t *xb = ab + (2 * j + (qq >> 1)) * kFmXbColStride + n * 16 + (qq & 1) * 8;
#pragma unroll
        for (int k = 0; k < 3; ++k) *reinterpret_cast<uint2 *>(xb + k * (kFmN * 16)) = words[k];
        if (qq == 0) {
            uint4 ent;
            ent.x = __float_as_uint(s);
            ent.y = 0x4B400000u - 128u * (uint32_t)sum[0];
            ent.z = 0x4B400000u - 128u * (uint32_t)sum[1];
            ent.w = 0x4B400000u - 128u * (uint32_t)sum[2];
            *reinterpret_cast<uint4 *>(ab + kFmTabOff + (j * kFmN + n) * 16) = ent;
        }
    }
}

// Epilogue of LB blocks of a stage for one thread (one weight row) and TOK
// activation rows: acc += d_w * s * (D0 + D1 / 254 + D2 / 254^2), with the
// three TMEM dots in v and (s, corrections) from the activation buffer's
// table.  FULL: every block of the batch is inside the K range.
template <bool FULL, int TOK, int LB>
__device__ __forceinline__ void fm_epilogue_blocks(float (&acc)[TOK], const uint32_t (&v)[LB][kFmPieces][TOK],
                                                   int jb, int nb, const uint8_t *st, const uint8_t *ab, int g, int r,
                                                   int n0) {
#pragma unroll
    for (int jj = 0; jj < LB; ++jj) {
        const int j = jb + jj;
        if (!FULL && j >= nb) break;
        const float dw = __half2float(*reinterpret_cast<const __half *>(st + kFmDOff + (g * kFmSB + j) * 16 + r * 2));
        const uint4 *tab = reinterpret_cast<const uint4 *>(ab + kFmTabOff + (j * kFmN + n0) * 16);
#pragma unroll
        for (int t = 0; t < TOK; ++t) {
            const uint4 e = tab[t];
            const float f0 = __uint_as_float(v[jj][0][t] + e.y) - 12582912.0f;
            const float f1 = __uint_as_float(v[jj][1][t] + e.z) - 12582912.0f;
            const float f2 = __uint_as_float(v[jj][2][t] + e.w) - 12582912.0f;
            const float c = fmaf(f2, 1.0f / 64516.0f, fmaf(f1, 1.0f / 254.0f, f0));
            acc[t] = fmaf(c, dw * __uint_as_float(e.x), acc[t]);
        }
    }
}

// TOK: activation rows per epilogue warp (1 for N <= 4, 2 for N <= 8, else 4).
template <bool SWIGLU, int TOK>
__global__ void __launch_bounds__(kFmThreads, 1)
    f32_mma_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap td,
                   const float *__restrict__ x, const FmArgs a) {
    constexpr int LB = TOK == 1 ? 4 : 8 / TOK;  // blocks per TMEM load batch (at most 24 registers)
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.split;
    uint8_t *act = smem + fm_act_off(a.stages);
    const uint32_t full0 = smem_u32(smem + fm_bar_off(a.stages));
    const uint32_t empty0 = full0 + 8 * a.stages;
    const uint32_t bready0 = empty0 + 8 * a.stages;  // [kFmNB] activation buffer written
    const uint32_t bfree0 = bready0 + 8 * kFmNB;     // [kFmNB] activation buffer consumed
    const uint32_t tfull0 = bfree0 + 8 * kFmNB;
    const uint32_t tempty0 = tfull0 + 8 * kFmHalves;
    const uint32_t done_bar = tempty0 + 8 * kFmHalves;
    const uint32_t redfull = done_bar + 8, redfree = redfull + 8;
    float *red = reinterpret_cast<float *>(smem + fm_red_off(a.stages));
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + fm_misc_off(a.stages));
    volatile uint32_t *tmem_slot = misc;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
    volatile int *issued = reinterpret_cast<volatile int *>(misc + 2);

    {
        // the launch must match the plan: uniform over the grid, so every CTA
        // leaves here together (no cluster barrier yet)
        uint32_t dyn, nct = 1;
        asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if (S > 1) asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(nct));
        if (dyn < fm_smem_bytes(a.stages) || nct != (uint32_t)S || gridDim.x % S != 0 || a.stages < 1) {
            if (threadIdx.x == 0) record_error(kErrLaunchConfig);
            return;
        }
    }
    const int rank = S > 1 ? (int)cluster_ctarank() : 0;
    const int ci = blockIdx.x / S, P = gridDim.x / S;
    const int t0 = (int)(((long long)a.tiles * ci) / P);
    const int t1 = (int)(((long long)a.tiles * (ci + 1)) / P);
    const int b_lo = (int)(((long long)a.B * rank) / S);
    const int b_hi = (int)(((long long)a.B * (rank + 1)) / S);
    const int nblk = b_hi - b_lo;
    const int ksteps = (nblk + kFmSB - 1) / kFmSB;
    int n_tiles = t1 - t0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1 + kFmEpiWarps);  // MMA commit + epilogue warps (scales)
        }
        for (int b = 0; b < kFmNB; ++b) {
            mbar_init(bready0 + 8 * b, kFmSplitWarps);   // every splitter warp
            mbar_init(bfree0 + 8 * b, 1 + kFmEpiWarps);  // MMA commit + epilogue warps (table)
        }
        for (int h = 0; h < kFmHalves; ++h) {
            mbar_init(tfull0 + 8 * h, 1);
            mbar_init(tempty0 + 8 * h, kFmEpiWarps);
        }
        mbar_init(done_bar, 1);
        mbar_init(redfull, S > 1 ? kFmEpiThreads * (S - 1) : 1);
        mbar_init(redfree, kFmEpiThreads);
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(misc), kFmTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    if (S > 1) cluster_sync_all();  // peers' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if ((tmem >> 16) != 0 || (tmem & 0xFFFFu) + kFmTmemCols > 512) {  // lane 0, columns in range
        if (threadIdx.x == 0) record_error(kErrLaunchConfig);
        n_tiles = 0;
    }
    const int total = n_tiles * ksteps;

    if (warp == 0) {
        // --------------------------- producer (weights) ---------------------------
        if (lane == 0 && total > 0) {
            const uint64_t pw = policy_evict_first();
            // ring slot/phase and (tile, k step) are carried along: no
            // division by a runtime value per stage
            auto issue_w = [&](int slot, int tile_i, int ks) {
                const int tile = t0 + tile_i;
                const int b0 = b_lo + ks * kFmSB;
                const uint32_t st = smem_u32(smem + (size_t)slot * kFmStageBytes);
                const uint32_t full = full0 + 8 * slot;
                const int ga = SWIGLU ? 8 * tile : 16 * tile;
                const int gb = SWIGLU ? a.up_group0 + 8 * tile : 16 * tile + 8;
                mbar_arrive_expect_tx(full, kFmStageBytes);
                tma_load_3d(st, &tq, full, 0, 2 * b0, ga, pw);
                tma_load_3d(st + kFmQBox, &tq, full, 0, 2 * b0, gb, pw);
                tma_load_3d(st + kFmDOff, &td, full, 0, b0, ga, pw);
                tma_load_3d(st + kFmDOff + kFmDBox, &td, full, 0, b0, gb, pw);
            };
            const int pro = total < a.stages ? total : a.stages;
            int it = 0, tile = 0, ks = 0;
            for (; it < pro; ++it) {  // weights never depend on the previous grid
                issue_w(it, tile, ks);
                if (++ks == ksteps) { ks = 0; ++tile; }
            }
            pdl_wait_and_trigger();
            int slot = pro % a.stages, phase = pro / a.stages;  // ring position of iteration `pro`
            for (; it < total; ++it) {
                if (!mbar_wait(empty0 + 8 * slot, (phase & 1) ^ 1, abort_flag)) break;
                issue_w(slot, tile, ks);
                if (++ks == ksteps) { ks = 0; ++tile; }
                if (++slot == a.stages) { slot = 0; ++phase; }
            }
            *issued = it;
        } else {
            pdl_wait_and_trigger();
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        pdl_wait_and_trigger();
        if (lane == 0) {
            bool ok = true;
            int slot = 0, phase = 0, ks = 0;  // ring position and k step of iteration `it`
            for (int it = 0; it < total && ok;
                 ++it, ks = ks + 1 == ksteps ? 0 : ks + 1, slot = slot + 1 == a.stages ? 0 : slot + 1,
                     phase ^= slot == 0 ? 1 : 0) {
                const int ab = it % kFmNB;
                if (!mbar_wait(full0 + 8 * slot, phase, abort_flag)) break;
                if (!mbar_wait(bready0 + 8 * ab, (it / kFmNB) & 1, abort_flag)) break;
                tc_fence_after();
                const int nb = min(kFmSB, nblk - ks * kFmSB);
                const uint32_t st = smem_u32(smem + (size_t)slot * kFmStageBytes);
                const uint32_t xb = smem_u32(act + ab * kFmActBytes);
                for (int h = 0; h < kFmHalves; ++h) {
                    // the epilogue has read this half of the previous stage
                    if (!mbar_wait(tempty0 + 8 * h, (it & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = h * kFmHalfBlocks; j < (h + 1) * kFmHalfBlocks && j < nb; ++j) {
                        // A: columns 2j, 2j+1 (128 B apart), groups kFmCS * 128 B apart
                        const uint64_t ad = mma_smem_desc(st + j * 2 * kColBytes, kColBytes, kFmCS * kColBytes);
                        // B: columns kFmXbColStride apart, 8-row groups 128 B apart
                        const uint64_t bd = mma_smem_desc(xb + j * 2 * kFmXbColStride, kFmXbColStride, 8 * 16);
                        mma_i8(tmem + j * kFmBlockCols, ad, bd, kFmIdesc);
                    }
                    mma_commit(tfull0 + 8 * h);
                }
                if (ok) {
                    mma_commit(empty0 + 8 * slot);
                    mma_commit(bfree0 + 8 * ab);
                }
            }
            // nothing may still read shared memory or write TMEM when the CTA
            // frees them
            mma_commit(done_bar);
            mbar_drain(done_bar, 0);
        }
        __syncwarp();
    } else if (warp < 2 + kFmSplitWarps) {
        // ------------------------------ splitters -----------------------------
        const int sw = warp - 2;  // activation rows sw and sw + 8
        const int K = 32 * a.B;
        pdl_wait_and_trigger();   // the activations belong to the previous grid until now
        uint4 xr[2][2];
        auto load = [&](int ks) {
            const int b0 = b_lo + ks * kFmSB, nb = min(kFmSB, nblk - ks * kFmSB);
            fm_load_x(x, K, sw, a.N, b0, nb, lane, xr[0]);
            fm_load_x(x, K, sw + 8, a.N, b0, nb, lane, xr[1]);
        };
        if (total > 0) load(0);
        for (int it = 0, ks = 0; it < total; ++it, ks = ks + 1 == ksteps ? 0 : ks + 1) {
            const int ab = it % kFmNB;
            // the buffer's previous stage (it - kFmNB) has been read by its MMAs and epilogue
            const bool ok =
                it < kFmNB || mbar_wait_warp(bfree0 + 8 * ab, ((it / kFmNB) - 1) & 1, abort_flag);
            if (ok) {
                const int nb = min(kFmSB, nblk - ks * kFmSB);
                uint8_t *abuf = act + ab * kFmActBytes;
                if (sw < a.N) fm_split_row(abuf, xr[0], sw, lane, nb);
                if (sw + 8 < a.N) fm_split_row(abuf, xr[1], sw + 8, lane, nb);
            }
            fence_proxy_async_smem();  // the MMA reads the pieces through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(bready0 + 8 * ab);
            if (it + 1 < total) load(ks + 1 == ksteps ? 0 : ks + 1);  // lands while this stage's pieces are consumed
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        const int ew = warp - 2 - kFmSplitWarps;  // epilogue warp 0..15
        const int q = warp & 3;                   // TMEM lane quarter of this warp
        const int n0 = TOK * (ew >> 2);           // its activation rows n0 .. n0 + TOK - 1
        const bool active = n0 < a.N;
        const int row = 32 * q + lane;            // tile row = TMEM lane
        const int g = row >> 3, r = row & 7;      // packed group (0..15) and row in it
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + n0;
        pdl_wait_and_trigger();  // the outputs belong to the previous grid until now
        float acc[TOK];
        int it = 0, slot = 0, phase = 0;  // ring position of iteration `it`, carried along
        for (int tl = 0; tl < n_tiles; ++tl) {
#pragma unroll
            for (int t = 0; t < TOK; ++t) acc[t] = 0.f;
            for (int ks = 0; ks < ksteps;
                 ++ks, ++it, slot = slot + 1 == a.stages ? 0 : slot + 1, phase ^= slot == 0 ? 1 : 0) {
                const int ab = it % kFmNB;
                const uint8_t *st = smem + (size_t)slot * kFmStageBytes;
                const uint8_t *abuf = act + ab * kFmActBytes;
                // the stage's table entries are written, and its weights (their
                // scales) have landed
                bool ok = mbar_wait_warp(bready0 + 8 * ab, (it / kFmNB) & 1, abort_flag);
                ok = ok && mbar_wait_warp(full0 + 8 * slot, phase, abort_flag);
                const int nb = min(kFmSB, nblk - ks * kFmSB);
                for (int h = 0; h < kFmHalves && ok; ++h) {
                    const bool okh = mbar_wait_warp(tfull0 + 8 * h, it & 1, abort_flag);
                    if (okh && active) tc_fence_after();
#pragma unroll
                    for (int bt = 0; bt < kFmHalfBlocks / LB; ++bt) {
                        const int jb = h * kFmHalfBlocks + bt * LB;
                        const bool work = okh && active && jb < nb;
                        uint32_t v[LB][kFmPieces][TOK];
                        if (work) {
#pragma unroll
                            for (int jj = 0; jj < LB; ++jj)
#pragma unroll
                                for (int k = 0; k < kFmPieces; ++k) {
                                    const uint32_t ta = taddr + (jb + jj) * kFmBlockCols + k * kFmN;
                                    if (TOK == 4)
                                        tmem_ld4_async(ta, v[jj][k]);
                                    else if (TOK == 2)
                                        tmem_ld2_async(ta, v[jj][k]);
                                    else
                                        tmem_ld1_async(ta, v[jj][k]);
                                }
                            uint32_t *vf = &v[0][0][0];
                            tmem_wait_ld8(vf);
                            tmem_wait_ld8(vf + 8);
                            tmem_wait_ld8(vf + 16);
                        }
                        if (bt == kFmHalfBlocks / LB - 1) {
                            // every load of this half is done: the MMAs may refill it
                            if (work) tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(tempty0 + 8 * h);
                        }
                        if (work) {
                            if (nb == kFmSB)
                                fm_epilogue_blocks<true, TOK, LB>(acc, v, jb, nb, st, abuf, g, r, n0);
                            else
                                fm_epilogue_blocks<false, TOK, LB>(acc, v, jb, nb, st, abuf, g, r, n0);
                        }
                    }
                    if (!okh) break;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(empty0 + 8 * slot);
                    mbar_arrive(bfree0 + 8 * ab);
                }
            }
            // ---- tile done: K-split partials meet in the leader, rank order ----

            bool store = true;
            if (S > 1) {
                if (rank != 0) {
                    store = false;
                    if (tl == 0 || mbar_wait_cluster(redfree, (tl - 1) & 1, abort_flag)) {
                        if (active) {
#pragma unroll
                            for (int t = 0; t < TOK; ++t) red[(n0 + t) * 128 + row] = acc[t];
                        }
                    }
                    mbar_arrive_cluster(map_to_rank(redfull, 0));
                } else {
                    if (mbar_wait_cluster(redfull, tl & 1, abort_flag)) {
                        if (active) {
                            for (int p = 1; p < S; ++p) {
                                const uint32_t base = map_to_rank(smem_u32(red), (uint32_t)p);
#pragma unroll
                                for (int t = 0; t < TOK; ++t)
                                    acc[t] += ld_cluster_f32(base + ((n0 + t) * 128 + row) * 4);
                            }
                        }
                    } else {
                        store = false;
                    }
                    for (int p = 1; p < S; ++p) mbar_arrive_cluster(map_to_rank(redfree, (uint32_t)p));
                }
            }
            if (SWIGLU) {
                // lanes 64..127 hold u for the outputs of lanes 0..63; the
                // leader's own partial-sum area is free for the exchange
                if (rank == 0) {
                    if (store && active && q >= 2) {
#pragma unroll
                        for (int t = 0; t < TOK; ++t) red[(n0 + t) * 64 + row - 64] = acc[t];
                    }
                    named_barrier(1, kFmEpiThreads);
                    const int orow = (t0 + tl) * 64 + row;
                    if (store && active && q < 2 && orow < a.M_out) {
#pragma unroll
                        for (int t = 0; t < TOK; ++t)
                            if (n0 + t < a.N)
                                a.y[(size_t)(n0 + t) * a.M_out + orow] =
                                    silu_mul(acc[t], red[(n0 + t) * 64 + row]);
                    }
                    named_barrier(1, kFmEpiThreads);
                }
            } else {
                const int orow = (t0 + tl) * 128 + row;
                if (store && active && orow < a.M_out) {
#pragma unroll
                    for (int t = 0; t < TOK; ++t)
                        if (n0 + t < a.N) {
                            const size_t o = (size_t)(n0 + t) * a.M_out + orow;
                            a.y[o] = a.res ? __fadd_rn(acc[t], a.res[o]) : acc[t];  // y may be res
                        }
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kFmTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag) {
        const int n_issued = *issued;
        for (int i = n_issued > a.stages ? n_issued - a.stages : 0; i < n_issued; ++i)
            mbar_drain(full0 + 8 * (i % a.stages), (i / a.stages) & 1);
    }
    __syncwarp();
    // no CTA leaves while a peer may still read its partials
    if (S > 1) cluster_sync_all();
}

}  // namespace q8
