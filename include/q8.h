/*
 * q8.h -- C ABI of libq8: decode-time products of GGUF Q8_0 block-quantised
 * weights with activations, for NVIDIA B200 (sm_100a).
 *
 * A Q8_0 block holds 32 int8 values q and one binary16 scale d; the weight is
 * d*q.  The product this library serves is the one the Qwen inference pages
 * keep returning to: "Lumen v0.3.0 -- profile, parallelize, 4x faster than
 * v0.2.0" (Phase 7.E.0) measures gate_up, lm_head and down matmuls at most of
 * a decode step, and "skuznetsov/cogni-ml" README ("Build Qwen CLIs") runs a
 * Q8_0 GEMV straight over the GGUF block layout.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Shapes: M output rows, K reduction length (a multiple of 32), N activation
 *    columns (tokens, 1..16).  Activations x are [N][K] fp32 row-major (one
 *    token per row); outputs are [N][M] fp32 row-major.
 *  - Memory: every pointer argument is DEVICE memory owned by the caller,
 *    16-byte aligned.  The library allocates, frees and synchronises nothing in
 *    these calls; scratch, where a call needs it, is passed in by the caller
 *    and sized by the matching *_bytes query.
 *  - Streams: work is enqueued on `stream` (0 = the legacy default stream) and
 *    returns immediately; results are ready when the stream reaches them.  The
 *    launches use programmatic dependent launch: a kernel may start streaming
 *    its weights while the previous kernel on the stream finishes, and reads
 *    its activations only after that kernel has completed.
 *  - Errors: arguments are checked on the host before anything is enqueued.
 *    A rejected call returns a non-zero q8_status and enqueues nothing.  A
 *    failed launch returns Q8_ERR_CUDA (q8_last_cuda_error() names it).
 *    Kernels bound every internal wait; a wait that runs out sets a sticky
 *    device error word that q8_read_device_error() returns.
 *  - Device data that the host cannot see (expert indices, activation
 *    values) is trusted: out-of-range expert indices and NaN router logits are
 *    undefined behaviour, as in "fusedtok 1.3.0" ("Roadmap", 1.2.1: host-side
 *    validation with a documented device-tensor trust boundary).
 *
 * Packed weight layout (what q8_pack_weights writes)
 * --------------------------------------------------
 * Rows are taken in groups of 8 (the last group is padded with zero rows).
 * With B = K/32 blocks per row, group g occupies 272*B bytes at offset
 * g*272*B:
 *    q part, 256*B bytes: for each 16-byte column c in [0, 2B) (half a block)
 *        and each row r in [0, 8): the 16 values q[8g+r][16c .. 16c+15],
 *        each stored as the byte (q + 128), i.e. q XOR 0x80;
 *    d part, 16*B bytes: for each block b and row r: the binary16 d[8g+r][b].
 * Every 16-byte piece is aligned, each (group, column) piece is one 8-row x
 * 16-byte core matrix of the tensor cores' K-major operand layout, and the
 * size is exactly 34 bytes per 32 weights (plus the zero rows of the last
 * group).  q8_unpack_weights restores the GGUF bytes exactly.
 */
#ifndef Q8_H_
#define Q8_H_

#include <stddef.h>
#include <stdint.h>
#include <string.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st *q8_stream_t;

typedef enum q8_status {
    Q8_OK = 0,
    Q8_ERR_INVALID = 1,      /* null pointer or bad enum / flag                 */
    Q8_ERR_SHAPE = 2,        /* non-positive size, K % 32 != 0, size mismatch   */
    Q8_ERR_ALIGN = 3,        /* pointer not 16-byte aligned                     */
    Q8_ERR_NOT_DEVICE = 4,   /* pointer is not device memory                    */
    Q8_ERR_UNSUPPORTED = 5,  /* legal but outside what the kernels serve (N>16) */
    Q8_ERR_CUDA = 6,         /* a CUDA call or launch failed                    */
    Q8_ERR_DEVICE_TIMEOUT = 7 /* a kernel's bounded wait ran out (see below)    */
} q8_status;

/* Static text for a status code. */
const char *q8_status_string(int status);

/* Text of the last CUDA error seen by this thread inside the library
 * ("no error" when none). */
const char *q8_last_cuda_error(void);

/* Synchronises the current device, then returns and clears the sticky device
 * error word of the current device: Q8_OK when no kernel recorded a problem,
 * Q8_ERR_DEVICE_TIMEOUT otherwise.  *detail (nullable) receives the raw word,
 * an OR of: 1 = a bounded wait ran out (the kernel returned early and its
 * outputs are incomplete), 2 = waiting for in-flight copies at exit ran out,
 * 4 = q8_moe_gemv skipped an expert pick (out of range, or repeated within a
 * token), 8 = a kernel found its launch configuration differing from its
 * plan (it returned without computing). */
q8_status q8_read_device_error(uint32_t *detail);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int q8_version(void);

/* ---------------------------------------------------------------------- */
/* S1  Weight packer                                                       */
/* ---------------------------------------------------------------------- */

/* Bytes of the packed layout for an M x K matrix: ceil(M/8) * 8.5 * K.
 * Returns 0 for invalid shapes (M <= 0, K <= 0, K % 32 != 0). */
size_t q8_packed_bytes(int64_t M, int64_t K);

/* Re-lay GGUF Q8_0 blocks into the packed layout above.
 * gguf_blocks: device, M*K/32*34 bytes, row-major blocks [M][K/32], each block
 *   34 bytes = little-endian binary16 d, then 32 int8 q (the raw GGUF Q8_0
 *   layout the "skuznetsov/cogni-ml" Q8_0 GEMV probe reads, "Build Qwen CLIs").
 *   Any byte alignment.
 * packed: device, q8_packed_bytes(M, K) bytes, 16-byte aligned; fully written.
 * Pure re-layout: bit-exact and invertible.  One-time cost, not a hot call. */
q8_status q8_pack_weights(const void *gguf_blocks, int64_t M, int64_t K, void *packed,
                          q8_stream_t stream);

/* Inverse of q8_pack_weights (test aid): packed -> GGUF bytes [M][K/32][34]. */
q8_status q8_unpack_weights(const void *packed, int64_t M, int64_t K, void *gguf_blocks,
                            q8_stream_t stream);

/* ---------------------------------------------------------------------- */
/* S2/S3  Q8_0 GEMV (N = 1) and small-batch GEMM (N = 2..16), fp32 x       */
/* ---------------------------------------------------------------------- */

/* y[n][m] = sum_k d[m][k/32] * q[m][k] * x[n][k]   for n < N, m < M.
 * W: packed (q8_pack_weights) M x K.  x: [N][K] fp32.  y: [N][M] fp32, fully
 * overwritten.  fp32 arithmetic on the CUDA cores, and its only error is
 * rounding: each weight d * q is exact in fp32, and each output is a sum of
 * fp32 products in a fixed order (16-term packed dots, a chain per lane over
 * its columns, then shuffle and cross-warp sums), so |y - y_exact| <=
 * D * 2^-24 * sum_k |w x| for every input, D the longest chain of roundings:
 * D <= K/512 + 30 for N <= 4 (1e-5 * sum|w x| up to K = 70000) and
 * D <= K/64 + 30 for 5 <= N <= 16 (up to K = 8800; at K = 18944 the worst
 * case is 1.9e-5 * sum|w x|).  Typical errors are far smaller (the tests
 * measure below 1e-6 * sum|w x| at every shape).  The Q8 N=1 decode product
 * of "Lumen v0.3.0" (Phase 7.G) and the "skuznetsov/cogni-ml"
 * cuda_q8_gemv_probe ("Build Qwen CLIs"), extended to N <= 16 columns.
 * N > 16 -> Q8_ERR_UNSUPPORTED.  Bit-identical results from run to run.
 * See q8_gemv_split for the tensor-core variant. */
q8_status q8_gemv(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                  q8_stream_t stream);

/* q8_gemv with the tensor cores allowed: where it is faster (N >= 5, or
 * N >= 3 for matrices with at least 148 tiles of 128 rows), tcgen05.mma
 * kind::i8 takes the packed int8 q against an exact-scale three-term int8
 * split of each 32-block of x, x = s (q0 + q1/254 + q2/254^2) with a
 * power-of-two s per block, one MMA per Q8_0 block and an fp32 epilogue that
 * applies d and s; elsewhere it is q8_gemv.  The split's residual is below
 * 2.5e-7 of the block's max |x|, so it adds at most
 *   2.5e-7 * sum_b amax_b * sum_{k in b} |w_k|     (amax_b: block b's max |x|)
 * to the fp32 error: far inside the 1e-5 * sum_k |w x| bar for activations
 * whose blocks carry no value much larger than the rest at a near-zero
 * weight, but that bar is not guaranteed for every input (a block whose only
 * large value meets a zero weight breaks it), which is why this is a
 * separate entry point.  x -> 2x still doubles y bit for bit, and unit-scale
 * one-hot inputs come out exactly.  Blocks whose max |x| is below 2^-121
 * lose relative accuracy; non-finite x is undefined.  Shapes and limits as
 * q8_gemv.  Measured on the 7B-class shapes: 37888x3584 SwiGLU at N = 4 /
 * 8 / 16 in 49 / 59 / 83 us (CUDA cores: 77 / 92 / 197 us). */
q8_status q8_gemv_split(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                        q8_stream_t stream);

/* y[n][m] = (W x)[n][m] + residual[n][m]: the q8_gemv product with the
 * residual-stream add of the projections that feed it (attention output and
 * MLP down projection) done in the kernel's store, so the sum costs no extra
 * pass over y ("fusedtok 1.3.0": fused residual add; the residual adds of the
 * "skuznetsov/cogni-ml" layer tail).  residual: [N][M] fp32 device; it may be
 * y itself (in-place update), any other overlap is undefined.  The add is one
 * fp32 rounding of q8_gemv's own value: bit-identical to adding residual to
 * the output q8_gemv writes for the same call shape.  Shapes, limits and the
 * 1e-5 * sum|w x| bound (plus the add's rounding) as q8_gemv. */
q8_status q8_gemv_residual(const void *W, const float *x, const float *residual, float *y, int64_t M,
                           int64_t K, int64_t N, q8_stream_t stream);

/* Greedy-decode head: the GEMV of q8_gemv with the arg-max over the M outputs
 * of each column fused into it, so the logits need not be written or read
 * back ("skuznetsov/cogni-ml" README, its resident top-1 decode step; ties go
 * to the earliest index, as in the "fusedtok 1.3.0" "API stability" note).
 * best: [N] uint64 keys, device, 8-byte aligned, overwritten (a first small
 * kernel on `stream` zeroes them, then the GEMV's CTAs combine theirs with
 * atomicMax; two launches, both in the dependent-launch chain).  Key =
 * (order-preserving bits of the max value) << 32 | (0xFFFFFFFF - index): the
 * row index is q8_argmax_index(key), the value q8_argmax_value(key).  Among
 * equal values the lowest index wins; -0 counts as +0; NaN outputs are
 * undefined.  y: [N][M] fp32, or NULL to skip writing the logits; when given
 * it holds the logits the pick was taken from (best[n] is exactly the first
 * maximum of y[n]); they meet q8_gemv's tolerance, and match q8_gemv's bits
 * wherever q8_gemv takes the same column-owner kernel (large M).
 * 1 <= N <= 4 (larger N -> Q8_ERR_UNSUPPORTED). */
q8_status q8_gemv_argmax(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                         uint64_t *best, q8_stream_t stream);

static inline int32_t q8_argmax_index(uint64_t key) {
    return (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFu));
}
static inline float q8_argmax_value(uint64_t key) {
    const uint32_t h = (uint32_t)(key >> 32);
    const uint32_t u = (h & 0x80000000u) ? (h & 0x7FFFFFFFu) : ~h;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ---------------------------------------------------------------------- */
/* K-quant GEMV: Q4_K and Q6_K weights in their raw GGUF layout            */
/* ---------------------------------------------------------------------- */

/* y[n][m] = sum_k w[m][k] * x[n][k] for a matrix stored as GGUF K-quant
 * super-blocks of 256 weights (the Q4_K / Q6_K GEMV probes of the
 * "skuznetsov/cogni-ml" README, "Build Qwen CLIs", which also read the raw
 * blocks).  W: [M][K/256] blocks, rows contiguous, unpacked.  x: [N][K] fp32,
 * 16-byte aligned.  y: [N][M] fp32.  K % 256 == 0; 1 <= N <= 4.  Each output
 * is within 1e-5 * sum_k |w x| of the exact value (every weight formed with
 * at most one fp32 rounding).  CUDA cores: Q4_K in tiles of 32 rows fed by
 * TMA boxes (activation rows two per launch), Q6_K one warp per row.
 * Q4_K, 144-byte blocks, W 16-byte aligned: d (binary16) | dmin (binary16) |
 *   scales[12] | qs[128].  Sub-block j (weights 32j..32j+31) has a 6-bit
 *   scale sc and min m: j < 4: sc = scales[j] & 63, m = scales[j+4] & 63;
 *   j >= 4: sc = (scales[j+4] & 15) | (scales[j-4] >> 6) << 4,
 *   m = (scales[j+4] >> 4) | (scales[j] >> 6) << 4.  Weight e: byte
 *   qs[32(e/64) + e%32], low nibble if e%64 < 32 else high; w = d sc q - dmin m.
 * Q6_K, 210-byte blocks: ql[128] | qh[64] | scales[16] (int8) | d (binary16).
 *   Weight e: h = e/128, c = (e%128)/32, l = e%32; q = ((ql[64h + 32(c&1) + l]
 *   >> 4(c>>1)) & 15) | ((qh[32h + l] >> 2c) & 3) << 4, minus 32;
 *   w = d * scales[8h + 2c + l/16] * q. */
q8_status q8_q4k_gemv(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                      q8_stream_t stream);
q8_status q8_q6k_gemv(const void *W, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                      q8_stream_t stream);

/* Q6_K packed for the tile kernel.  Raw 210-byte blocks start on 2-byte
 * boundaries, which TMA and 16-byte copies cannot fetch, so the blocks are
 * re-laid once into 6720-byte units, one per (tile of 32 rows, block):
 *   unit (t, b) at byte (t * (K/256) + b) * 6720; row i of the tile (matrix
 *   row 32t + i) at byte 208 i of the unit holds bytes 0..207 of its raw
 *   block b (ql | qh | scales); bytes 6656 + 2i and 6657 + 2i hold its d;
 *   rows past M are zero.
 * q8_q6k_packed_bytes: ceil(M/32) * (K/256) * 6720 (0 for a bad shape).
 * q8_q6k_pack_weights: raw (device, [M][K/256] blocks, any alignment) ->
 *   packed (device, 16-byte aligned, fully written).  q8_q6k_unpack_weights:
 *   the inverse (bit-exact round trip).  q8_q6k_gemv_packed: the product of
 *   q8_q6k_gemv from the packed units, same arguments, bound and N <= 4
 *   (activation rows two per launch); each 16-weight run is summed as
 *   sum (q - 32) x and scaled once by d * scale (exact), so the bound is
 *   unchanged.  Shape and pointer errors are reported before anything is
 *   enqueued. */
size_t q8_q6k_packed_bytes(int64_t M, int64_t K);
q8_status q8_q6k_pack_weights(const void *raw, int64_t M, int64_t K, void *packed, q8_stream_t stream);
q8_status q8_q6k_unpack_weights(const void *packed, int64_t M, int64_t K, void *raw, q8_stream_t stream);
q8_status q8_q6k_gemv_packed(const void *packed, const float *x, float *y, int64_t M, int64_t K, int64_t N,
                             q8_stream_t stream);

/* ---------------------------------------------------------------------- */
/* S4  Fused gate_up + SwiGLU                                              */
/* ---------------------------------------------------------------------- */

/* h[n][i] = silu(g) * u,  g = (W x)[n][i],  u = (W x)[n][I + i],
 * silu(g) = g / (1 + exp(-g)).  W: packed [2I][K] with the gate rows first
 * and the up rows after them (the concatenation of the ffn_gate and ffn_up
 * projections of the "skuznetsov/cogni-ml" FFN probe, "Build Qwen CLIs"; the
 * SwiGLU MLP of the "augur" README, "Features").  I must be a multiple of 8.
 * x: [N][K] fp32.  h: [N][I] fp32, fully overwritten.  One launch; g and u
 * never leave the chip.  g and u each within q8_gemv's bound; h within the
 * bound that carries through silu and the product. */
q8_status q8_gate_up_swiglu(const void *W, const float *x, float *h, int64_t I, int64_t K,
                            int64_t N, q8_stream_t stream);

/* q8_gate_up_swiglu with the tensor cores allowed, as q8_gemv_split (a tile
 * holds 64 gate rows and their 64 up rows; g and u carry q8_gemv_split's
 * bound). */
q8_status q8_gate_up_swiglu_split(const void *W, const float *x, float *h, int64_t I, int64_t K,
                                  int64_t N, q8_stream_t stream);

/* ---------------------------------------------------------------------- */
/* S5  MoE router                                                          */
/* ---------------------------------------------------------------------- */

/* For each token t < T: p = softmax(logits[t][0..E)); idx[t][0..top_k) = the
 * top_k experts by logit value in descending order, ties to the lowest expert
 * index ("fusedtok 1.3.0", "API stability"); w[t][j] = p[idx[t][j]], divided
 * by the sum of the picked p when renormalize != 0.  The router + top-k
 * expert step of "Add Qwen1.5-MoE Q8_0 CPU and single-token TornadoVM GPU
 * inference - #144" (PR summary).
 * logits: [T][E] fp32.  idx: [T][top_k] int32.  w: [T][top_k] fp32.
 * Limits: 1 <= T <= 16, 1 <= top_k <= min(E, 8), E <= 256. */
q8_status q8_moe_route(const float *logits, int64_t T, int64_t E, int64_t top_k,
                       int renormalize, int32_t *idx, float *w, q8_stream_t stream);

/* ---------------------------------------------------------------------- */
/* S6  Grouped MoE GEMV over the routed experts                            */
/* ---------------------------------------------------------------------- */

/* Scratch bytes q8_moe_gemv needs for these sizes. */
size_t q8_moe_workspace_bytes(int64_t T, int64_t E, int64_t top_k, int64_t H, int64_t I,
                              int64_t I_shared);

/* Zero-fill workspace_bytes bytes of a MoE workspace (asynchronous on
 * `stream`).  A workspace must be zero-filled once before its first
 * q8_moe_gemv call; each call that completes without a device error leaves it
 * ready for the next one.  After a call that recorded a device error
 * (q8_read_device_error), zero-fill it again. */
q8_status q8_moe_workspace_init(void *workspace, size_t workspace_bytes, q8_stream_t stream);

/* y[t] = sum_{s < top_k} w[t][s] * Down_e(SwiGLU(GateUp_e x[t]))  (e = idx[t][s])
 *        + Down_sh(SwiGLU(GateUp_sh x[t]))             (when a shared expert is given)
 * in one launch of one CTA per SM.  The CTAs first compute SwiGLU(gate_up) for
 * every selected (expert, token) pair and the shared expert, then the down
 * projection of each selected expert for its own tokens, then the weighted
 * sum; counters in the workspace order the phases between CTAs (a down tile
 * starts once its expert's SwiGLU rows are all stored; the CTA that stores
 * an output group's last down tile adds that group up), so the down weights
 * stream while the last SwiGLU rows are still being finished.  Only the
 * selected experts' weights are read, each once for all of its tokens, and
 * only their tokens' activations.  The slot weighting and shared expert
 * follow the router + top-k expert + shared-expert FFN block of "Add
 * Qwen1.5-MoE Q8_0 ... - #144" (PR summary); folding the per-slot launches
 * into one grid follows the routed-expert launch fusion in that PR's
 * conversation.  Every output is summed in a fixed order (routed experts by
 * ascending expert id, then the shared expert), so results are bit-identical
 * from run to run.
 *   gate_up_experts: E consecutive packed matrices [2I][H], each
 *       q8_packed_bytes(2I, H) bytes (gate rows first, as q8_gate_up_swiglu).
 *   down_experts:    E consecutive packed matrices [H][I], each
 *       q8_packed_bytes(H, I) bytes.
 *   shared_gate_up / shared_down: packed [2*I_shared][H] / [H][I_shared], or
 *       both NULL (with I_shared = 0) for no shared expert.
 *   idx, w: [T][top_k] as written by q8_moe_route.  A pick outside [0, E), or
 *       a token's repeated pick of one expert, is skipped (it adds nothing)
 *       and sets bit 4 of the device error word (q8_read_device_error).
 *   x: [T][H] fp32.  y: [T][H] fp32, fully overwritten.
 *   workspace: >= q8_moe_workspace_bytes(...) bytes of device memory, 16-byte
 *       aligned, zero-filled before its first use (q8_moe_workspace_init) and
 *       then left to the library; calls that may run at the same time must
 *       not share one.
 * Limits: 1 <= T <= 16, top_k <= 8, E <= 256, H, I, I_shared multiples of 32,
 * H, I, I_shared <= 65536. */
q8_status q8_moe_gemv(const void *gate_up_experts, const void *down_experts,
                      const void *shared_gate_up, const void *shared_down,
                      const int32_t *idx, const float *w, const float *x, float *y, int64_t T,
                      int64_t E, int64_t top_k, int64_t H, int64_t I, int64_t I_shared,
                      void *workspace, size_t workspace_bytes, q8_stream_t stream);

/* Same product as q8_moe_gemv, without a workspace argument.  The pages have
 * no counterpart: this variant exists for callers that cannot allocate device
 * memory when they call -- for example a plug-in that is handed finished
 * device buffers by a host framework that owns the memory pool and gives it
 * no allocator, or a decode loop that must not risk an allocation's implicit
 * synchronisation in the middle of a token.
 * Scratch comes from a fixed 4 MiB array in the library's device memory, held
 * by every GPU that loads the library until the process exits.  Sizes whose
 * q8_moe_workspace_bytes() exceeds 4 MiB are rejected with
 * Q8_ERR_UNSUPPORTED (q8_last_cuda_error() gives the byte counts).  Nothing is
 * allocated or freed.
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * Every argument is checked, as for q8_moe_gemv, before anything is
 * enqueued.  All calls share the one array, which keeps the last call's
 * contents: each call first launches a one-warp kernel on `stream` that, once
 * the work before it on the stream is done, clears the array's counter region,
 * then the MoE kernel (both as dependent launches, so the MoE kernel still
 * prefetches its weights early).  Calls that may run at the same time on the
 * GPU (different streams without an ordering between them) race on the array
 * and must not be issued. */
q8_status q8_moe_gemv_noalloc(const void *gate_up_experts, const void *down_experts,
                              const void *shared_gate_up, const void *shared_down,
                              const int32_t *idx, const float *w, const float *x, float *y,
                              int64_t T, int64_t E, int64_t top_k, int64_t H, int64_t I,
                              int64_t I_shared, q8_stream_t stream);

/* ---------------------------------------------------------------------- */
/* S7  Activation quantisation to Q8_0                                     */
/* ---------------------------------------------------------------------- */

/* Per 32-block of each row of x: amax = max |x|, d32 = amax / 127 (IEEE fp32
 * division), q = round-half-away-from-zero(x / d32) (IEEE fp32 division),
 * clamped to [-127, 127]; amax == 0 gives d = 0 and q = 0; xd = binary16 of
 * d32, round to nearest even.  Bit-exact.  The per-block int8 quantisation of
 * fp32 activations in "Add Qwen1.5-MoE Q8_0 ... - #144" ("Key implementation
 * notes").
 * x: [N][K] fp32.  xq: [N][K] int8.  xd: [N][K/32] binary16 bits. */
q8_status q8_quantize_act(const float *x, int8_t *xq, uint16_t *xd, int64_t N, int64_t K,
                          q8_stream_t stream);

/* RMSNorm fused in front of the quantiser (the prologue of the integer
 * product; the norm that precedes every Qwen projection, "augur" README,
 * "Features"; "fusedtok 1.3.0" rmsnorm(x, w, eps)).  Per row n:
 *   r = 1 / sqrt(sum_k x^2 / K + eps), fp32, the sum taken in a fixed order
 *   inside one CTA (no cross-CTA reduction: the race of "Add Qwen1.5-MoE Q8_0
 *   ... - #144", conversation), the division, add and reciprocal square root
 *   correctly rounded;
 *   xhat[k] = (x[k] * r) * gamma[k], two fp32 roundings in that order;
 *   xq, xd = the q8_quantize_act rule applied to xhat.
 * x: [N][K] fp32, 16-byte aligned.  gamma: [K] fp32.  xq: [N][K] int8.
 * xd: [N][K/32] binary16 bits.  rinv: [N] fp32, the r of each row, or NULL.
 * Given r, xq and xd are bit-exact; r is within (K/256 + 12) * 2^-24
 * (relative) of the exact value: each thread sums about K/256 squares, all
 * positive, before an 8-level tree (about 5e-6 at K = 18944, and far less on
 * typical data).  eps must be >= 0 and finite (else Q8_ERR_INVALID); a zero row with
 * eps == 0, or non-finite x or gamma, gives undefined codes. */
q8_status q8_rmsnorm_quantize_act(const float *x, const float *gamma, float eps, int8_t *xq,
                                  uint16_t *xd, float *rinv, int64_t N, int64_t K,
                                  q8_stream_t stream);

/* ---------------------------------------------------------------------- */
/* S8  Q8_0 x Q8_0 integer product                                         */
/* ---------------------------------------------------------------------- */

/* y[n][m] = sum_b d_w[m][b] * d_x[n][b] * dot[n][m][b],
 * dot[n][m][b] = sum_{i<32} q_w[m][32b+i] * xq[n][32b+i]  (exact int32).
 * The int8 x int8 accumulation with the Q8_0 scales of "Add Qwen1.5-MoE Q8_0
 * ... - #144" ("Key implementation notes"), the Q8-native integer dot named
 * as the next step in "Lumen v0.3.0" ("v0.3 -> v0.4 candidate moves").
 * N <= 4: the int32 block dots run on the integer dot-product (dp4a) units.
 * 5 <= N <= 16: they run on the tensor cores (tcgen05.mma kind::i8, one
 * 128 x 16 x 32 MMA per block, activation rows past N read as zero); a launch
 * with fewer 128-row tiles than SMs splits K over a thread-block cluster of up
 * to 8 CTAs and adds the partial sums in rank order.  Both are deterministic.
 * W: packed M x K.  xq, xd: as written by q8_quantize_act.  y: [N][M] fp32.
 * fp32 result within 1e-5 * sum_b |d_w d_x| sum_i |q_w q_x| of the exact. */
q8_status q8q8_gemv(const void *W, const int8_t *xq, const uint16_t *xd, float *y, int64_t M,
                    int64_t K, int64_t N, q8_stream_t stream);

/* Test aid: the int32 block dots themselves, dots[n][m][b] (layout
 * [N][M][K/32]); bit-exact. */
q8_status q8q8_block_dots(const void *W, const int8_t *xq, int32_t *dots, int64_t M, int64_t K,
                          int64_t N, q8_stream_t stream);

/* ---------------------------------------------------------------------- */
/* Test aid: the failure-detection protocol                                */
/* ---------------------------------------------------------------------- */

/* Launches one CTA whose four warps wait, through the same bounded-wait code
 * as the pipelines' barriers, on a shared-memory barrier that nothing ever
 * completes, with a limit of `limit_us` microseconds (1 .. 1,000,000) in
 * place of the pipelines' 2 s.  The first wait to run out sets the timeout
 * bit (1) of the sticky device error word and the CTA's abort flag; the other
 * warps leave their waits on seeing the flag, and the kernel returns: no
 * fault, no hang, and the context stays usable.  out: 2 device int32,
 * written with the number of warps whose wait succeeded (0) and the abort
 * flag (1).  q8_read_device_error() then returns Q8_ERR_DEVICE_TIMEOUT with
 * detail bit 1 set, and clears the word.  Host-side failure handling
 * (hardened host validation and a device-data trust boundary) follows
 * "fusedtok 1.3.0", Roadmap 1.2.1; the device-side bound is this library's. */
q8_status q8_test_wait_timeout(uint32_t limit_us, int32_t *out, q8_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* Q8_H_ */
