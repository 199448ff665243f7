/*
 * q8_oracle.c -- the CPU oracle for the Q8_0 decode-product hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline use it.  It shares no code, header, table or helper with the CUDA
 * library and is deliberately plain: straight loops, fp64 accumulation, no
 * SIMD, no blocking, no reordering beyond the definitions below.  Build flags:
 * -O2 -ffp-contract=off (no fused multiply-add, so every float operation is the
 * IEEE operation written), optional -fopenmp over independent output rows.
 *
 * Sources (page title, section):
 *   [cogni-ml]  "skuznetsov/cogni-ml" README, "Build Qwen CLIs": the Q8_0 GEMV
 *               probe runs over the raw GGUF block layout and is checked against
 *               a CPU QuantMatmul reference.
 *   [lumen]     "Lumen v0.3.0 -- profile, parallelize, 4x faster than v0.2.0",
 *               Phase 7.E.0 (gate_up / down / lm_head matmuls dominate decode),
 *               Phase 7.G (Q8 N=1 decode kernel), Phase 7.J (output rows split
 *               across threads -- the same split the optional OpenMP loop uses).
 *   [pr144]     "Add Qwen1.5-MoE Q8_0 CPU and single-token TornadoVM GPU
 *               inference - #144" (GPULlama3.java): router + top-k expert +
 *               shared-expert FFN block (PR summary); "Key implementation
 *               notes": activations quantised per block to int8, int8 x int8
 *               accumulation with the Q8_0 scales.
 *   [augur]     "augur" README, "Features": Qwen MLP is SwiGLU.
 *   [fusedtok]  "fusedtok 1.3.0" PKG-INFO, "API stability": selection ties
 *               resolve to the earliest index.
 *
 * Readings where the pages are silent:
 *   - A Q8_0 block is 34 bytes: a little-endian binary16 scale d, then 32 int8
 *     values q; a weight is d*q.  Blocks run along K, rows are contiguous.
 *   - A fused gate_up matrix has the gate rows first ([0, I)) and the up rows
 *     after them ([I, 2I)).
 *   - Activation quantisation: amax = max|x| over the 32-block, d32 = amax/127
 *     as an IEEE fp32 division, q = round-half-away(x / d32) (fp32 division),
 *     clamped to [-127, 127]; amax == 0 gives d = 0 and q = 0; the stored scale
 *     is binary16 round-to-nearest-even of d32.
 *   - MoE: top-k taken on the fp32 logits (softmax is monotone), descending,
 *     ties to the lowest expert index; slot weights are the softmax
 *     probabilities over all E experts (renormalised over the k picks only when
 *     asked); the shared expert is added with weight 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define QK 32          /* weights per Q8_0 block                         */
#define BLOCK_BYTES 34 /* 2-byte binary16 scale + 32 int8                */

/* ------------------------------------------------------------------------- */
/* binary16 <-> real, written from the IEEE 754 binary16 definition           */
/* ------------------------------------------------------------------------- */

/* Value of a binary16 bit pattern: sign, 5-bit biased exponent (bias 15),
 * 10-bit fraction; exponent 0 is subnormal (fraction * 2^-24). */
double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Round an fp32 value to the nearest binary16, ties to even. */
uint16_t oracle_float_to_half_rn(float x) {
    if (isnan(x)) return 0x7e00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double v = fabs((double)x);
    /* 65504 is the largest finite half; the midpoint to 65536 rounds to even,
     * i.e. up, so everything from 65520 on overflows to infinity. */
    if (v >= 65520.0) return sign | 0x7c00;
    double quantum;
    if (v < ldexp(1.0, -14)) {
        quantum = ldexp(1.0, -24); /* subnormal spacing */
    } else {
        int e;
        frexp(v, &e);                    /* v in [2^(e-1), 2^e) */
        quantum = ldexp(1.0, e - 1 - 10); /* 10 fraction bits   */
    }
    double w = rint(v / quantum) * quantum; /* rint: ties to even */
    if (w == 0.0) return sign;
    if (w < ldexp(1.0, -14)) return sign | (uint16_t)(w / ldexp(1.0, -24));
    int e;
    double m = frexp(w, &e); /* w = m * 2^e, m in [0.5, 1) */
    uint16_t biased = (uint16_t)(e - 1 + 15);
    uint16_t frac = (uint16_t)((m * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)(biased << 10) | frac;
}

/* ------------------------------------------------------------------------- */
/* GGUF Q8_0 block access                                                     */
/* ------------------------------------------------------------------------- */

static const uint8_t *block_at(const uint8_t *gguf, int64_t row, int64_t blk, int64_t B) {
    return gguf + (row * B + blk) * BLOCK_BYTES;
}

static double block_scale(const uint8_t *blk) {
    return oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
}

static int block_q(const uint8_t *blk, int i) { return (int)(int8_t)blk[2 + i]; }

static int pick_threads(int nthreads) { return nthreads > 0 ? nthreads : 1; }

/* ------------------------------------------------------------------------- */
/* O1: y[n,m] = sum_k w[m,k] * x[n,k],  w = d*q  (fp64)                       */
/* ------------------------------------------------------------------------- */

/* One output element of the dense product over rows [row] of a GGUF matrix
 * with B blocks per row.  Also returns sum_k |w x| (the tolerance scale).
 * Each w*x is exact in fp64 (d*q has <= 18 significant bits, x 24). */
static void dot_row(const uint8_t *gguf, int64_t row, int64_t B, const float *xrow,
                    double *out, double *out_abs) {
    double s = 0.0, a = 0.0;
    for (int64_t b = 0; b < B; ++b) {
        const uint8_t *blk = block_at(gguf, row, b, B);
        double d = block_scale(blk);
        for (int i = 0; i < QK; ++i) {
            double w = d * (double)block_q(blk, i);
            double t = w * (double)xrow[b * QK + i];
            s += t;
            a += fabs(t);
        }
    }
    *out = s;
    *out_abs = a;
}

/* x: [N][K] fp32 row-major; y, y_abs: [N][M] fp64. */
void oracle_gemv(const uint8_t *gguf, const float *x, int64_t M, int64_t K, int64_t N,
                 double *y, double *y_abs, int nthreads) {
    int64_t B = K / QK;
    (void)nthreads;
#pragma omp parallel for num_threads(pick_threads(nthreads)) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            dot_row(gguf, m, B, x + n * K, &y[n * M + m], &y_abs[n * M + m]);
}

/* ------------------------------------------------------------------------- */
/* O2: fused gate_up + SwiGLU                                                 */
/* ------------------------------------------------------------------------- */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* W: GGUF [2I][K], gate rows [0, I), up rows [I, 2I).  h = silu(g) * u.
 * g, u, g_abs, u_abs, h: [N][I] fp64. */
void oracle_gate_up_swiglu(const uint8_t *gguf, const float *x, int64_t I, int64_t K,
                           int64_t N, double *h, double *g, double *u, double *g_abs,
                           double *u_abs, int nthreads) {
    int64_t B = K / QK;
    (void)nthreads;
#pragma omp parallel for num_threads(pick_threads(nthreads)) schedule(static)
    for (int64_t i = 0; i < I; ++i)
        for (int64_t n = 0; n < N; ++n) {
            int64_t o = n * I + i;
            dot_row(gguf, i, B, x + n * K, &g[o], &g_abs[o]);
            dot_row(gguf, I + i, B, x + n * K, &u[o], &u_abs[o]);
            h[o] = silu(g[o]) * u[o];
        }
}

/* ------------------------------------------------------------------------- */
/* O3: router -- softmax over E logits, top-k by value, ties to lowest index  */
/* ------------------------------------------------------------------------- */

/* logits: [T][E] fp32.  idx: [T][k] int32 (descending logit order),
 * w: [T][k] fp64 softmax probabilities of the picks (renormalised over the
 * picks when renormalize != 0).  Returns 0, or -1 on a NaN logit. */
int oracle_route(const float *logits, int64_t T, int64_t E, int64_t k, int renormalize,
                 int32_t *idx, double *w) {
    char *taken = (char *)malloc((size_t)E);
    if (!taken) return -2;
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        for (int64_t e = 0; e < E; ++e)
            if (isnan(l[e])) {
                free(taken);
                return -1;
            }
        double mx = l[0];
        for (int64_t e = 1; e < E; ++e)
            if (l[e] > mx) mx = l[e];
        double z = 0.0;
        for (int64_t e = 0; e < E; ++e) z += exp((double)l[e] - mx);
        memset(taken, 0, (size_t)E);
        double picked = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) /* strict '>' keeps the lowest index */
                if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
            taken[best] = 1;
            idx[t * k + j] = (int32_t)best;
            w[t * k + j] = exp((double)l[best] - mx) / z;
            picked += w[t * k + j];
        }
        if (renormalize)
            for (int64_t j = 0; j < k; ++j) w[t * k + j] /= picked;
    }
    free(taken);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* O4: MoE block = sum over slots of w * Down_e(SwiGLU(GateUp_e x))           */
/*                 + Down_sh(SwiGLU(GateUp_sh x))                             */
/* ------------------------------------------------------------------------- */

/* Error bound carried through SwiGLU when g and u each carry an fp32-GEMV
 * error of at most 1e-5 * sum|w x| (|silu'| <= 1.1 everywhere). */
static double swiglu_tol(double g, double u, double h, double g_abs, double u_abs) {
    double tg = 1e-5 * g_abs, tu = 1e-5 * u_abs;
    return 1.1 * tg * fabs(u) + fabs(silu(g)) * tu + 1.1 * tg * tu + 4.0 * ldexp(fabs(h), -23);
}

/* One expert's MLP for one token: h = SwiGLU(gate_up x) [I], then
 * out[m] = sum_k down[m,k] h[k], out_abs[m] = sum |down h|,
 * out_prop[m] = sum |down[m,k]| * tol_h[k]  (the h error propagated). */
static void expert_mlp(const uint8_t *gate_up, const uint8_t *down, int64_t H, int64_t I,
                       const float *xt, double *hbuf, double *tolh, double *out,
                       double *out_abs, double *out_prop) {
    int64_t Bh = H / QK, Bi = I / QK;
    for (int64_t i = 0; i < I; ++i) {
        double g, ga, u, ua;
        dot_row(gate_up, i, Bh, xt, &g, &ga);
        dot_row(gate_up, I + i, Bh, xt, &u, &ua);
        hbuf[i] = silu(g) * u;
        tolh[i] = swiglu_tol(g, u, hbuf[i], ga, ua);
    }
    for (int64_t m = 0; m < H; ++m) {
        double s = 0.0, a = 0.0, p = 0.0;
        for (int64_t b = 0; b < Bi; ++b) {
            const uint8_t *blk = block_at(down, m, b, Bi);
            double d = block_scale(blk);
            for (int i = 0; i < QK; ++i) {
                double w = d * (double)block_q(blk, i);
                double t = w * hbuf[b * QK + i];
                s += t;
                a += fabs(t);
                p += fabs(w) * tolh[b * QK + i];
            }
        }
        out[m] = s;
        out_abs[m] = a;
        out_prop[m] = p;
    }
}

/* gate_up_all: E consecutive GGUF matrices [2I][H]; down_all: E consecutive
 * GGUF matrices [H][I]; shared_* may be NULL (no shared expert).
 * idx [T][k], w [T][k] (fp64, from oracle_route), x [T][H] fp32.
 * Outputs (fp64): y [T][H]; bound [T][H] = sum_s w_s (1e-5 abs_s + prop_s)
 * + (1e-5 abs_sh + prop_sh); slot_out [T][k][H] = each routed expert's output
 * (so a caller can add sum_s |dw_s| |slot_out_s| for its own weight error). */
void oracle_moe(const uint8_t *gate_up_all, const uint8_t *down_all, const uint8_t *shared_gate_up,
                const uint8_t *shared_down, const int32_t *idx, const double *w, const float *x,
                int64_t T, int64_t E, int64_t k, int64_t H, int64_t I, int64_t I_sh, double *y,
                double *bound, double *slot_out, int nthreads) {
    size_t gu_bytes = (size_t)(2 * I) * (size_t)(H / QK) * BLOCK_BYTES;
    size_t dn_bytes = (size_t)H * (size_t)(I / QK) * BLOCK_BYTES;
    int64_t Imax = I > I_sh ? I : I_sh;
    (void)E;
    (void)nthreads;
#pragma omp parallel for num_threads(pick_threads(nthreads)) schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double *hbuf = (double *)malloc(sizeof(double) * (size_t)Imax);
        double *tolh = (double *)malloc(sizeof(double) * (size_t)Imax);
        double *o = (double *)malloc(sizeof(double) * (size_t)H);
        double *oa = (double *)malloc(sizeof(double) * (size_t)H);
        double *op = (double *)malloc(sizeof(double) * (size_t)H);
        const float *xt = x + t * H;
        for (int64_t m = 0; m < H; ++m) y[t * H + m] = bound[t * H + m] = 0.0;
        for (int64_t s = 0; s < k; ++s) {
            int64_t e = idx[t * k + s];
            double ws = w[t * k + s];
            expert_mlp(gate_up_all + (size_t)e * gu_bytes, down_all + (size_t)e * dn_bytes, H, I,
                       xt, hbuf, tolh, o, oa, op);
            for (int64_t m = 0; m < H; ++m) {
                y[t * H + m] += ws * o[m];
                bound[t * H + m] += ws * (1e-5 * oa[m] + op[m]);
                slot_out[(t * k + s) * H + m] = o[m];
            }
        }
        if (shared_gate_up && shared_down && I_sh > 0) {
            expert_mlp(shared_gate_up, shared_down, H, I_sh, xt, hbuf, tolh, o, oa, op);
            for (int64_t m = 0; m < H; ++m) {
                y[t * H + m] += o[m];
                bound[t * H + m] += 1e-5 * oa[m] + op[m];
            }
        }
        free(hbuf);
        free(tolh);
        free(o);
        free(oa);
        free(op);
    }
}

/* ------------------------------------------------------------------------- */
/* O5: quantise fp32 activations to Q8_0 (bit-exact contract, fp32 ops)       */
/* ------------------------------------------------------------------------- */

/* Round half away from zero, written out: C99 roundf semantics. */
static float round_half_away(float v) { return roundf(v); }

/* x [N][K] fp32 -> q [N][K] int8, d [N][K/32] binary16 bits.
 * Also returns the unrounded fp32 scales in d32 (may be NULL). */
void oracle_quantize_act(const float *x, int64_t N, int64_t K, int8_t *q, uint16_t *d,
                         float *d32_out) {
    int64_t B = K / QK;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < B; ++b) {
            const float *xb = x + n * K + b * QK;
            float amax = 0.0f;
            for (int i = 0; i < QK; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            float d32 = amax / 127.0f;
            for (int i = 0; i < QK; ++i) {
                int v = 0;
                if (d32 != 0.0f) {
                    float r = round_half_away(xb[i] / d32);
                    if (r > 127.0f) r = 127.0f;
                    if (r < -127.0f) r = -127.0f;
                    v = (int)r;
                }
                q[n * K + b * QK + i] = (int8_t)v;
            }
            d[n * B + b] = oracle_float_to_half_rn(d32);
            if (d32_out) d32_out[n * B + b] = d32;
        }
}

/* ------------------------------------------------------------------------- */
/* O6: Q8_0 x Q8_0 -- int32 block dots, then y = sum_b d_w d_x dot_b          */
/* ------------------------------------------------------------------------- */

/* W GGUF [M][K]; xq [N][K] int8; xd [N][K/32] binary16 bits.
 * dots (may be NULL): [N][M][K/32] int32.  y, y_abs: [N][M] fp64.
 * y_abs = sum_b |d_w d_x| * sum_i |q_w q_x|. */
void oracle_q8q8(const uint8_t *gguf, const int8_t *xq, const uint16_t *xd, int64_t M, int64_t K,
                 int64_t N, int32_t *dots, double *y, double *y_abs, int nthreads) {
    int64_t B = K / QK;
    (void)nthreads;
#pragma omp parallel for num_threads(pick_threads(nthreads)) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0, a = 0.0;
            for (int64_t b = 0; b < B; ++b) {
                const uint8_t *blk = block_at(gguf, m, b, B);
                const int8_t *xb = xq + n * K + b * QK;
                int32_t dot = 0, adot = 0;
                for (int i = 0; i < QK; ++i) {
                    int32_t p = (int32_t)block_q(blk, i) * (int32_t)xb[i];
                    dot += p;
                    adot += p < 0 ? -p : p;
                }
                if (dots) dots[(n * M + m) * B + b] = dot;
                double dd = block_scale(blk) * oracle_half_to_double(xd[n * B + b]);
                s += dd * (double)dot;
                a += fabs(dd) * (double)adot;
            }
            y[n * M + m] = s;
            y_abs[n * M + m] = a;
        }
}

/* ------------------------------------------------------------------------- */
/* O7: quantise fp32 weights to GGUF Q8_0 blocks (test aid)                   */
/* ------------------------------------------------------------------------- */

/* w [M][K] fp32 -> gguf [M][K/32][34 bytes], same per-block rule as O5.
 * d32_out (may be NULL): [M][K/32] unrounded fp32 scales. */
void oracle_quantize_weights(const float *w, int64_t M, int64_t K, uint8_t *gguf,
                             float *d32_out) {
    int64_t B = K / QK;
    int8_t qb[QK];
    uint16_t dh;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t b = 0; b < B; ++b) {
            float d32;
            oracle_quantize_act(w + m * K + b * QK, 1, QK, qb, &dh, &d32);
            uint8_t *blk = gguf + (m * B + b) * BLOCK_BYTES;
            blk[0] = (uint8_t)(dh & 0xff);
            blk[1] = (uint8_t)(dh >> 8);
            memcpy(blk + 2, qb, QK);
            if (d32_out) d32_out[m * B + b] = d32;
        }
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* -------------------------------------------------------------------------
 * K-quant formats (the Q4_K and Q6_K GEMV probes of [cogni-ml], "Build Qwen
 * CLIs", which lists the fields of each block: for Q4_K two binary16 scales,
 * twelve bytes of packed 6-bit scales and mins, and 128 bytes of 4-bit
 * values; for Q6_K low-bit and high-bit value arrays, signed 8-bit scales and
 * one binary16 scale).  The pages give no bit packing; the one below is the
 * GGUF one (a reading).  A super-block covers 256 consecutive weights of a
 * row; rows are contiguous runs of K/256 super-blocks.
 *
 * Q4_K, 144 bytes: d (binary16) | dmin (binary16) | scales[12] | qs[128].
 *   Sub-block j (0..7) covers weights 32j .. 32j+31 and has a 6-bit scale
 *   sc_j and a 6-bit min m_j:
 *     j < 4:  sc_j = scales[j] & 63,        m_j = scales[j+4] & 63
 *     j >= 4: sc_j = (scales[j+4] & 15) | ((scales[j-4] >> 6) << 4)
 *             m_j  = (scales[j+4] >> 4) | ((scales[j]   >> 6) << 4)
 *   Weight e (0..255): byte qs[32*(e/64) + e%32], its low nibble when
 *   (e%64) < 32, else its high nibble; w = d*sc_j*q - dmin*m_j, j = e/32.
 *
 * Q6_K, 210 bytes: ql[128] | qh[64] | scales[16] (int8) | d (binary16).
 *   Weight e: h = e/128, c = (e%128)/32, l = e%32;
 *     low 4 bits  = ql[64h + 32*(c&1) + l] >> (4*(c>>1)) & 15
 *     high 2 bits = qh[32h + l] >> (2c) & 3
 *     q = low | high << 4, minus 32 (so -32..31)
 *     scale = scales[8h + 2c + l/16];  w = d*scale*q.
 * ------------------------------------------------------------------------- */
#define QK_K 256
#define Q4K_BYTES 144
#define Q6K_BYTES 210

static double q4k_weight(const uint8_t *blk, int e) {
    const double d = oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    const double dmin = oracle_half_to_double((uint16_t)(blk[2] | (blk[3] << 8)));
    const uint8_t *scales = blk + 4, *qs = blk + 16;
    const int j = e / 32;
    int sc, m;
    if (j < 4) {
        sc = scales[j] & 63;
        m = scales[j + 4] & 63;
    } else {
        sc = (scales[j + 4] & 15) | ((scales[j - 4] >> 6) << 4);
        m = (scales[j + 4] >> 4) | ((scales[j] >> 6) << 4);
    }
    const uint8_t byte = qs[32 * (e / 64) + e % 32];
    const int q = (e % 64) < 32 ? (byte & 15) : (byte >> 4);
    return d * sc * q - dmin * m;
}

static double q6k_weight(const uint8_t *blk, int e) {
    const uint8_t *ql = blk, *qh = blk + 128;
    const int8_t *scales = (const int8_t *)(blk + 192);
    const double d = oracle_half_to_double((uint16_t)(blk[208] | (blk[209] << 8)));
    const int h = e / 128, c = (e % 128) / 32, l = e % 32;
    const int low = (ql[64 * h + 32 * (c & 1) + l] >> (4 * (c >> 1))) & 15;
    const int high = (qh[32 * h + l] >> (2 * c)) & 3;
    const int q = (low | (high << 4)) - 32;
    return d * scales[8 * h + 2 * c + l / 16] * q;
}

/* y[n][m] = sum_k w[m][k] x[n][k] in fp64 for a K-quant matrix (fmt 4: Q4_K,
 * 6: Q6_K); y_abs[n][m] = sum_k |w x| (the tolerance scale).  Also the
 * dequantised weights, when w_out is not NULL ([M][K] fp64). */
void oracle_kquant_gemv(int fmt, const uint8_t *blocks, const float *x, int64_t M, int64_t K,
                        int64_t N, double *y, double *y_abs, double *w_out, int nthreads) {
    const int64_t SB = K / QK_K;
    const int64_t bytes = fmt == 4 ? Q4K_BYTES : Q6K_BYTES;
    (void)nthreads;
#ifdef _OPENMP
#pragma omp parallel for num_threads(pick_threads(nthreads)) schedule(static)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const uint8_t *blk = blocks + (m * SB + k / QK_K) * bytes;
                const double w = fmt == 4 ? q4k_weight(blk, (int)(k % QK_K)) : q6k_weight(blk, (int)(k % QK_K));
                const double p = w * (double)x[n * K + k];
                acc += p;
                aacc += fabs(p);
                if (w_out && n == 0) w_out[m * K + k] = w;
            }
            y[n * M + m] = acc;
            y_abs[n * M + m] = aacc;
        }
    }
}
