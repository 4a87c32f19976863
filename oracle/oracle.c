/*
 * oracle.c -- plain, slow, obviously correct CPU oracle for the affine-quantized
 * GEMV / MoE-layer path.  TEST INFRASTRUCTURE ONLY: nothing on the product path
 * links, loads or calls this file; only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg do.
 *
 * Every floating-point step runs in fp64 on the exact values of the fp16 inputs
 * and is rounded once, to the stated output type, at the end.  Loops run in
 * index order; there is no blocking, fusion or reordering.
 *
 * What the pages fix (TurboFieldfare article, jeff.news, section "성능과 제약"
 * -- performance and constraints): the weights are MLX affine 4-bit with
 * group size 64; the router is 8-bit; routed and shared experts are 4-bit.
 * Section "내부 구조가 진짜 흥미로운 부분" (internal structure) of the same page:
 * the router picks the top-8 experts; a resident shared expert runs beside the
 * routed ones and the two outputs are added; prefill runs in chunks of at most
 * 128 tokens so one fetched expert serves several rows.
 *
 * Readings taken where the pages are silent:
 *   - affine dequantisation  w = scale*q + bias, fp16 scale and bias per group
 *     of 64 consecutive inputs (K) of one output row;
 *   - packing: element k of a row lives in word k/(32/bits), at bit offset
 *     bits*(k % (32/bits)), least-significant field first;
 *   - router: logits -> softmax over all experts -> the top_k largest logits
 *     (ties: lower expert index first), listed in descending order ->
 *     weights renormalised to sum to one over the selected experts;
 *   - expert MLP: SwiGLU, h = silu(gate x) * (up x), silu(z) = z / (1 + e^-z),
 *     r = down h;
 *   - layer output: y = shared(x) + sum_j wt_j * expert_{idx_j}(x), no residual,
 *     no normalisation, no gate on the shared expert.
 *
 * Parity status: every function below is pinned by the CPU test suite against
 * hand-packed words, closed forms, invariants or fp64 brute force; none is
 * "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 <-> binary64                                            */
/* ------------------------------------------------------------------------ */

/* binary16 bit pattern -> exact fp64 value (IEEE 754-2008 section 3.4). */
double or_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* fp64 -> binary16, round to nearest, ties to even. */
uint16_t or_f64_to_f16(double v)
{
    if (isnan(v))
        return 0x7E00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    /* the largest finite half is 65504; everything at or above the midpoint
       65520 rounds (ties to even) to infinity */
    if (a >= 65520.0)
        return sign | 0x7C00;
    int e2;
    frexp(a, &e2);            /* a = f * 2^e2 with f in [0.5, 1) */
    int E = e2 - 1;           /* exponent of the leading bit */
    if (E < -14)
        E = -14;              /* subnormal range shares the quantum 2^-24 */
    double quantum = ldexp(1.0, E - 10);
    double n = a / quantum;   /* exact: division by a power of two */
    double r = floor(n);
    double frac = n - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))
        r += 1.0;
    /* r in [0, 2048]; r == 2048 means the rounding carried into the exponent */
    long ir = (long)r;
    if (ir < 1024) /* subnormal (only possible when E == -14) */
        return sign | (uint16_t)ir;
    int biased = E + 15;
    if (ir == 2048) {
        ir = 1024;
        biased += 1;
    }
    if (biased >= 31)
        return sign | 0x7C00;
    return sign | (uint16_t)((biased << 10) | (ir - 1024));
}

/* fp64 -> binary32, round to nearest even (the C conversion does exactly that
   under the default rounding mode). */
float or_f64_to_f32(double v) { return (float)v; }

/* ------------------------------------------------------------------------ */
/* Packing (codes are `bits` wide, bits in {4, 8}; 32/bits codes per word)   */
/* ------------------------------------------------------------------------ */

int or_unpack(const uint32_t *packed, int64_t N, int64_t K, int bits, uint8_t *codes)
{
    if (bits != 4 && bits != 8)
        return -1;
    int64_t per = 32 / bits;
    if (K % per)
        return -1;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint32_t word = packed[n * (K / per) + k / per];
            codes[n * K + k] = (uint8_t)((word >> (bits * (k % per))) & mask);
        }
    return 0;
}

int or_pack(const uint8_t *codes, int64_t N, int64_t K, int bits, uint32_t *packed)
{
    if (bits != 4 && bits != 8)
        return -1;
    int64_t per = 32 / bits;
    if (K % per)
        return -1;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t w = 0; w < K / per; ++w) {
            uint32_t word = 0;
            for (int64_t j = 0; j < per; ++j)
                word |= ((uint32_t)codes[n * K + w * per + j] & mask) << (bits * j);
            packed[n * (K / per) + w] = word;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantisation and the quantized matrix-vector product                    */
/* ------------------------------------------------------------------------ */

/* Element (n, k) of an affine-quantized matrix: scale[n][k/64]*q + bias[n][k/64]. */
static double weight_at(const uint32_t *P, const uint16_t *S, const uint16_t *Bi,
                        int64_t K, int bits, int64_t n, int64_t k)
{
    int64_t per = 32 / bits;
    int64_t G = K / 64;
    uint32_t word = P[n * (K / per) + k / per];
    uint32_t q = (word >> (bits * (k % per))) & ((1u << bits) - 1u);
    double s = or_f16_to_f64(S[n * G + k / 64]);
    double b = or_f16_to_f64(Bi[n * G + k / 64]);
    return s * (double)q + b;
}

/* Dense fp64 copy of the dequantised N x K matrix. */
int or_dequant(const uint32_t *P, const uint16_t *S, const uint16_t *Bi,
               int64_t N, int64_t K, int bits, double *W)
{
    if ((bits != 4 && bits != 8) || K % 64)
        return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            W[n * K + k] = weight_at(P, S, Bi, K, bits, n, k);
    return 0;
}

/* y[b][n] = sum_k w[n][k] * x[b][k]   (fp64, k in increasing order).
   x is given as fp64 values (exact copies of fp16 inputs, or fp64
   intermediates of a larger computation).  The scale and bias of a group are
   decoded once per (row, group); each weight is still formed as s*q + b. */
static void qmatvec_f64(const uint32_t *P, const uint16_t *S, const uint16_t *Bi,
                        int64_t N, int64_t K, int bits,
                        const double *x, int64_t B, double *y)
{
    int64_t per = 32 / bits;
    int64_t G = K / 64;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t b = 0; b < B; ++b)
        /* rows are independent: the threaded build (-fopenmp) splits them over
           threads; each row's sum keeps the index order, so the result is the
           same bit for bit */
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            const uint32_t *row = P + n * (K / per);
            double acc = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                double s = or_f16_to_f64(S[n * G + g]);
                double bias = or_f16_to_f64(Bi[n * G + g]);
                for (int64_t k = g * 64; k < g * 64 + 64; ++k) {
                    uint32_t q = (row[k / per] >> (bits * (k % per))) & mask;
                    double w = s * (double)q + bias;
                    acc += w * x[b * K + k];
                }
            }
            y[b * N + n] = acc;
        }
}

/* Affine qGEMV: x [B][K] fp16 bits, y64 [B][N] fp64 (exact-ish), y16 [B][N]
   fp16 bits (y64 rounded once, RNE).  Either output may be NULL. */
int or_qgemv(const uint32_t *P, const uint16_t *S, const uint16_t *Bi,
             int64_t N, int64_t K, int bits,
             const uint16_t *x16, int64_t B, double *y64, uint16_t *y16)
{
    if ((bits != 4 && bits != 8) || K % 64)
        return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)(B * K));
    double *y = (double *)malloc(sizeof(double) * (size_t)(B * N));
    if (!x || !y) {
        free(x);
        free(y);
        return -2;
    }
    for (int64_t i = 0; i < B * K; ++i)
        x[i] = or_f16_to_f64(x16[i]);
    qmatvec_f64(P, S, Bi, N, K, bits, x, B, y);
    for (int64_t i = 0; i < B * N; ++i) {
        if (y64)
            y64[i] = y[i];
        if (y16)
            y16[i] = or_f64_to_f16(y[i]);
    }
    free(x);
    free(y);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Format variants: zero-point 4-bit and symmetric 8-bit with bf16 scales,   */
/* and the block-32 random Hadamard rotation of the input                     */
/* ------------------------------------------------------------------------ */
/* uzu page (discuss.pytorch.kr), section "uzu의 모델 변환과 Mirai 양자화 형식":
   Mirai-M is 4-bit asymmetric integer quantisation with a 4-bit zero point
   and a bf16 scale (group 64 per the model card); Mirai-L is 8-bit symmetric;
   both quantise after a random Hadamard transform with block size 32.
   Readings (the page gives the formats by name only):
     - ZP4:  w = s * (q - z), q and z unsigned 4-bit, s bf16, one (s, z) per
             group of 64 inputs of a row;
     - SYM8: w = s * q, q a two's-complement 8-bit code, s bf16 per group;
     - per-group parameters are one uint32: bits 0..15 the bf16 scale,
       bits 16..23 the zero point (0 for SYM8);
     - rotation: the weights were quantised in the rotated basis, so the
       product is y = W_q (R x) with R = blockdiag(H_32 D / sqrt(32)),
       H_32[i][j] = (-1)^popcount(i & j) (Sylvester), D = diag(+-1) from one
       sign bit per input (bit i % 32 of word i / 32; set = -1). */

/* bf16 bit pattern -> value (exact: a bf16 is the top half of an fp32). */
double or_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int popcount32(uint32_t v)
{
    int c = 0;
    while (v) {
        c += (int)(v & 1u);
        v >>= 1;
    }
    return c;
}

/* out[b][k] = (R x)[b][k] for K inputs (K % 32 == 0); signs may be NULL
   (NULL: D = I, so R = H_32 / sqrt(32)). */
int or_rht32(const double *x, const uint32_t *signs, int64_t B, int64_t K, double *out)
{
    if (K % 32)
        return -1;
    const double inv = 1.0 / sqrt(32.0);
    for (int64_t b = 0; b < B; ++b)
        for (int64_t blk = 0; blk < K / 32; ++blk) {
            double d[32];
            for (int i = 0; i < 32; ++i) {
                int neg = signs ? (int)((signs[blk] >> i) & 1u) : 0;
                d[i] = (neg ? -1.0 : 1.0) * x[b * K + blk * 32 + i];
            }
            for (int i = 0; i < 32; ++i) {
                double acc = 0.0;
                for (int j = 0; j < 32; ++j)
                    acc += ((popcount32((uint32_t)(i & j)) & 1) ? -1.0 : 1.0) * d[j];
                out[b * K + blk * 32 + i] = acc * inv;
            }
        }
    return 0;
}

/* Element (n, k) of a format-variant matrix (format 1 = ZP4, 2 = SYM8). */
static double weight_fmt(const uint32_t *P, const uint32_t *params, int64_t K, int format,
                         int64_t n, int64_t k)
{
    int bits = format == 1 ? 4 : 8;
    int64_t per = 32 / bits;
    uint32_t word = P[n * (K / per) + k / per];
    uint32_t q = (word >> (bits * (k % per))) & ((1u << bits) - 1u);
    uint32_t prm = params[n * (K / 64) + k / 64];
    double s = or_bf16_to_f64((uint16_t)(prm & 0xFFFFu));
    if (format == 1)
        return s * ((double)q - (double)((prm >> 16) & 0xFFu));
    int sq = q >= 128u ? (int)q - 256 : (int)q;   /* two's complement */
    return s * (double)sq;
}

int or_dequant_fmt(const uint32_t *P, const uint32_t *params, int64_t N, int64_t K, int format,
                   double *W)
{
    if ((format != 1 && format != 2) || K % 64)
        return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            W[n * K + k] = weight_fmt(P, params, K, format, n, k);
    return 0;
}

/* y = W (R x) (R omitted when signs == NULL and rotate == 0), fp64, k in
   increasing order; y64 / y16 as or_qgemv. */
int or_qgemv_fmt(const uint32_t *P, const uint32_t *params, int64_t N, int64_t K, int format,
                 const uint32_t *signs, int rotate, const uint16_t *x16, int64_t B, double *y64,
                 uint16_t *y16)
{
    if ((format != 1 && format != 2) || K % 64)
        return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)(B * K));
    double *xr = (double *)malloc(sizeof(double) * (size_t)(B * K));
    if (!x || !xr) {
        free(x);
        free(xr);
        return -2;
    }
    for (int64_t i = 0; i < B * K; ++i)
        x[i] = or_f16_to_f64(x16[i]);
    if (rotate)
        or_rht32(x, signs, B, K, xr);
    else
        memcpy(xr, x, sizeof(double) * (size_t)(B * K));
    for (int64_t b = 0; b < B; ++b)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += weight_fmt(P, params, K, format, n, k) * xr[b * K + k];
            if (y64)
                y64[b * N + n] = acc;
            if (y16)
                y16[b * N + n] = or_f64_to_f16(acc);
        }
    free(x);
    free(xr);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Router: softmax, top-k, renormalisation                                   */
/* ------------------------------------------------------------------------ */

/* From one token's logits l[0..E): softmax over all E, then the k largest
   logits (ties -> lower index first) in descending order, then the selected
   probabilities divided by their sum.  Selection is on the logits; softmax
   is monotone so this is the same set as selecting on probabilities. */
static int select_topk(const double *l, int64_t E, int64_t k, int32_t *idx, double *wt)
{
    double m = -INFINITY;
    for (int64_t e = 0; e < E; ++e)
        if (l[e] > m)
            m = l[e];
    double z = 0.0;
    for (int64_t e = 0; e < E; ++e)
        z += exp(l[e] - m);
    unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
    double psum = 0.0;
    double *p = (double *)malloc(sizeof(double) * (size_t)k);
    if (!taken || !p) {
        free(taken);
        free(p);
        return -2;
    }
    for (int64_t j = 0; j < k; ++j) {
        int64_t best = -1;
        for (int64_t e = 0; e < E; ++e) {
            if (taken[e])
                continue;
            if (best < 0 || l[e] > l[best])  /* strict '>' keeps the lower index on ties */
                best = e;
        }
        taken[best] = 1;
        idx[j] = (int32_t)best;
        p[j] = exp(l[best] - m) / z;
        psum += p[j];
    }
    for (int64_t j = 0; j < k; ++j)
        wt[j] = p[j] / psum;
    free(p);
    free(taken);
    return 0;
}

/* Full router on T tokens: 8-bit (or 4-bit) affine router matrix [E][K].
   logits64 [T][E] fp64, idx [T][k], wt [T][k] fp64. */
int or_router(const uint32_t *P, const uint16_t *S, const uint16_t *Bi,
              int64_t E, int64_t K, int bits,
              const uint16_t *x16, int64_t T, int64_t k,
              double *logits64, int32_t *idx, double *wt)
{
    if ((bits != 4 && bits != 8) || K % 64 || k < 1 || k > E)
        return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)(T * K));
    if (!x)
        return -2;
    for (int64_t i = 0; i < T * K; ++i)
        x[i] = or_f16_to_f64(x16[i]);
    qmatvec_f64(P, S, Bi, E, K, bits, x, T, logits64);
    int rc = 0;
    for (int64_t t = 0; t < T && rc == 0; ++t)
        rc = select_topk(logits64 + t * E, E, k, idx + t * k, wt + t * k);
    free(x);
    return rc;
}

/* The same selection applied to given fp32 logits (e.g. a device's own). */
int or_topk_from_logits(const float *logits32, int64_t T, int64_t E, int64_t k,
                        int32_t *idx, double *wt)
{
    if (k < 1 || k > E)
        return -1;
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    if (!l)
        return -2;
    int rc = 0;
    for (int64_t t = 0; t < T && rc == 0; ++t) {
        for (int64_t e = 0; e < E; ++e)
            l[e] = (double)logits32[t * E + e];
        rc = select_topk(l, E, k, idx + t * k, wt + t * k);
    }
    free(l);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Expert MLP and the MoE layer                                              */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint32_t *packed;   /* stacked: [E][rows][cols*bits/32] */
    const uint16_t *scales;   /* [E][rows][cols/64] fp16 bits */
    const uint16_t *biases;   /* [E][rows][cols/64] fp16 bits */
} or_mat;

typedef struct {
    or_mat gate, up, down;            /* routed experts, stacked over E */
    or_mat sh_gate, sh_up, sh_down;   /* the shared expert (one matrix each) */
    int64_t E, H, I;                  /* experts, hidden size, intermediate size */
    int64_t bits;                     /* 4 */
} or_layer;

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One SwiGLU expert on one token: r = down (silu(gate x) * (up x)).
   gate/up are [I][H], down is [H][I]; x has H fp64 entries; r has H. */
static int expert_mlp(const or_mat *gate, const or_mat *up, const or_mat *down,
                      int64_t e, int64_t H, int64_t I, int bits,
                      const double *x, double *r)
{
    int64_t per = 32 / bits;
    const uint32_t *Pg = gate->packed + e * I * (H / per);
    const uint16_t *Sg = gate->scales + e * I * (H / 64);
    const uint16_t *Bg = gate->biases + e * I * (H / 64);
    const uint32_t *Pu = up->packed + e * I * (H / per);
    const uint16_t *Su = up->scales + e * I * (H / 64);
    const uint16_t *Bu = up->biases + e * I * (H / 64);
    const uint32_t *Pd = down->packed + e * H * (I / per);
    const uint16_t *Sd = down->scales + e * H * (I / 64);
    const uint16_t *Bd = down->biases + e * H * (I / 64);
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    if (!g || !u || !h) {
        free(g);
        free(u);
        free(h);
        return -2;
    }
    qmatvec_f64(Pg, Sg, Bg, I, H, bits, x, 1, g);
    qmatvec_f64(Pu, Su, Bu, I, H, bits, x, 1, u);
    for (int64_t i = 0; i < I; ++i)
        h[i] = silu(g[i]) * u[i];
    qmatvec_f64(Pd, Sd, Bd, H, I, bits, h, 1, r);
    free(g);
    free(u);
    free(h);
    return 0;
}

/* Routed expert e of the layer on one fp16 token (exposed for composition
   tests).  r has H fp64 entries.  e < 0 selects the shared expert. */
int or_expert(const or_layer *L, int64_t e, const uint16_t *x16, double *r)
{
    if (L->H % 64 || L->I % 64 || e >= L->E)
        return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)L->H);
    if (!x)
        return -2;
    for (int64_t i = 0; i < L->H; ++i)
        x[i] = or_f16_to_f64(x16[i]);
    int rc;
    if (e < 0)
        rc = expert_mlp(&L->sh_gate, &L->sh_up, &L->sh_down, 0, L->H, L->I, (int)L->bits, x, r);
    else
        rc = expert_mlp(&L->gate, &L->up, &L->down, e, L->H, L->I, (int)L->bits, x, r);
    free(x);
    return rc;
}

/* MoE layer on T tokens with given routing: y[t] = shared(x_t) +
   sum_j wt[t][j] * expert_{idx[t][j]}(x_t).  idx [T][k], wt [T][k] fp64.
   y64 [T][H] fp64 and/or y16 [T][H] fp16 bits (rounded once). */
int or_moe_layer(const or_layer *L, const uint16_t *x16, int64_t T,
                 const int32_t *idx, const double *wt, int64_t k,
                 double *y64, uint16_t *y16)
{
    int64_t H = L->H;
    if (H % 64 || L->I % 64)
        return -1;
    for (int64_t i = 0; i < T * k; ++i)
        if (idx[i] < 0 || idx[i] >= L->E)
            return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)H);
    double *r = (double *)malloc(sizeof(double) * (size_t)H);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    int rc = (x && r && y) ? 0 : -2;
    for (int64_t t = 0; t < T && rc == 0; ++t) {
        for (int64_t i = 0; i < H; ++i)
            x[i] = or_f16_to_f64(x16[t * H + i]);
        rc = expert_mlp(&L->sh_gate, &L->sh_up, &L->sh_down, 0, H, L->I, (int)L->bits, x, y);
        for (int64_t j = 0; j < k && rc == 0; ++j) {
            rc = expert_mlp(&L->gate, &L->up, &L->down, idx[t * k + j], H, L->I, (int)L->bits,
                            x, r);
            for (int64_t i = 0; i < H && rc == 0; ++i)
                y[i] += wt[t * k + j] * r[i];
        }
        for (int64_t i = 0; i < H && rc == 0; ++i) {
            if (y64)
                y64[t * H + i] = y[i];
            if (y16)
                y16[t * H + i] = or_f64_to_f16(y[i]);
        }
    }
    free(x);
    free(r);
    free(y);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Prefill grouping: tokens of a chunk listed per expert                     */
/* ------------------------------------------------------------------------ */

/* counts[e] = number of (token, slot) pairs routed to e; offsets[0..E] the
   exclusive prefix sum; pairs[offsets[e] .. offsets[e+1]) the flat indices
   t*k + j of those pairs, ascending (i.e. by token, then slot). */
int or_group(const int32_t *idx, int64_t T, int64_t k, int64_t E,
             int32_t *counts, int32_t *offsets, int32_t *pairs)
{
    for (int64_t e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t i = 0; i < T * k; ++i) {
        if (idx[i] < 0 || idx[i] >= E)
            return -1;
        counts[idx[i]] += 1;
    }
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!fill)
        return -2;
    for (int64_t e = 0; e < E; ++e)
        fill[e] = offsets[e];
    for (int64_t i = 0; i < T * k; ++i)
        pairs[fill[idx[i]]++] = (int32_t)i;
    free(fill);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Expert cache: the per-layer 16-slot LFU plan                               */
/* ------------------------------------------------------------------------ */
/* TurboFieldfare article, section "내부 구조가 진짜 흥미로운 부분": the CPU
   takes the router's top-8 expert ids and plans the misses against the
   layer's 16-slot LFU cache; missed experts are read into the cache before
   the routed experts run.
   Readings (the page names the policy only):
     - a slot holds one expert and a use count; a hit adds one to the count;
       an expert loaded on a miss starts at one; an evicted expert's count is
       forgotten;
     - the token's hits are found first (they stay), then its misses are
       placed in the order the ids are given: into the lowest-index empty
       slot, else into the unpinned slot with the smallest count, ties to the
       lowest index (slots holding an expert of this token are pinned).
   One step: slot_of[j] = slot of ids[j]; misses listed in order as
   (expert, slot) pairs; returns the number of misses, or -1 if k > nslots,
   nslots is outside 1..256, or the ids repeat. */
int64_t or_lfu_step(int64_t nslots, int32_t *slot_expert, int64_t *slot_count,
                    const int32_t *ids, int64_t k, int32_t *slot_of, int32_t *miss_expert,
                    int32_t *miss_slot)
{
    if (k > nslots || nslots < 1 || nslots > 256)   /* the pinned flags hold 256 slots */
        return -1;
    for (int64_t a = 0; a < k; ++a)
        for (int64_t b = a + 1; b < k; ++b)
            if (ids[a] == ids[b])
                return -1;
    int pinned[256];
    for (int64_t s = 0; s < nslots; ++s)
        pinned[s] = 0;
    for (int64_t j = 0; j < k; ++j) {
        slot_of[j] = -1;
        for (int64_t s = 0; s < nslots; ++s)
            if (slot_expert[s] == ids[j]) {
                slot_of[j] = (int32_t)s;
                slot_count[s] += 1;
                pinned[s] = 1;
            }
    }
    int64_t nm = 0;
    for (int64_t j = 0; j < k; ++j) {
        if (slot_of[j] >= 0)
            continue;
        int64_t v = -1;
        for (int64_t s = 0; s < nslots && v < 0; ++s)
            if (slot_expert[s] < 0 && !pinned[s])
                v = s;
        if (v < 0)
            for (int64_t s = 0; s < nslots; ++s)
                if (!pinned[s] && (v < 0 || slot_count[s] < slot_count[v]))
                    v = s;
        slot_expert[v] = ids[j];
        slot_count[v] = 1;
        pinned[v] = 1;
        slot_of[j] = (int32_t)v;
        miss_expert[nm] = ids[j];
        miss_slot[nm] = (int32_t)v;
        ++nm;
    }
    return nm;
}

