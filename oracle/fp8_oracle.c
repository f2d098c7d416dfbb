/*
 * fp8_oracle.c -- plain, slow, scalar CPU oracle for the FP8 W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU baseline leg of
 * the benchmark do.  It shares no code, header, table or constant generator with
 * the CUDA library: every formula below is written out again from the pages.
 *
 * Sources (page title, then the section the step follows):
 *  [P1] "ROCm 7 原生 FP8/MXFP8 ... AITER" (devpress.csdn.net), section 1.1 table
 *       (E4M3 range +-448, E5M2 range +-57344) and section 4.3 "延迟缩放"
 *       (divide by the scale, clamp to +-448, cast to float8_e4m3fn).
 *  [P2] "LLM 推理的 FP8 混合精度工程 2026" (blog.lonae.com), section 2, the
 *       quantisation operator Q(x) = clamp(round(x*s), -Fmax, Fmax) * s^-1 with
 *       Fmax = 448 (E4M3) / 57344 (E5M2); section 3, FP32 accumulation of FP8
 *       products.
 *  [P3] "FP8 推理" (luoboask.github.io), "Dynamic Scaling": FP8 = FP32 / scale,
 *       scale = max(|tensor|) / 448.
 *  [P4] "FP8 推理提速 83.6%: DeepSeek-V3 在 AMD MI250 上的完整落地指南" (xdnf.cn),
 *       "FP8 权重转换命令与关键配置参数" (e4m3 weights with 128x128 block
 *       scale_inv; scale_fmt ue8m0) and "运行时" (act_quant per token per 128
 *       channels, then fp8_gemm(x, scale, weight, weight.scale)).
 *  [P5] "量化：FP8 与混合精度推理" (charles2530.github.io), "FP8 也需要 scale":
 *       x_fp8 = FP8Cast(x / s), x_hat = s * x_fp8.
 *  [P1] section 1.2 also fixes the microscaling variant: MXFP8 splits a tensor
 *       into blocks of 32 elements, each with its own scale factor, and the
 *       format table of section 1.1 lists MXFP8 as 8 bits plus a shared exponent.
 *
 * Readings taken where the pages are silent or disagree (scale direction: [P3]
 * and [P5] divide where [P2] multiplies; the rest is not stated on any page):
 *  - the scale divides (x / s), it is stored as the dequantisation multiplier;
 *  - the division x / s is one IEEE fp32 division, then round-to-nearest-even
 *    to FP8 with saturation to +-Fmax (no Inf is ever produced);
 *  - s = max(fl32(amax / Fmax), 2^-126); ue8m0 rounds fl32(amax / Fmax) up to
 *    a power of two 2^e with e >= -126;
 *  - a negative value that rounds to zero keeps its sign (code 0x80);
 *  - NaN inputs are ignored by amax and encode as 0x7F.
 *
 * Build: gcc -O1 -std=c99 -fPIC -shared -ffp-contract=off (no fast-math), so
 * every float operation below is one correctly rounded IEEE operation.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>

#define ORC_E4M3 0
#define ORC_E5M2 1
#define ORC_SCALE_FP32 0
#define ORC_SCALE_UE8M0 1

/* ------------------------------------------------------------------ codec */

/* Decode one FP8 code.  [P1] 1.1 / [P2] 2: E4M3 = 1 sign, 4 exponent (bias 7),
 * 3 mantissa bits, largest finite 448, no infinity, S.1111.111 is NaN.
 * E5M2 = 1 sign, 5 exponent (bias 15), 2 mantissa bits, largest finite 57344,
 * exponent 31 is Inf (mantissa 0) or NaN. */
double orc_decode(uint8_t code, int fmt)
{
    int neg = code >> 7;
    double v;
    if (fmt == ORC_E4M3) {
        int e = (code >> 3) & 15, m = code & 7;
        if (e == 15 && m == 7) return NAN;
        if (e == 0) v = ldexp((double)m, -9);            /* (m/8) * 2^(1-7)   */
        else        v = ldexp((double)(8 + m), e - 10);  /* (1+m/8) * 2^(e-7) */
    } else {
        int e = (code >> 2) & 31, m = code & 3;
        if (e == 31) return m == 0 ? (neg ? -INFINITY : INFINITY) : NAN;
        if (e == 0) v = ldexp((double)m, -16);           /* (m/4) * 2^(1-15)  */
        else        v = ldexp((double)(4 + m), e - 17);  /* (1+m/4) * 2^(e-15) */
    }
    return neg ? -v : v;
}

/* Largest finite code below the sign bit: 0x7E (448) for E4M3, 0x7B (57344)
 * for E5M2.  Non-negative finite codes are 0 .. top and increase with the code. */
static int top_code(int fmt) { return fmt == ORC_E4M3 ? 0x7E : 0x7B; }

double orc_fmax(int fmt) { return orc_decode((uint8_t)top_code(fmt), fmt); }

/* Values of the non-negative finite codes 0 .. top of each format, filled once
 * by the decoder above (no constants are typed in). */
static double g_tab[2][128];
static int g_tab_ready[2];

static const double *value_table(int fmt)
{
    if (!g_tab_ready[fmt]) {
        for (int c = 0; c <= top_code(fmt); ++c) g_tab[fmt][c] = orc_decode((uint8_t)c, fmt);
        g_tab_ready[fmt] = 1;
    }
    return g_tab[fmt];
}

/* Encode one fp32 value: the nearest FP8 value, ties to the code with an even
 * mantissa, anything at or beyond Fmax (including Inf) clamps to Fmax ([P1] 4.3
 * clamp-then-cast, [P2] 2 clamp(round(.))).  A binary search finds the two
 * neighbouring table values; the distances are exact in double. */
uint8_t orc_encode(float x, int fmt)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    int top = top_code(fmt);
    const double *tab = value_table(fmt);
    if (a >= tab[top]) return (uint8_t)(sign | top);
    int lo = 0, hi = top;                  /* invariant: tab[lo] <= a < tab[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (tab[mid] <= a) lo = mid; else hi = mid;
    }
    double dlo = a - tab[lo];              /* exact: Sterbenz, or tab[lo] == 0 */
    double dhi = tab[hi] - a;
    int c;
    if (dlo < dhi) c = lo;
    else if (dhi < dlo) c = hi;
    else c = (lo & 1) ? hi : lo;           /* tie: even mantissa LSB */
    return (uint8_t)(sign | c);
}

/* ------------------------------------------------------------------ scales */

/* Group / block / tensor scale from its amax.  [P3] Dynamic Scaling:
 * scale = amax / Fmax.  FP32 format: the quotient in IEEE fp32, floored at
 * 2^-126 so an all-zero group never divides by zero.  UE8M0 ([P4] scale_fmt):
 * the same quotient rounded UP to a power of two, exponent >= -126. */
float orc_scale_from_amax(float amax, int fmt, int scale_fmt)
{
    float fmax = (float)orc_fmax(fmt);
    float v = amax / fmax;
    if (scale_fmt == ORC_SCALE_FP32) {
        return v < 0x1p-126f ? 0x1p-126f : v;
    }
    int e;
    if (v == 0.0f) {
        e = -126;
    } else {
        int p;
        double m = frexp((double)v, &p);   /* v = m * 2^p, m in [0.5, 1) */
        e = (m == 0.5) ? p - 1 : p;        /* ceil(log2 v) */
        if (e < -126) e = -126;
    }
    return ldexpf(1.0f, e);
}

/* bf16 bit pattern -> fp32 (exact: bf16 is the top half of an fp32). */
static float bf16_to_f32(uint16_t h)
{
    union { uint32_t u; float f; } c;
    c.u = (uint32_t)h << 16;
    return c.f;
}

/* |x| max over a set of bf16 values; NaN never wins a comparison. */
static float amax_accum(float amax, float x)
{
    float a = fabsf(x);
    return a > amax ? a : amax;
}

/* --------------------------------------------------------------- quantisers */

/* Per-token, per-group activation quantisation ([P4] 运行时 act_quant; [P2] 4
 * per-block activation scales of 128 elements).  x is [M][ldx] bf16, q is
 * [M][K] codes, s is [M][ceil(K/group)] scales.  The last group of a row may
 * be short; its amax covers only the valid elements. */
void orc_act_quant(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                   int64_t group, int fmt, int scale_fmt,
                   uint8_t *q, float *s)
{
    int64_t ng = (K + group - 1) / group;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < ng; ++g) {
            int64_t k0 = g * group, k1 = k0 + group < K ? k0 + group : K;
            float amax = 0.0f;
            for (int64_t k = k0; k < k1; ++k)
                amax = amax_accum(amax, bf16_to_f32(x[m * ldx + k]));
            float sc = orc_scale_from_amax(amax, fmt, scale_fmt);
            s[m * ng + g] = sc;
            for (int64_t k = k0; k < k1; ++k) {
                float t = bf16_to_f32(x[m * ldx + k]) / sc;   /* one IEEE division */
                q[m * K + k] = orc_encode(t, fmt);
            }
        }
    }
}

/* 128x128 block weight quantisation ([P4] FP8 权重转换: e4m3 weights with a
 * 128x128 block scale_inv).  w is [N][K] bf16 (row stride K), q is [N][K],
 * s_inv is [ceil(N/block)][ceil(K/block)]. */
void orc_weight_quant_block(const uint16_t *w, int64_t N, int64_t K, int64_t block,
                            int fmt, int scale_fmt, uint8_t *q, float *s_inv)
{
    int64_t nbn = (N + block - 1) / block, nbk = (K + block - 1) / block;
    for (int64_t bn = 0; bn < nbn; ++bn) {
        for (int64_t bk = 0; bk < nbk; ++bk) {
            int64_t n0 = bn * block, n1 = n0 + block < N ? n0 + block : N;
            int64_t k0 = bk * block, k1 = k0 + block < K ? k0 + block : K;
            float amax = 0.0f;
            for (int64_t n = n0; n < n1; ++n)
                for (int64_t k = k0; k < k1; ++k)
                    amax = amax_accum(amax, bf16_to_f32(w[n * K + k]));
            float sc = orc_scale_from_amax(amax, fmt, scale_fmt);
            s_inv[bn * nbk + bk] = sc;
            for (int64_t n = n0; n < n1; ++n)
                for (int64_t k = k0; k < k1; ++k)
                    q[n * K + k] = orc_encode(bf16_to_f32(w[n * K + k]) / sc, fmt);
        }
    }
}

/* The cast step under a given scale: q[i] = FP8Cast(x[i] / s) ([P5] FP8 也需要
 * scale), one IEEE fp32 division then the encoder above. */
void orc_cast_with_scale(const uint16_t *x, int64_t n, float s, int fmt, uint8_t *q)
{
    for (int64_t i = 0; i < n; ++i) q[i] = orc_encode(bf16_to_f32(x[i]) / s, fmt);
}

/* Per-tensor quantisation ([P1] 1.2 OCP-FP8 one scale per tensor; [P3] scale =
 * max(|tensor|)/448; [P2] Fmax 57344 for E5M2).  One scale for all n elements. */
void orc_tensor_quant(const uint16_t *x, int64_t n, int fmt, int scale_fmt,
                      uint8_t *q, float *s)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) amax = amax_accum(amax, bf16_to_f32(x[i]));
    float sc = orc_scale_from_amax(amax, fmt, scale_fmt);
    s[0] = sc;
    orc_cast_with_scale(x, n, sc, fmt, q);
}

/* -------------------------------------------------------------------- GEMM */

/* Block-scaled GEMM, selected rows ([P4] 运行时 fp8_gemm(x, scale, weight,
 * weight.scale); [P5] x_hat = s * x_fp8; [P2] 3 FP32 accumulation):
 *   y[m][n] = sum_k (dec(qa[m][k]) * sa[m][k/128]) * (dec(qw[n][k]) * sw[n/128][k/128])
 * summed in fp64 in k order.  bound[m][n] = sum_k |a_k * w_k| (the tolerance
 * scale).  rows lists the nr rows to compute; outputs are [nr][N]. */
/* Decoded value of every E4M3 code, filled once by orc_decode so the GEMM's inner
 * loop looks values up instead of re-deriving them (same doubles, fewer calls). */
static double g_dec_e4m3[256];
static int g_dec_ready;

static const double *e4m3_values(void)
{
    if (!g_dec_ready) {
        for (int c = 0; c < 256; ++c) g_dec_e4m3[c] = orc_decode((uint8_t)c, ORC_E4M3);
        g_dec_ready = 1;
    }
    return g_dec_e4m3;
}

void orc_gemm_rows(const uint8_t *qa, const float *sa, const uint8_t *qw, const float *sw,
                   int64_t N, int64_t K, const int64_t *rows, int64_t nr,
                   double *y, double *bound)
{
    const int64_t nkb = K / 128;
    const double *dec = e4m3_values();
    for (int64_t i = 0; i < nr; ++i) {
        int64_t m = rows[i];
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, b = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double a = dec[qa[m * K + k]] * (double)sa[m * nkb + k / 128];
                double w = dec[qw[n * K + k]] * (double)sw[(n / 128) * nkb + k / 128];
                acc += a * w;
                b += fabs(a * w);
            }
            y[i * N + n] = acc;
            bound[i * N + n] = b;
        }
    }
}

/* Grouped (MoE expert) GEMM, selected rows: row m belongs to the expert e with
 * off[e] <= m < off[e+1] and uses that expert's weights qw[e] ([N][K]) and
 * scales sw[e] ([N/128][K/128]).  Rows outside every group get y = 0. */
void orc_grouped_gemm_rows(const uint8_t *qa, const float *sa, const uint8_t *qw,
                           const float *sw, const int32_t *off, int64_t E,
                           int64_t N, int64_t K, const int64_t *rows, int64_t nr,
                           double *y, double *bound)
{
    const int64_t nkb = K / 128, nbn = (N + 127) / 128;
    for (int64_t i = 0; i < nr; ++i) {
        int64_t m = rows[i], e = -1;
        for (int64_t j = 0; j < E; ++j)
            if (off[j] <= m && m < off[j + 1]) { e = j; break; }
        if (e < 0) {
            for (int64_t n = 0; n < N; ++n) { y[i * N + n] = 0.0; bound[i * N + n] = 0.0; }
            continue;
        }
        orc_gemm_rows(qa, sa, qw + e * N * K, sw + e * nbn * nkb, N, K, &m, 1,
                      y + i * N, bound + i * N);
    }
}

/* ---------------------------------------------------------------- rounding */

/* Round a double straight to bf16 (8-bit significand), ties to even, with
 * gradual underflow; no intermediate fp32 rounding.  Used to state the bf16
 * output the oracle expects. */
uint16_t orc_round_bf16(double v)
{
    union { uint32_t u; float f; } c;
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    if (a == 0.0) return sign;
    int p;
    frexp(a, &p);                          /* a in [2^(p-1), 2^p) */
    int q = p - 1 - 7;                     /* quantum exponent for a normal bf16 */
    if (q < -133) q = -133;                /* subnormal quantum 2^-133 */
    double r = nearbyint(ldexp(a, -q));    /* exact scaling; RNE (default mode) */
    double out = ldexp(r, q);
    if (out > 0x1.FEp127) return sign | 0x7F80;   /* overflow -> Inf */
    c.f = (float)out;                      /* exact: out is a bf16 value */
    return (uint16_t)(sign | (c.u >> 16));
}

/* ------------------------------------------------------------- MXFP8 ([P1] 1.2) */

/* Value of an E8M0 shared-exponent byte: 2^(b - 127); the byte 0xFF is NaN.
 * (An E8M0 number has 8 exponent bits, no sign and no mantissa.) */
double orc_e8m0_decode(uint8_t b)
{
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* MXFP8 quantisation of bf16 x [M][ldx] in blocks of `block` (32) consecutive
 * elements of a row ([P1] 1.2: 32-element blocks with their own scale; 1.1: a
 * shared exponent).  The pages do not say how the shared exponent follows from
 * the block; the reading taken is the power-of-two rule the pages fix for
 * scale_fmt ue8m0 ([P4]), applied per block: s = 2^ceil(log2(amax / Fmax)),
 * e >= -126, so that no element saturates.  The exponent is stored as the E8M0
 * byte e + 127 in e8 [M][ceil(K/block)]; codes are the cast of x / s. */
void orc_mx_quant(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, int64_t block,
                  int fmt, uint8_t *q, uint8_t *e8)
{
    int64_t nb = (K + block - 1) / block;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < nb; ++g) {
            int64_t k0 = g * block, k1 = k0 + block < K ? k0 + block : K;
            float amax = 0.0f;
            for (int64_t k = k0; k < k1; ++k)
                amax = amax_accum(amax, bf16_to_f32(x[m * ldx + k]));
            float sc = orc_scale_from_amax(amax, fmt, ORC_SCALE_UE8M0);
            int p;
            double mant = frexp((double)sc, &p);   /* sc = 0.5 * 2^p exactly */
            (void)mant;
            e8[m * nb + g] = (uint8_t)(p - 1 + 127);
            for (int64_t k = k0; k < k1; ++k)
                q[m * K + k] = orc_encode(bf16_to_f32(x[m * ldx + k]) / sc, fmt);
        }
    }
}

/* MXFP8 GEMM, selected rows: every element of either operand carries the E8M0
 * scale of its own 32-element block along K,
 *   y[m][n] = sum_k dec(qa[m][k]) 2^(ea[m][k/32]-127) * dec(qw[n][k]) 2^(ew[n][k/32]-127)
 * summed in fp64 in k order; bound[m][n] = sum_k |a_k w_k|.  qa [.][K], ea
 * [.][K/32], qw [N][K], ew [N][K/32], K % 32 == 0. */
void orc_mx_gemm_rows(const uint8_t *qa, const uint8_t *ea, const uint8_t *qw, const uint8_t *ew,
                      int64_t N, int64_t K, const int64_t *rows, int64_t nr,
                      double *y, double *bound)
{
    const int64_t nb = K / 32;
    const double *dec = e4m3_values();
    for (int64_t i = 0; i < nr; ++i) {
        int64_t m = rows[i];
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, b = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double a = dec[qa[m * K + k]] * orc_e8m0_decode(ea[m * nb + k / 32]);
                double w = dec[qw[n * K + k]] * orc_e8m0_decode(ew[n * nb + k / 32]);
                acc += a * w;
                b += fabs(a * w);
            }
            y[i * N + n] = acc;
            bound[i * N + n] = b;
        }
    }
}

/* ----------------------------------------------- delayed scaling ([P1] 4.3, 6) */

/* One step of delayed per-tensor scaling as the ROCm/AITER page describes it
 * ([P1] 4.3 "延迟缩放", the FP8DelayedScaling listing; [P1] section 6, amax history
 * length and "max" over the history):
 *   1. the tensor is divided by the scale of the PREVIOUS step (*scale; the page
 *      starts from 1.0), clamped to +-Fmax and cast -- q[i] = enc(x[i] / s_prev);
 *      elements whose quotient lies beyond +-Fmax are the clipped ones the page's
 *      checklist asks to count ("FP8 溢出率": *n_clipped);
 *   2. the current amax max|x| goes into the history ring at slot *pos;
 *   3. the next step's scale is (max over the history if algo == 1, else the amax
 *      just recorded) / target, target = 400 for E4M3 on the page (a margin below
 *      448), floored at 2^-126 (reading shared with the other quantisers: a zero
 *      amax must not give a zero divisor); the slot after *pos is cleared for the
 *      next step and *pos advances.
 * *s_used receives the scale the codes were made with (x ~= dec(q) * s_used).
 * The history holds non-negative amaxes; zeros are slots not yet filled. */
void orc_delayed_quant(const uint16_t *x, int64_t n, int fmt, float target, int64_t hist_len,
                       int algo, float *scale, int32_t *pos, float *history,
                       uint8_t *q, uint64_t *n_clipped, float *s_used)
{
    const double fmax = orc_fmax(fmt);
    const float s_prev = *scale;
    uint64_t clipped = 0;
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float v = bf16_to_f32(x[i]);
        float t = v / s_prev;                  /* one IEEE division */
        if (fabs((double)t) > fmax) ++clipped;
        q[i] = orc_encode(t, fmt);             /* clamp to +-Fmax, then round */
        amax = amax_accum(amax, v);
    }
    *n_clipped = clipped;
    *s_used = s_prev;
    int32_t p = *pos;
    history[p] = amax;
    float a = amax;
    if (algo == 1)
        for (int64_t h = 0; h < hist_len; ++h) a = history[h] > a ? history[h] : a;
    float s_next = a / target;
    *scale = s_next < 0x1p-126f ? 0x1p-126f : s_next;
    p = (int32_t)((p + 1) % hist_len);
    history[p] = 0.0f;
    *pos = p;
}

/* ------------------------------------------------------ weight dequantisation */

/* The BF16 path of the DeepSeek-V3 page ([P4] 运行时: weight = weight_dequant(weight,
 * weight.scale), then a plain GEMM; FP8 权重转换: fp8_cast_bf16.py turns the FP8
 * checkpoint into BF16): w[n][k] = dec(q[n][k]) * s_inv[n/block][k/block] formed as one
 * IEEE fp32 product (the reading taken: the codes are widened to fp32 and multiplied
 * by the fp32 scale, as a GEMM input would be), then rounded to bf16 to nearest even.
 * block == 0 uses the single per-tensor scale s_inv[0].  out holds bf16 bit patterns. */
void orc_weight_dequant(const uint8_t *q, const float *s_inv, int64_t N, int64_t K, int64_t block,
                        int fmt, uint16_t *out)
{
    int64_t nbk = block > 0 ? (K + block - 1) / block : 1;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            float s = block > 0 ? s_inv[(n / block) * nbk + k / block] : s_inv[0];
            float v = (float)orc_decode(q[n * K + k], fmt) * s;     /* one fp32 rounding */
            out[n * K + k] = orc_round_bf16((double)v);             /* exact widening, one bf16 rounding */
        }
    }
}

/* ------------------------------------------------------------ MoE routing */

/* Routing and permutation around the grouped GEMM ([P4] 官方配置中最关键的四个参数:
 * 256 routed experts, n_activated_experts = 8 per token; [P1] 2.3 block-scale fused
 * MoE).  The pages fix only the counts; the reading taken is the plainest one:
 *   - each token selects the k experts of largest score (non-negative affinities,
 *     e.g. sigmoid outputs), in descending score order, a tie going to the lower
 *     expert index;
 *   - its gate weights are the selected scores normalised to sum 1: sum = s_0 + ... +
 *     s_{k-1} accumulated in fp32 in selection order, w_j = fl32(s_j / sum); if the sum
 *     is 0 every weight is fl32(1 / k);
 *   - the (token, j) pairs are sorted by (expert, token) -- stable, each token picks an
 *     expert at most once -- giving offsets [E+1] (rows of expert e are
 *     [off[e], off[e+1])), row_token / row_weight of every sorted row, and token_row,
 *     the sorted row of pair (t, j).
 * ids / w are [T][k]; row_token, row_weight, token_row are [T*k]. */
void orc_moe_route(const float *scores, int64_t T, int64_t E, int64_t k, int32_t *ids, float *w,
                   int32_t *offsets, int32_t *row_token, float *row_weight, int32_t *token_row)
{
    for (int64_t t = 0; t < T; ++t) {
        const float *s = scores + t * E;
        float sum = 0.0f;
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                int taken = 0;
                for (int64_t i = 0; i < j; ++i) taken |= (ids[t * k + i] == (int32_t)e);
                if (taken) continue;
                if (best < 0 || s[e] > s[best]) best = e;      /* strict: ties keep the lower index */
            }
            ids[t * k + j] = (int32_t)best;
            sum += s[best];
        }
        for (int64_t j = 0; j < k; ++j)
            w[t * k + j] = sum == 0.0f ? 1.0f / (float)k : s[ids[t * k + j]] / sum;
    }
    for (int64_t e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t i = 0; i < T * k; ++i) offsets[ids[i] + 1] += 1;
    for (int64_t e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    for (int64_t e = 0; e < E; ++e) {                     /* stable: pairs visited in (t, j) order */
        int32_t pos = offsets[e];
        for (int64_t t = 0; t < T; ++t)
            for (int64_t j = 0; j < k; ++j)
                if (ids[t * k + j] == (int32_t)e) {
                    row_token[pos] = (int32_t)t;
                    row_weight[pos] = w[t * k + j];
                    token_row[t * k + j] = pos;
                    ++pos;
                }
    }
}

/* MoE output of selected tokens ([P1] 2.3 fused MoE: expert GEMMs then the gate-weighted
 * sum): out[t][n] = sum_j w[t][j] * y_j[n], y_j = the block-scaled GEMM of token t's
 * activation row (qa / sa rows are token-major [T][K]) with expert ids[t][j]'s weights
 * qw[e] [N][K], sw[e] [N/128][K/128]; fp64, j in order.  bound[t][n] = sum_j |w_j| *
 * sum_k |a_k w_k| of that expert (the GEMM tolerance scale). */
void orc_moe_combine_rows(const uint8_t *qa, const float *sa, const uint8_t *qw, const float *sw,
                          const int32_t *ids, const float *w, int64_t k, int64_t N, int64_t K,
                          const int64_t *tokens, int64_t nt, double *out, double *bound)
{
    const int64_t nkb = K / 128, nbn = (N + 127) / 128;
    double *y = (double *)malloc(sizeof(double) * (size_t)N);
    double *b = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t i = 0; i < nt; ++i) {
        int64_t t = tokens[i];
        for (int64_t n = 0; n < N; ++n) { out[i * N + n] = 0.0; bound[i * N + n] = 0.0; }
        for (int64_t j = 0; j < k; ++j) {
            int64_t e = ids[t * k + j];
            orc_gemm_rows(qa, sa, qw + e * N * K, sw + e * nbn * nkb, N, K, &t, 1, y, b);
            for (int64_t n = 0; n < N; ++n) {
                out[i * N + n] += (double)w[t * k + j] * y[n];
                bound[i * N + n] += fabs((double)w[t * k + j]) * b[n];
            }
        }
    }
    free(y);
    free(b);
}
