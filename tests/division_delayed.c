/*
 * division_delayed.c -- host check of the division used by the delayed-scaling
 * quantiser kernel.  There the scale s is the previous step's scale (any positive
 * normal fp32) and x any bf16 value, so the quotient may exceed Fmax by any amount
 * (clipped elements) or overflow fp32.  The kernel computes
 *     pre = 2^64 if s < 2^-64, 2^-64 if s >= 2^64, else 1;   s' = s * pre,   r = RN(1 / s')
 *     x' = x * pre,  q0 = RN(x' r)
 *     q  = q0                          if |q0| >= 2^100 (saturates either way)
 *        = fma(fma(-q0, s', x'), r, q0) otherwise (Markstein's correction),
 *     with the sign of x copied onto q,
 * then code = the FP8 code of q and clipped = |q| > Fmax.  Both must equal what the
 * IEEE quotient fl32(x / s) gives (encoded by the oracle's encoder): for every
 * finite bf16 x, both signs, and a stratified set of scales -- every binary exponent
 * from -126 to 127 with 8 significands each (the power of two, the largest
 * significand and 6 seeded ones).  Test-side code, run by
 * tests/test_division_identity.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

uint8_t orc_encode(float x, int fmt);

static float bf(uint32_t h) { uint32_t u = h << 16; float f; memcpy(&f, &u, 4); return f; }
static float f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

#define NT 8
typedef struct { int t, fmt; float fmax; long long pairs, bad_code, bad_clip; } Job;

static void *run(void *p) {
    Job *j = (Job *)p;
    uint32_t lcg = 12345u + 977u * (uint32_t)j->t;
    for (int ex = 1; ex <= 254; ++ex) {
        if ((ex % NT) != j->t) continue;
        for (int mi = 0; mi < 8; ++mi) {
            uint32_t mant;
            if (mi == 0) mant = 0;
            else if (mi == 1) mant = 0x7FFFFFu;
            else { lcg = lcg * 1664525u + 1013904223u; mant = lcg >> 9; }
            const float s = f32(((uint32_t)ex << 23) | mant);
            const float pre = (s < 0x1p-64f) ? 0x1p64f : (s >= 0x1p64f ? 0x1p-64f : 1.0f);
            const float ss = s * pre, r = 1.0f / ss;
            for (uint32_t hx = 0; hx < 0x7F80; ++hx) {
                const float x = bf(hx);
                for (int sg = 0; sg < 2; ++sg) {
                    const float xv = sg ? -x : x;
                    const float xs = xv * pre;
                    const float q0 = xs * r;
                    float q;
                    if (fabsf(q0) >= 0x1p100f) q = q0;
                    else q = copysignf(fmaf(fmaf(-q0, ss, xs), r, q0), xv);
                    const float qi = xv / s;
                    j->pairs++;
                    if (orc_encode(q, j->fmt) != orc_encode(qi, j->fmt)) {
                        if (j->bad_code < 3) fprintf(stderr, "code fmt=%d s=%a x=%a\n", j->fmt, s, xv);
                        j->bad_code++;
                    }
                    if ((fabsf(q) > j->fmax) != (fabsf(qi) > j->fmax)) {
                        if (j->bad_clip < 3) fprintf(stderr, "clip fmt=%d s=%a x=%a\n", j->fmt, s, xv);
                        j->bad_clip++;
                    }
                }
            }
        }
    }
    return NULL;
}

int main(void) {
    const float fmaxes[2] = {448.0f, 57344.0f};
    long long total_bad = 0;
    for (int f = 0; f < 2; ++f) {
        pthread_t th[NT];
        Job jobs[NT];
        for (int t = 0; t < NT; ++t) {
            jobs[t] = (Job){t, f, fmaxes[f], 0, 0, 0};
            pthread_create(&th[t], NULL, run, &jobs[t]);
        }
        long long pairs = 0, bc = 0, bl = 0;
        for (int t = 0; t < NT; ++t) {
            pthread_join(th[t], NULL);
            pairs += jobs[t].pairs; bc += jobs[t].bad_code; bl += jobs[t].bad_clip;
        }
        printf("fmt=%d pairs=%lld code_mismatches=%lld clip_mismatches=%lld\n", f, pairs, bc, bl);
        total_bad += bc + bl;
    }
    return total_bad != 0;
}
