/*
 * division_identity.c -- checks, on the CPU, the division the quantiser kernels use
 * in place of an IEEE fp32 division (see GroupScale in the CUDA sources): for a
 * group scale s = max(fl32(amax / Fmax), 2^-126),
 *     pre = 2^64 if s < 2^-64 else 1,   s' = s * pre,   r = RN(1 / s')
 *     x' = x * pre,  q0 = RN(x' r),  e = fma(-q0, s', x'),  q = fma(e, r, q0)
 *     with the sign of x copied onto q
 * and the FP8 code of q must equal the FP8 code of the IEEE quotient fl32(x / s),
 * both encoded by the oracle's encoder, for every bf16 x with |x| <= amax.
 * Test-side code: it restates that arithmetic (fmaf and IEEE division of the host
 * C library) and is built and run by tests/test_division_identity.py only.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

uint8_t orc_encode(float x, int fmt);

static float bf(uint32_t h) { uint32_t u = h << 16; float f; memcpy(&f, &u, 4); return f; }

typedef struct { int t, nt, fmt, stride; float fmax; long long pairs, bad; } Job;

static int selected(uint32_t ha, int stride) {
    uint32_t ex = (ha >> 7) & 0xFF;
    if (stride <= 1) return 1;
    /* every stride-th amax, plus every amax whose scale lands near 2^-126 or 2^-64 */
    return (ha % (uint32_t)stride) == 0 || ex < 12 || (ex >= 50 && ex <= 74);
}

static void *run(void *p) {
    Job *j = (Job *)p;
    for (uint32_t ha = 1 + (uint32_t)j->t; ha < 0x7F80; ha += (uint32_t)j->nt) {
        if (!selected(ha, j->stride)) continue;
        const float amax = bf(ha);
        float s = amax / j->fmax;
        if (s < 0x1p-126f) s = 0x1p-126f;
        const float pre = (s < 0x1p-64f) ? 0x1p64f : 1.0f;
        const float ss = s * pre, r = 1.0f / ss;
        for (uint32_t hx = 0; hx < 0x7F80; ++hx) {
            const float x = bf(hx);
            if (x > amax) break;
            for (int sg = 0; sg < 2; ++sg) {
                const float xv = sg ? -x : x;
                const float xs = xv * pre;
                const float q0 = xs * r;
                const float e = fmaf(-q0, ss, xs);
                const float q = copysignf(fmaf(e, r, q0), xv);
                j->pairs++;
                if (orc_encode(q, j->fmt) != orc_encode(xv / s, j->fmt)) {
                    if (j->bad < 3) fprintf(stderr, "mismatch fmt=%d amax=%a x=%a\n", j->fmt, amax, xv);
                    j->bad++;
                }
            }
        }
    }
    return NULL;
}

int main(int argc, char **argv) {
    int stride = argc > 1 ? atoi(argv[1]) : 1;
    const float fmaxes[2] = {448.0f, 57344.0f};
    long long total_bad = 0;
    for (int f = 0; f < 2; ++f) {
        pthread_t th[8];
        Job jobs[8];
        for (int t = 0; t < 8; ++t) {
            jobs[t] = (Job){t, 8, f, stride, fmaxes[f], 0, 0};
            pthread_create(&th[t], NULL, run, &jobs[t]);
        }
        long long pairs = 0, bad = 0;
        for (int t = 0; t < 8; ++t) { pthread_join(th[t], NULL); pairs += jobs[t].pairs; bad += jobs[t].bad; }
        printf("fmt=%d pairs=%lld code_mismatches=%lld\n", f, pairs, bad);
        total_bad += bad;
    }
    return total_bad != 0;
}
