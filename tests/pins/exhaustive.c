/*
 * Exhaustive pins of the oracle's two rounding functions (test code).
 *
 * The reference answer is a brute-force nearest-value search over a value
 * table handed in by the test (E2M1: the list printed in "NVFP4: how NVIDIA
 * pre-trained a 12B model on 10T tokens", section "E2M1 format and two-level
 * scaling"; E4M3: the 127 non-negative finite values built by the test from
 * the format's definition).  Ties go to the code whose lowest bit is 0.
 *
 * A full brute force over all 2^31 non-negative binary32 patterns costs
 * 2^31 x |table| comparisons, so the sweep instead checks that the oracle is
 * monotone over every pattern in order and agrees with the brute force on
 * both sides of every step.  A monotone step function that matches a
 * monotone target at both ends of each of its steps matches it everywhere.
 * The E2M1 sweep also checks sign symmetry on every pattern.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

uint8_t nvo_e2m1_rne_satfinite(float y);
uint8_t nvo_e4m3_rne_satfinite(float v);

typedef struct {
    const double *vals;   /* non-negative finite values */
    const uint8_t *codes; /* their codes */
    int n;
} table_t;

static uint8_t brute(const table_t *t, double a)
{
    /* At or above the largest value every distance a - v is smallest for
     * the largest v; handled apart because for huge a the double
     * differences a - v all round to the same number. */
    int top = 0;
    for (int i = 1; i < t->n; ++i)
        if (t->vals[i] > t->vals[top])
            top = i;
    if (a >= t->vals[top])
        return t->codes[top];
    int best = 0;
    double bd = fabs(a - t->vals[0]);
    for (int i = 1; i < t->n; ++i) {
        double d = fabs(a - t->vals[i]);
        if (d < bd || (d == bd && (t->codes[i] & 1) == 0 && (t->codes[best] & 1) == 1)) {
            best = i;
            bd = d;
        }
    }
    return t->codes[best];
}

static float from_bits(uint32_t u)
{
    float f;
    memcpy(&f, &u, 4);
    return f;
}

typedef struct {
    const table_t *t;
    int which;      /* 0: e2m1, 1: e4m3 */
    uint32_t lo, hi; /* pattern range [lo, hi) */
    int64_t bad;
    int64_t steps;
} job_t;

static uint8_t eval(int which, float f)
{
    return which == 0 ? (uint8_t)(nvo_e2m1_rne_satfinite(f) & 7) : nvo_e4m3_rne_satfinite(f);
}

static void *run(void *p)
{
    job_t *j = (job_t *)p;
    uint32_t u = j->lo;
    uint8_t prev = eval(j->which, from_bits(u));
    if (prev != brute(j->t, (double)from_bits(u)))
        j->bad++;
    if (u > 0) { /* step across the range boundary */
        uint8_t before = eval(j->which, from_bits(u - 1));
        if (before != prev) {
            j->steps++;
            if (before > prev)
                j->bad++;
        }
    }
    for (u = j->lo + 1; u < j->hi; ++u) {
        float f = from_bits(u);
        uint8_t c = eval(j->which, f);
        if (j->which == 0) {
            uint8_t neg = nvo_e2m1_rne_satfinite(-f);
            if (neg != (uint8_t)(c | 8))
                j->bad++;
        }
        if (c != prev) {
            j->steps++;
            if (c < prev)
                j->bad++;
            if (prev != brute(j->t, (double)from_bits(u - 1)))
                j->bad++;
            if (c != brute(j->t, (double)f))
                j->bad++;
        }
        prev = c;
    }
    if (prev != brute(j->t, (double)from_bits(j->hi - 1)))
        j->bad++;
    return NULL;
}

/* Returns the number of violations; *steps receives the number of steps. */
int64_t pins_sweep(int which, const double *vals, const uint8_t *codes, int n, int threads,
                   int64_t *steps)
{
    table_t t = {vals, codes, n};
    const uint32_t end = 0x7F800000u; /* all non-negative finite patterns */
    pthread_t th[64];
    job_t jobs[64];
    if (threads > 64)
        threads = 64;
    if (threads < 1)
        threads = 1;
    uint32_t chunk = end / (uint32_t)threads + 1;
    for (int i = 0; i < threads; ++i) {
        uint32_t lo = (uint32_t)i * chunk, hi = lo + chunk;
        if (hi > end)
            hi = end;
        jobs[i] = (job_t){&t, which, lo, hi, 0, 0};
        pthread_create(&th[i], NULL, run, &jobs[i]);
    }
    int64_t bad = 0, st = 0;
    for (int i = 0; i < threads; ++i) {
        pthread_join(th[i], NULL);
        bad += jobs[i].bad;
        st += jobs[i].steps;
    }
    *steps = st;
    return bad;
}
