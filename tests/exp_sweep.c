/*
 * exp_sweep.c -- pins the oracle's exp and sigmoid against float64 libm on
 * EVERY fp32 input of their working domain (test infrastructure: built and
 * run by tests/test_oracle_exhaustive.py, linked against oracle/liboracle.so).
 *
 *   oracle_dexp(y),    y in [-87, 88]  vs  exp((double)y)
 *   oracle_sigmoid(x), x in [-88, 87]  vs  1 / (1 + exp(-(double)x))
 *
 * For each it prints the largest error in units in the last place of the
 * fp32 result (ulp = spacing of the fp32 nearest the exact value, as
 * numpy.spacing), the mean error, the number of inputs and the number of
 * neighbouring input pairs where the routine is not monotone (where it
 * decreases as its input grows) with the largest such step in ulps.  One
 * line per routine:
 *   <name> n=<count> max_ulp=<x> mean_ulp=<x> argmax=<bits> nonmonotone=<count>
 *   max_drop_ulp=<x>
 *
 * The domain is walked by bit pattern: +0 .. hi for the non-negative half,
 * -0 .. lo for the negative half, split over threads (argv[1], default 8).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

float oracle_dexp(float y);
float oracle_sigmoid(float x);

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static double ulp_of(double exact)
{
    float a = (float)fabs(exact);
    return (double)nextafterf(a, INFINITY) - (double)a;
}

typedef struct {
    int which;             /* 0 = exp, 1 = sigmoid */
    uint32_t first, last;  /* bit patterns, inclusive, one sign */
    int negative;          /* patterns walk away from zero on the negative side */
    double max_ulp, sum_ulp;
    uint32_t argmax;
    uint64_t n, nonmono;
    double max_drop;       /* largest non-monotone step, in ulps of the larger value */
} job_t;

static void* run(void* p)
{
    job_t* j = (job_t*)p;
    float prev = 0.0f;
    int have_prev = 0;
    /* one pattern before the range, so monotonicity is checked across the
     * boundary with the previous thread's range as well */
    uint32_t start = j->first > (j->negative ? 0x80000000u : 0u) ? j->first - 1 : j->first;
    for (uint64_t b = start; b <= j->last; ++b) {
        const float x = from_bits((uint32_t)b);
        double exact;
        float got;
        if (j->which == 0) {
            got = oracle_dexp(x);
            exact = exp((double)x);
        } else {
            got = oracle_sigmoid(x);
            exact = 1.0 / (1.0 + exp(-(double)x));
        }
        /* positive side: x grows with the pattern; negative side: x shrinks */
        if (have_prev && (j->negative ? got > prev : got < prev)) {
            const float hi = got > prev ? got : prev, lo = got > prev ? prev : got;
            const double drop = ((double)hi - (double)lo) / ((double)nextafterf(lo, INFINITY) - (double)lo);
            j->nonmono++;
            if (drop > j->max_drop) j->max_drop = drop;
        }
        prev = got;
        have_prev = 1;
        if (b < j->first) continue;
        const double e = fabs((double)got - exact) / ulp_of(exact);
        j->n++;
        j->sum_ulp += e;
        if (e > j->max_ulp) {
            j->max_ulp = e;
            j->argmax = (uint32_t)b;
        }
    }
    return NULL;
}

static void sweep(const char* name, int which, float lo, float hi, int threads)
{
    /* two halves: [+0, hi] and [-0, lo] by pattern */
    const uint32_t ranges[2][2] = {{0x00000000u, to_bits(hi)}, {0x80000000u, to_bits(lo)}};
    job_t* jobs = (job_t*)calloc((size_t)threads * 2, sizeof(job_t));
    pthread_t* tid = (pthread_t*)calloc((size_t)threads * 2, sizeof(pthread_t));
    int nj = 0;
    for (int h = 0; h < 2; ++h) {
        const uint64_t a = ranges[h][0], z = ranges[h][1];
        const uint64_t span = z - a + 1;
        for (int t = 0; t < threads; ++t) {
            job_t* j = &jobs[nj];
            j->which = which;
            j->negative = h;
            j->first = (uint32_t)(a + span * (uint64_t)t / (uint64_t)threads);
            j->last = (uint32_t)(a + span * (uint64_t)(t + 1) / (uint64_t)threads - 1);
            pthread_create(&tid[nj], NULL, run, j);
            ++nj;
        }
    }
    double mx = 0.0, sum = 0.0;
    uint64_t n = 0, nonmono = 0;
    uint32_t arg = 0;
    double drop = 0.0;
    for (int i = 0; i < nj; ++i) {
        pthread_join(tid[i], NULL);
        if (jobs[i].max_ulp > mx) {
            mx = jobs[i].max_ulp;
            arg = jobs[i].argmax;
        }
        sum += jobs[i].sum_ulp;
        n += jobs[i].n;
        nonmono += jobs[i].nonmono;
        if (jobs[i].max_drop > drop) drop = jobs[i].max_drop;
    }
    printf("%s n=%llu max_ulp=%.6f mean_ulp=%.6f argmax=0x%08x nonmonotone=%llu max_drop_ulp=%.3f\n",
           name, (unsigned long long)n, mx, sum / (double)n, arg, (unsigned long long)nonmono, drop);
    free(jobs);
    free(tid);
}

int main(int argc, char** argv)
{
    const int threads = argc > 1 ? atoi(argv[1]) : 8;
    const int which = argc > 2 ? atoi(argv[2]) : -1;   /* -1: both */
    if (which != 1) sweep("exp", 0, -87.0f, 88.0f, threads < 1 ? 1 : threads);
    if (which != 0) sweep("sigmoid", 1, -88.0f, 87.0f, threads < 1 ? 1 : threads);
    return 0;
}
