/* Exhaustive check of the oracle's fp32 sigmoid against the fp64 definition
 * 1 / (1 + exp(-l)), over every fp32 l in [lo, hi], on n_threads threads.
 * Reports the largest error in fp32 ulps of the exact value and the number
 * of places where the sequence decreases (it must be monotone). */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

float orc_sigmoid(float l);

typedef struct { int64_t i0, i1; int64_t neg_count; uint32_t neg_top; double max_ulp; float worst; int64_t nonmono; } job;

/* value of the i-th fp32 in increasing order over the swept range:
 * i < neg_count: negatives from neg_top (most negative) towards -0. */
static float nth(int64_t i, int64_t neg_count, uint32_t neg_top)
{
    uint32_t u = i < neg_count ? (uint32_t)(neg_top - (uint32_t)i) : (uint32_t)(i - neg_count);
    float f; memcpy(&f, &u, 4); return f;
}

static void* run(void* p)
{
    job* j = (job*)p;
    double mx = 0.0; float worst = 0.0f; int64_t nm = 0;
    float prev = j->i0 > 0 ? orc_sigmoid(nth(j->i0 - 1, j->neg_count, j->neg_top)) : -1.0f;
    for (int64_t i = j->i0; i < j->i1; ++i) {
        float l = nth(i, j->neg_count, j->neg_top);
        float s = orc_sigmoid(l);
        double ref = 1.0 / (1.0 + exp(-(double)l));
        int e; frexp(ref, &e);
        int q = e - 1 - 23; if (q < -149) q = -149;
        double err = fabs((double)s - ref) / ldexp(1.0, q);
        if (err > mx) { mx = err; worst = l; }
        if (s < prev) nm++;
        prev = s;
    }
    j->max_ulp = mx; j->worst = worst; j->nonmono = nm;
    return NULL;
}

/* returns max ulp; *worst = argument where it occurs; *nonmono = decreases */
double sigmoid_sweep(float lo, float hi, int n_threads, float* worst, int64_t* nonmono)
{
    uint32_t blo, bhi; memcpy(&blo, &lo, 4); memcpy(&bhi, &hi, 4);
    /* lo < 0 <= hi assumed */
    int64_t neg_count = (int64_t)(blo - 0x80000000u) + 1;   /* lo .. -0 */
    int64_t total = neg_count + (int64_t)bhi + 1;            /* +0 .. hi */
    pthread_t th[256]; job jb[256];
    if (n_threads > 256) n_threads = 256;
    for (int t = 0; t < n_threads; ++t) {
        jb[t].i0 = total * t / n_threads; jb[t].i1 = total * (t + 1) / n_threads;
        jb[t].neg_count = neg_count; jb[t].neg_top = blo;
        pthread_create(&th[t], NULL, run, &jb[t]);
    }
    double mx = 0.0; int64_t nm = 0; *worst = 0.0f;
    for (int t = 0; t < n_threads; ++t) {
        pthread_join(th[t], NULL);
        if (jb[t].max_ulp > mx) { mx = jb[t].max_ulp; *worst = jb[t].worst; }
        nm += jb[t].nonmono;
    }
    *nonmono = nm;
    return mx;
}
