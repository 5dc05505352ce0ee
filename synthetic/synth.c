/*
 * synth.c -- seeded synthetic inputs (bf16 tensors) for tests and benchmarks.
 *
 * This module holds no arithmetic of the FP8 method. It draws the input
 * tensors that both the CPU oracle and the CUDA library consume.
 *
 * Generator (counter based, so any element can be drawn independently):
 *   mix64(z)      : the SplitMix64 output function (Steele, Lea, Flood,
 *                   "Fast splittable pseudorandom number generators", 2014):
 *                   z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
 *                   z *= 0x94D049BB133111EB; z ^= z>>31.
 *   stream key    : key = mix64(mix64(mix64(seed + G) ^ (tensor_id*G + 1))
 *                           ^ (stream*G + 2)),  G = 0x9E3779B97F4A7C15.
 *   i-th word     : w(key, i) = mix64(key + (i + 1) * G)   (SplitMix64 state
 *                   sequence started at key).
 *   uniform       : u = (w >> 11) * 2^-53 in [0, 1).
 *   normal        : element i uses u1 = u(2i), u2 = u(2i+1) of stream 0:
 *                   z = sqrt(-2 ln(1 - u1)) * cos(2 pi u2)   (Box-Muller).
 *   outlier       : element i is an outlier iff w(key of stream 1, i) <
 *                   p * 2^64; its value is multiplied by `factor`.
 *   value         : std * z (* factor) in fp64, rounded to fp32 (RNE), then
 *                   to bf16 (RNE).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define G64 0x9E3779B97F4A7C15ULL

uint64_t synth_mix64(uint64_t z)
{
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

uint64_t synth_key(uint64_t seed, uint64_t tensor_id, uint64_t stream)
{
    uint64_t k = synth_mix64(seed + G64);
    k = synth_mix64(k ^ (tensor_id * G64 + 1ULL));
    return synth_mix64(k ^ (stream * G64 + 2ULL));
}

static uint64_t word(uint64_t key, uint64_t i)
{
    return synth_mix64(key + (i + 1ULL) * G64);
}

static double uni(uint64_t w) { return (double)(w >> 11) * 0x1.0p-53; }

static uint16_t f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u)      /* inf / nan: truncate */
        return (uint16_t)(u >> 16);
    u += 0x7FFFu + ((u >> 16) & 1u);           /* round to nearest even */
    return (uint16_t)(u >> 16);
}

double synth_normal_at(uint64_t key, uint64_t i)
{
    double u1 = uni(word(key, 2 * i));
    double u2 = uni(word(key, 2 * i + 1));
    return sqrt(-2.0 * log(1.0 - u1)) * cos(6.283185307179586 * u2);
}

typedef struct {
    uint64_t kn, ko, thresh;
    double std, factor;
    int use_outliers;
    uint16_t* out;
    int64_t begin, end;
} job;

static void* run(void* arg)
{
    job* j = (job*)arg;
    int64_t i;
    for (i = j->begin; i < j->end; ++i) {
        double v = j->std * synth_normal_at(j->kn, (uint64_t)i);
        if (j->use_outliers && word(j->ko, (uint64_t)i) < j->thresh)
            v *= j->factor;
        j->out[i] = f32_to_bf16((float)v);
    }
    return NULL;
}

int synth_bf16_normal(uint64_t seed, uint64_t tensor_id, double std,
                      double outlier_p, double outlier_factor, uint16_t* out,
                      int64_t count, int nthreads)
{
    job jobs[64];
    pthread_t tids[64];
    int started[64];
    int t;
    if (!out || count < 0)
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 64)
        nthreads = 64;
    for (t = 0; t < nthreads; ++t) {
        jobs[t].kn = synth_key(seed, tensor_id, 0);
        jobs[t].ko = synth_key(seed, tensor_id, 1);
        jobs[t].use_outliers = outlier_p > 0.0;
        jobs[t].thresh = outlier_p >= 1.0 ? UINT64_MAX
                         : (uint64_t)ldexp(outlier_p, 64);
        jobs[t].std = std;
        jobs[t].factor = outlier_factor;
        jobs[t].out = out;
        jobs[t].begin = count * t / nthreads;
        jobs[t].end = count * (t + 1) / nthreads;
    }
    for (t = 1; t < nthreads; ++t)
        started[t] = pthread_create(&tids[t], NULL, run, &jobs[t]) == 0;
    run(&jobs[0]);
    for (t = 1; t < nthreads; ++t) {
        if (started[t])
            pthread_join(tids[t], NULL);
        else
            run(&jobs[t]);
    }
    return 0;
}
