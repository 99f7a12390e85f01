/*
 * Seeded synthetic inputs for the routed FP4 mixture-of-experts layer.
 *
 * This file holds random-number generation and input preparation only; it
 * contains none of the layer's arithmetic (no routing, sorting, quantisation,
 * FP4 decoding, GEMM or combine).  Both the CUDA path and the CPU oracle are
 * fed from here, and nothing here depends on either of them.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014; constants as in Vigna's public-domain
 * reference).  Output number i of a generator started in state s is
 * mix(s + (i+1)*GAMMA), so every element is computed from its own index and
 * generation parallelises without changing any value.
 *
 * The stream of tensor `tid` for a config seed is the generator whose start
 * state is output number `tid` of the generator started in state `seed`.
 * Tensor ids: 0 x, 1 router weight, 2 W1 codes, 3 W1 scales, 4 W2 codes,
 * 5 W2 scales.
 *
 * Normals use the Box-Muller transform: pair j takes outputs 2j and 2j+1,
 * u1 = (o>>11 + 1) * 2^-53 in (0,1], u2 = (o>>11) * 2^-53 in [0,1),
 * z0 = sqrt(-2 ln u1) cos(2 pi u2), z1 = sqrt(-2 ln u1) sin(2 pi u2).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* output i (0-based) of the SplitMix64 generator started in state s */
static inline uint64_t sm_at(uint64_t s, uint64_t i) { return mix64(s + (i + 1) * GAMMA); }

uint64_t synth_stream_key(uint64_t seed, uint32_t tid) { return sm_at(seed, tid); }

uint64_t synth_u64(uint64_t seed, uint32_t tid, uint64_t i) {
    return sm_at(synth_stream_key(seed, tid), i);
}

static inline double normal_at(uint64_t key, uint64_t i) {
    uint64_t j = i >> 1;
    uint64_t a = sm_at(key, 2 * j), b = sm_at(key, 2 * j + 1);
    double u1 = (double)((a >> 11) + 1) * 0x1.0p-53;
    double u2 = (double)(b >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double th = 2.0 * M_PI * u2;
    return (i & 1) ? r * sin(th) : r * cos(th);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ---- threaded driver over an index range ---- */
typedef struct {
    int kind;
    uint64_t key;
    void *out;
    int64_t lo, hi;
    float scale;
    uint32_t base, span;
} job_t;

static void *run_job(void *p) {
    job_t *j = (job_t *)p;
    for (int64_t i = j->lo; i < j->hi; ++i) {
        switch (j->kind) {
        case 0: /* normals * scale -> f32 */
            ((float *)j->out)[i] = (float)(j->scale * normal_at(j->key, (uint64_t)i));
            break;
        case 1: /* normals -> f32 -> bf16 RNE */
            ((uint16_t *)j->out)[i] = f32_to_bf16_rne((float)normal_at(j->key, (uint64_t)i));
            break;
        case 2: { /* raw bytes: output i gives bytes [8i, 8i+8), little endian */
            uint64_t o = sm_at(j->key, (uint64_t)i);
            uint8_t *dst = (uint8_t *)j->out + 8 * i;
            for (int b = 0; b < 8; ++b) dst[b] = (uint8_t)(o >> (8 * b));
            break;
        }
        case 3: { /* base + uniform{0..span-1} (Lemire multiply-shift on the top 32 bits) */
            uint64_t o = sm_at(j->key, (uint64_t)i) >> 32;
            ((uint8_t *)j->out)[i] = (uint8_t)(j->base + ((o * j->span) >> 32));
            break;
        }
        }
    }
    return NULL;
}

static void run_threaded(job_t proto, int64_t n, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 64) nthreads = 64;
    if (n < 65536) nthreads = 1;
    pthread_t th[64];
    job_t jobs[64];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = proto;
        jobs[t].lo = n * t / nthreads;
        jobs[t].hi = n * (t + 1) / nthreads;
        if (nthreads == 1) { run_job(&jobs[t]); return; }
        pthread_create(&th[t], NULL, run_job, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}

void synth_normals_f32(uint64_t seed, uint32_t tid, float scale, float *out, int64_t n, int nthreads) {
    job_t j = {0, synth_stream_key(seed, tid), out, 0, 0, scale, 0, 0};
    run_threaded(j, n, nthreads);
}

void synth_normals_bf16(uint64_t seed, uint32_t tid, uint16_t *out, int64_t n, int nthreads) {
    job_t j = {1, synth_stream_key(seed, tid), out, 0, 0, 1.0f, 0, 0};
    run_threaded(j, n, nthreads);
}

void synth_bytes(uint64_t seed, uint32_t tid, uint8_t *out, int64_t n, int nthreads) {
    uint64_t key = synth_stream_key(seed, tid);
    job_t j = {2, key, out, 0, 0, 1.0f, 0, 0};
    run_threaded(j, n / 8, nthreads); /* whole 8-byte words */
    if (n % 8) {                      /* tail word */
        uint64_t o = sm_at(key, (uint64_t)(n / 8));
        for (int64_t b = 0; b < n % 8; ++b) out[8 * (n / 8) + b] = (uint8_t)(o >> (8 * b));
    }
}

void synth_uniform_bytes(uint64_t seed, uint32_t tid, uint32_t base, uint32_t span, uint8_t *out,
                         int64_t n, int nthreads) {
    job_t j = {3, synth_stream_key(seed, tid), out, 0, 0, 1.0f, base, span};
    run_threaded(j, n, nthreads);
}

/* ---- router logits (the step before the layer): fp32(sum_h x*w_r + bias), fp64 sum ---- */
typedef struct {
    const uint16_t *x;
    const float *wr;
    const double *bias;
    int T, H, E;
    float *out;
    int t0, t1;
} lj_t;

static void *run_logits(void *p) {
    lj_t *j = (lj_t *)p;
    for (int t = j->t0; t < j->t1; ++t) {
        for (int e = 0; e < j->E; ++e) {
            const uint16_t *xr = j->x + (int64_t)t * j->H;
            const float *wr = j->wr + (int64_t)e * j->H;
            double acc = 0.0;
            for (int h = 0; h < j->H; ++h) {
                uint32_t u = (uint32_t)xr[h] << 16;
                float xf;
                memcpy(&xf, &u, 4);
                acc += (double)xf * (double)wr[h];
            }
            if (j->bias) acc += j->bias[e];
            j->out[(int64_t)t * j->E + e] = (float)acc;
        }
    }
    return NULL;
}

void synth_router_logits(const uint16_t *x_bf16, const float *wr, const double *bias, int T, int H,
                         int E, float *out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 64) nthreads = 64;
    if (nthreads > T) nthreads = T > 0 ? T : 1;
    pthread_t th[64];
    lj_t jobs[64];
    for (int i = 0; i < nthreads; ++i) {
        lj_t j = {x_bf16, wr, bias, T, H, E, out, (int)((int64_t)T * i / nthreads),
                  (int)((int64_t)T * (i + 1) / nthreads)};
        jobs[i] = j;
        if (nthreads == 1) { run_logits(&jobs[i]); return; }
        pthread_create(&th[i], NULL, run_logits, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
}

/* raw SplitMix64 output i of a generator started in state s (for known-answer tests) */
uint64_t synth_splitmix64_at(uint64_t s, uint64_t i) { return sm_at(s, i); }
