/*
 * Seeded synthetic inputs for causal grouped-query softmax attention.
 *
 * This file holds no attention arithmetic. It produces the bf16 bit patterns
 * of iid N(0,1) tensors, index-addressable, so that the fp64 oracle and the
 * GPU harness can both consume the same bytes (and the oracle can regenerate
 * any single row without generating the whole tensor).
 *
 * Definition (fixed, part of the input recipe):
 *   GOLDEN = 0x9E3779B97F4A7C15 (2^64 / golden ratio, splitmix64 increment)
 *   mix(z): splitmix64 finaliser (Steele, Lea & Flood, "Fast splittable
 *           pseudorandom number generators", OOPSLA 2014):
 *           z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *           z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31.
 *   key(seed, tensor_id) = mix(seed * GOLDEN + tensor_id)           (mod 2^64)
 *   word(n)              = mix(key + (n + 1) * GOLDEN)              (mod 2^64)
 *   Elements 2p and 2p+1 form one Box-Muller pair (Box & Muller, 1958):
 *     u1 = (word(2p)   >> 11) * 2^-53,  u2 = (word(2p+1) >> 11) * 2^-53
 *     r  = sqrt(-2 ln(1 - u1)),  theta = 2 pi u2     (in double)
 *     element 2p = r cos(theta),  element 2p+1 = r sin(theta)
 *   Each double is rounded to float (round-to-nearest-even), then the float
 *   to bf16 (round-to-nearest-even on the upper 16 bits).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GQA_GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    /* inputs are finite; round half to even on bit 16 */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static inline void pair_normals(uint64_t key, uint64_t p, double* z0, double* z1) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t w0 = mix64(key + (2 * p + 1) * GQA_GOLDEN);
    uint64_t w1 = mix64(key + (2 * p + 2) * GQA_GOLDEN);
    double u1 = (double)(w0 >> 11) * (1.0 / 9007199254740992.0);
    double u2 = (double)(w1 >> 11) * (1.0 / 9007199254740992.0);
    double r = sqrt(-2.0 * log(1.0 - u1));
    double th = two_pi * u2;
    *z0 = r * cos(th);
    *z1 = r * sin(th);
}

uint64_t gqa_gen_key(uint64_t seed, uint32_t tensor_id) {
    return mix64(seed * GQA_GOLDEN + (uint64_t)tensor_id);
}

/* Fill out[i] = element (start + i) of the stream, i in [0, count). */
static void fill_range(uint64_t key, uint64_t start, uint64_t count, uint16_t* out) {
    uint64_t i = 0;
    double z0, z1;
    if (count == 0) return;
    if (start & 1u) {
        pair_normals(key, start >> 1, &z0, &z1);
        out[0] = f32_to_bf16_rne((float)z1);
        i = 1;
    }
    for (; i + 1 < count; i += 2) {
        pair_normals(key, (start + i) >> 1, &z0, &z1);
        out[i] = f32_to_bf16_rne((float)z0);
        out[i + 1] = f32_to_bf16_rne((float)z1);
    }
    if (i < count) {
        pair_normals(key, (start + i) >> 1, &z0, &z1);
        out[i] = f32_to_bf16_rne((float)z0);
    }
}

typedef struct {
    uint64_t key, start, count;
    uint16_t* out;
} fill_job;

static void* fill_worker(void* arg) {
    fill_job* j = (fill_job*)arg;
    fill_range(j->key, j->start, j->count, j->out);
    return NULL;
}

/* Elements [start, start+count) of stream (seed, tensor_id) as bf16 bits.
 * n_threads <= 0 selects one thread. Returns 0 on success. */
int gqa_gen_normal_bf16(uint64_t seed, uint32_t tensor_id, uint64_t start, uint64_t count,
                        uint16_t* out, int n_threads) {
    uint64_t key = gqa_gen_key(seed, tensor_id);
    if (n_threads <= 1 || count < (1u << 16)) {
        fill_range(key, start, count, out);
        return 0;
    }
    if (n_threads > 256) n_threads = 256;
    pthread_t th[256];
    int joined[256];
    fill_job jobs[256];
    uint64_t per = (count + (uint64_t)n_threads - 1) / (uint64_t)n_threads;
    per = (per + 1) & ~(uint64_t)1; /* keep pairs inside one job */
    int launched = 0;
    for (int t = 0; t < n_threads; ++t) {
        uint64_t s = (uint64_t)t * per;
        if (s >= count) break;
        uint64_t c = count - s < per ? count - s : per;
        jobs[t].key = key;
        jobs[t].start = start + s;
        jobs[t].count = c;
        jobs[t].out = out + s;
        joined[t] = pthread_create(&th[t], NULL, fill_worker, &jobs[t]) == 0;
        if (!joined[t]) fill_worker(&jobs[t]);
        launched = t + 1;
    }
    for (int t = 0; t < launched; ++t)
        if (joined[t]) pthread_join(th[t], NULL);
    return 0;
}

/* Raw words word(start) .. word(start+count-1) of stream (seed, tensor_id): the
 * integer draws of the recipe (sequence lengths, page assignments) use these. */
void gqa_gen_words(uint64_t seed, uint32_t tensor_id, uint64_t start, uint64_t count, uint64_t* out) {
    uint64_t key = gqa_gen_key(seed, tensor_id);
    for (uint64_t i = 0; i < count; ++i) out[i] = mix64(key + (start + i + 1) * GQA_GOLDEN);
}
