/*
 * synth.c - seeded, counter-based input generator (host side).
 *
 * This module builds WORKLOADS, not results: it holds none of the arithmetic of
 * Memory Sparse Attention. Both the CPU oracle (oracle/) and the CUDA library
 * (long_context_doc_b200/) receive their inputs from here, so that the two sides
 * see bit-identical tensors.
 *
 * Generator (stated so that any side can re-implement it from its definition):
 *   mix64(z)        : the SplitMix64 output function (Steele, Lea & Flood,
 *                     "Fast splittable pseudorandom number generators", OOPSLA 2014;
 *                     finaliser constants of Stafford's variant 13):
 *                       z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *                       z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *                       return z ^ (z >> 31)
 *   key(seed, tag)  : mix64(seed * G ^ mix64(tag)),  G = 0x9E3779B97F4A7C15
 *   word(key, i)    : mix64(key + (i + 1) * G)       (the i-th SplitMix64 output)
 *   normal(key, e)  : the classic "sum of twelve uniforms minus six" approximation
 *                     of N(0,1): the three words 3e, 3e+1, 3e+2 give twelve 16-bit
 *                     integers u_j; S = sum u_j; x = (2 S - 12 * 65535) / 131072.
 *                     x has at most 21 significant bits, so it is EXACT in fp32 and
 *                     the same on every machine. Mean 0, variance 1 - 2^-32,
 *                     support [-6, 6].
 *   bf16(x)         : round-to-nearest-even of the fp32 bits to the upper 16 bits.
 *   uniform(key,i,n): floor(word(key, i) * n / 2^64)   (multiply-shift, exact).
 *
 * The device twin (synth_dev.cu) implements the same definitions with the same
 * integer operations; tests compare the two bit for bit.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#define SYN_G 0x9E3779B97F4A7C15ULL

static inline uint64_t syn_mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t syn_key(uint64_t seed, uint64_t tag) {
    return syn_mix64((seed * SYN_G) ^ syn_mix64(tag));
}

uint64_t syn_word(uint64_t key, uint64_t i) {
    return syn_mix64(key + (i + 1ULL) * SYN_G);
}

static inline float syn_normal_at(uint64_t key, uint64_t e) {
    int64_t s = 0;
    for (int w = 0; w < 3; ++w) {
        uint64_t r = syn_word(key, 3ULL * e + (uint64_t)w);
        s += (int64_t)(r & 0xFFFF) + (int64_t)((r >> 16) & 0xFFFF)
           + (int64_t)((r >> 32) & 0xFFFF) + (int64_t)(r >> 48);
    }
    /* 2S - 12*65535 is an integer of magnitude <= 786420; dividing by 2^17 is exact. */
    return (float)(2 * s - 12 * 65535) / 131072.0f;
}

static inline uint16_t syn_bf16_rne(float x) {
    uint32_t b;
    memcpy(&b, &x, 4);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

/* Fill out[0..n) with normal(key, first + i); dtype 0 = fp32, 1 = bf16 (uint16 bits).
 * `scale` multiplies the exact normal in fp32 before storage (1.0 leaves it exact). */
void syn_fill_normal(void* out, int64_t n, int dtype, uint64_t seed, uint64_t tag,
                     uint64_t first, float scale) {
    uint64_t key = syn_key(seed, tag);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float x = syn_normal_at(key, first + (uint64_t)i) * scale;
        if (dtype == 0) ((float*)out)[i] = x;
        else ((uint16_t*)out)[i] = syn_bf16_rne(x);
    }
}

/* Exact fp32 normals (for host-side workload construction in double). */
void syn_fill_normal_f64(double* out, int64_t n, uint64_t seed, uint64_t tag, uint64_t first) {
    uint64_t key = syn_key(seed, tag);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (double)syn_normal_at(key, first + (uint64_t)i);
}

/* Uniform integers in [0, hi). */
void syn_fill_uniform(int64_t* out, int64_t n, uint64_t seed, uint64_t tag, uint64_t hi) {
    uint64_t key = syn_key(seed, tag);
    for (int64_t i = 0; i < n; ++i) {
        uint64_t w = syn_word(key, (uint64_t)i);
        out[i] = (int64_t)(((unsigned __int128)w * hi) >> 64);
    }
}

/* k distinct integers in [0, hi), in draw order (rejection of repeats). */
int syn_distinct(int64_t* out, int64_t k, uint64_t seed, uint64_t tag, uint64_t hi) {
    if ((uint64_t)k > hi) return -1;
    uint64_t key = syn_key(seed, tag);
    uint64_t i = 0;
    for (int64_t got = 0; got < k; ) {
        uint64_t w = syn_word(key, i++);
        int64_t v = (int64_t)(((unsigned __int128)w * hi) >> 64);
        int dup = 0;
        for (int64_t j = 0; j < got; ++j) if (out[j] == v) { dup = 1; break; }
        if (!dup) out[got++] = v;
    }
    return 0;
}

/* fp32 -> bf16 RNE over an array (workload construction of planted rows). */
void syn_to_bf16(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = syn_bf16_rne(in[i]);
}
