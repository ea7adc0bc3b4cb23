/*
 * mokgen.c -- seeded synthetic-input generator shared by the tests, the
 * benchmark and the smoke check.
 *
 * This file holds no arithmetic of the MoE layer.  It only turns
 * (seed, stream, element index) into a value drawn from a caller-supplied
 * 65536-entry table, so that a table of inverse-normal-CDF quantiles yields
 * Gaussian data at bf16 / fp32 resolution.
 *
 * Counter-based generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Element i of a stream reads
 * 16 bits of mix(key + floor(i / 4)); because the value depends only on
 * (seed, stream, i), any slice can be generated independently and in
 * parallel, and the result does not depend on the thread count.
 */
#include <stdint.h>
#include <stddef.h>

#define MOKGEN_GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t mokgen_mix(uint64_t z) {
    z += MOKGEN_GOLDEN;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t mokgen_key(uint64_t seed, uint64_t stream) {
    return mokgen_mix(mokgen_mix(seed) ^ (stream * MOKGEN_GOLDEN));
}

/* Element index -> 16-bit table index for the stream `key`. */
static inline uint32_t mokgen_idx16(uint64_t key, uint64_t i) {
    uint64_t r = mokgen_mix(key + (i >> 2) * MOKGEN_GOLDEN);
    return (uint32_t)((r >> (16u * (unsigned)(i & 3u))) & 0xFFFFu);
}

/* out[j] = tab[idx16(key, first + j)], j in [0, n). 16-bit payload (bf16). */
void mokgen_fill_u16(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                     const uint16_t* tab, uint16_t* out) {
    const uint64_t key = mokgen_key(seed, stream);
    const int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nn; ++j) out[j] = tab[mokgen_idx16(key, first + (uint64_t)j)];
}

/* Same stream definition with a 32-bit payload (fp32 tables). */
void mokgen_fill_u32(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                     const uint32_t* tab, uint32_t* out) {
    const uint64_t key = mokgen_key(seed, stream);
    const int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nn; ++j) out[j] = tab[mokgen_idx16(key, first + (uint64_t)j)];
}

/* Raw 16-bit draws (used for small integer-valued logits in tie tests). */
void mokgen_fill_idx16(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n, uint16_t* out) {
    const uint64_t key = mokgen_key(seed, stream);
    const int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nn; ++j) out[j] = (uint16_t)mokgen_idx16(key, first + (uint64_t)j);
}
