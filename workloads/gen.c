/*
 * Seeded synthetic input streams shared by the CUDA path's tests/bench and the
 * CPU oracle.  This file holds random-number generation only: no attention,
 * paging or cache arithmetic lives here.
 *
 * Stream definition (counter based, so any element can be produced
 * independently and in parallel):
 *   word(seed, i)  = splitmix64 finaliser applied to seed + (i + 1) * 0x9E3779B97F4A7C15
 *   uniform(seed, i) = (word(seed, i) >> 11) * 2^-53                     in [0, 1)
 *   normal pair j  = Box-Muller on u0 = uniform(seed, 2j), u1 = uniform(seed, 2j + 1):
 *                    r = sqrt(-2 ln(1 - u0)), n_{2j} = r cos(2 pi u1), n_{2j+1} = r sin(2 pi u1)
 *   bf16 element i = round-to-nearest-even of (float) n_i to the upper 16 bits.
 *
 * splitmix64 is Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators" (OOPSLA 2014); Box-Muller is the 1958 polar-free transform.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static inline uint64_t gen_word(uint64_t seed, uint64_t i) {
    uint64_t z = seed + (i + 1u) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline double gen_unit(uint64_t seed, uint64_t i) {
    return (double)(gen_word(seed, i) >> 11) * 0x1.0p-53;
}

static inline double gen_normal_at(uint64_t seed, uint64_t i) {
    const uint64_t pair = i >> 1;
    const double u0 = gen_unit(seed, 2 * pair);
    const double u1 = gen_unit(seed, 2 * pair + 1);
    const double r = sqrt(-2.0 * log(1.0 - u0));
    const double theta = 6.283185307179586476925286766559 * u1;
    return (i & 1) ? r * sin(theta) : r * cos(theta);
}

static inline uint16_t gen_f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u) {          /* inf / nan: truncate, keep nan quiet */
        return (uint16_t)((u >> 16) | ((u & 0x007FFFFFu) ? 0x0040u : 0u));
    }
    const uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* n raw 64-bit words, elements [offset, offset + n) of stream `seed`. */
void gen_words(uint64_t seed, uint64_t offset, int64_t n, uint64_t* out) {
#pragma omp parallel for schedule(static) if (n > (1 << 16))
    for (int64_t i = 0; i < n; ++i) out[i] = gen_word(seed, offset + (uint64_t)i);
}

/* n uniforms in [0, 1). */
void gen_uniform_f64(uint64_t seed, uint64_t offset, int64_t n, double* out) {
#pragma omp parallel for schedule(static) if (n > (1 << 16))
    for (int64_t i = 0; i < n; ++i) out[i] = gen_unit(seed, offset + (uint64_t)i);
}

/* n standard normals (fp64). offset must be even so pairs stay aligned. */
void gen_normal_f64(uint64_t seed, uint64_t offset, int64_t n, double* out) {
#pragma omp parallel for schedule(static) if (n > (1 << 16))
    for (int64_t i = 0; i < n; ++i) out[i] = gen_normal_at(seed, offset + (uint64_t)i);
}

/* n standard normals rounded (RNE) to bf16 bit patterns. */
void gen_normal_bf16(uint64_t seed, uint64_t offset, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static) if (n > (1 << 16))
    for (int64_t i = 0; i < n; ++i) {
        out[i] = gen_f32_to_bf16_rne((float)gen_normal_at(seed, offset + (uint64_t)i));
    }
}

int gen_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
