/*
 * Seeded synthetic input generator (test and benchmark infrastructure).
 *
 * This file holds no part of the attention method: it only turns
 * (seed, tensor id, element index) into a normally distributed number and
 * stores it in the requested storage format.  Both the CUDA path and the
 * CPU oracle consume the bytes it writes, so the two sides always see
 * identical inputs.
 *
 * Generator (counter based, so any slice of any tensor can be produced
 * independently and in parallel):
 *   stream  = mix64(seed * GOLDEN + tensor_id + 1)
 *   h1, h2  = outputs 2i+1 and 2i+2 of a SplitMix64 sequence whose state
 *             starts at `stream` (output n = mix64(stream + n * GOLDEN))
 *   u1      = ((h1 >> 11) + 1) * 2^-53        in (0, 1]
 *   u2      =  (h2 >> 11)      * 2^-53        in [0, 1)
 *   z       = sqrt(-2 ln u1) * cos(2 pi u2)    (Box-Muller, fp64, host libm)
 *   value   = std * z, rounded to nearest-even into the storage format.
 * mix64 is the SplitMix64 output function (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014; constants
 * as in Vigna's public-domain splitmix64.c).
 */
#include <stdint.h>
#include <math.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* n-th output (n >= 1) of SplitMix64 started from `state`. */
uint64_t synth_splitmix64_nth(uint64_t state, uint64_t n) {
    return mix64(state + n * GOLDEN);
}

/* Round a double to the nearest bfloat16 (ties to even), directly from the
 * double so there is no double rounding through float. */
static uint16_t dbl_to_bf16_bits(double d) {
    uint64_t b;
    memcpy(&b, &d, 8);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    if (isnan(d)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(d);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1) -> unbiased exponent e-1 */
    int ue = e - 1;
    if (ue > 127) return (uint16_t)(sign | 0x7F80u);
    if (ue < -126) {       /* bf16 subnormal: multiples of 2^-133 */
        double q = nearbyint(ldexp(a, 133));
        return (uint16_t)(sign | (uint16_t)q);   /* q == 128 is the smallest normal */
    }
    double q = nearbyint(ldexp(a, 7 - ue));      /* in [128, 256] */
    if (q >= 256.0) { q = 128.0; ue += 1; }
    if (ue > 127) return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | (uint16_t)((ue + 127) << 7) | (uint16_t)((int)q - 128));
}

/* kind: 0 = float64, 1 = float32 (RNE), 2 = bfloat16 bits (RNE). */
void synth_normal(uint64_t seed, uint64_t tensor_id, uint64_t offset, int64_t n,
                  double stdev, int kind, void *out) {
    const uint64_t stream = mix64(seed * GOLDEN + tensor_id + 1);
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) {
        uint64_t i = offset + (uint64_t)k;
        uint64_t h1 = mix64(stream + (2 * i + 1) * GOLDEN);
        uint64_t h2 = mix64(stream + (2 * i + 2) * GOLDEN);
        double u1 = (double)((h1 >> 11) + 1) * 0x1.0p-53;
        double u2 = (double)(h2 >> 11) * 0x1.0p-53;
        double z = sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
        double v = stdev * z;
        if (kind == 0) ((double *)out)[k] = v;
        else if (kind == 1) ((float *)out)[k] = (float)v;
        else ((uint16_t *)out)[k] = dbl_to_bf16_bits(v);
    }
}

/* Exposed so the generator's own rounding can be checked against known cases. */
void synth_round_bf16(const double *x, int64_t n, uint16_t *out) {
    for (int64_t k = 0; k < n; ++k) out[k] = dbl_to_bf16_bits(x[k]);
}
