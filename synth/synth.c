/*
 * synth.c -- seeded synthetic inputs shared by the oracle tests and the GPU
 * path.  It holds none of the method's arithmetic: it only draws latent fp32
 * weights and int8 activations.
 *
 * Generator: a counter-based stream built on the splitmix64 output function
 * (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014):
 *     mix(z)   = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                z ^= z >> 27; z *= 0x94D049BB133111EB; z ^ (z >> 31)
 *     r(s, c)  = mix(mix(s + G) + (c + 1) * G),      G = 0x9E3779B97F4A7C15
 *     u(s, c)  = ((r(s, c) >> 11) + 0.5) * 2^-53      uniform on (0, 1)
 * Normal draw number i of seed s (Box-Muller, double precision):
 *     z(s, i)  = sqrt(-2 ln u(s, 2i)) * cos(2 pi u(s, 2i + 1))
 * int8 uniform on the 255 integers [-127, 127]:
 *     v(s, i)  = ((r(s, i) >> 32) * 255 >> 32) - 127
 * Clipped-normal int8 activations: round(127 * clip(z / 3, -1, 1)), round
 * half away from zero.
 */
#include <stdint.h>
#include <math.h>

#define SYN_G 0x9E3779B97F4A7C15ull

static inline uint64_t syn_mix(uint64_t z)
{
    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27; z *= 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t synth_u64(uint64_t seed, uint64_t ctr)
{
    return syn_mix(syn_mix(seed + SYN_G) + (ctr + 1) * SYN_G);
}

static inline double syn_uniform(uint64_t key, uint64_t ctr)
{
    uint64_t r = syn_mix(key + (ctr + 1) * SYN_G);
    return ((double)(r >> 11) + 0.5) * 0x1p-53;
}

static inline double syn_normal(uint64_t key, uint64_t i)
{
    const double two_pi = 6.283185307179586476925286766559;
    double u1 = syn_uniform(key, 2 * i), u2 = syn_uniform(key, 2 * i + 1);
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

/* out[j] = (float)(sigma * z(seed, offset + j)), j < n */
void synth_normal_f32(uint64_t seed, uint64_t offset, int64_t n, double sigma, float *out)
{
    const uint64_t key = syn_mix(seed + SYN_G);
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; j++)
        out[j] = (float)(sigma * syn_normal(key, offset + (uint64_t)j));
}

/* out[j] = v(seed, offset + j) in [-127, 127] */
void synth_int8_uniform(uint64_t seed, uint64_t offset, int64_t n, int8_t *out)
{
    const uint64_t key = syn_mix(seed + SYN_G);
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; j++) {
        uint64_t r = syn_mix(key + (offset + (uint64_t)j + 1) * SYN_G);
        out[j] = (int8_t)((int64_t)(((r >> 32) * 255u) >> 32) - 127);
    }
}

/* out[j] = round(127 * clip(z(seed, offset + j) / 3, -1, 1)) */
void synth_int8_clipped_normal(uint64_t seed, uint64_t offset, int64_t n, int8_t *out)
{
    const uint64_t key = syn_mix(seed + SYN_G);
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; j++) {
        double z = syn_normal(key, offset + (uint64_t)j) / 3.0;
        if (z > 1.0) z = 1.0;
        if (z < -1.0) z = -1.0;
        out[j] = (int8_t)round(127.0 * z);
    }
}
