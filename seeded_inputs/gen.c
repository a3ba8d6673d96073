/*
 * Seeded synthetic inputs: counter-based normal bf16 values.
 *
 * Element e of tensor (seed, stream) is drawn from two splitmix64 outputs
 * (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014; the finaliser constants are the published ones) turned into
 * one standard normal by the Box-Muller transform in double precision and
 * rounded to bf16 with round-to-nearest-even.  Values depend only on
 * (seed, stream, e), so any slice can be regenerated independently and the
 * result is identical for any thread count.
 *
 * This module holds no attention arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static uint64_t splitmix64(uint64_t x)
{
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

/* key of one (seed, stream) pair */
uint64_t seeded_key(uint64_t seed, uint64_t stream)
{
    return splitmix64(splitmix64(seed) ^ (stream * 0xD1B54A32D192ED03ull));
}

/* uniform in (0, 1]: 53 random bits */
static double unit(uint64_t bits)
{
    return ((double)(bits >> 11) + 1.0) * (1.0 / 9007199254740992.0);
}

static uint16_t to_bf16_rne(double v)
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* out[e] = bf16(scale * normal(key, first + e)), e in [0, n) */
void seeded_normal_bf16(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                        double scale, uint16_t *out)
{
    const uint64_t key = seeded_key(seed, stream);
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < (int64_t)n; ++e) {
        uint64_t c = first + (uint64_t)e;
        double u1 = unit(splitmix64(key ^ (2 * c)));
        double u2 = unit(splitmix64(key ^ (2 * c + 1)));
        double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        out[e] = to_bf16_rne(scale * z);
    }
}

/* uniform doubles in (0, 1] for selecting subsets (e.g. sharpened keys) */
void seeded_uniform(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n, double *out)
{
    const uint64_t key = seeded_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < (int64_t)n; ++e)
        out[e] = unit(splitmix64(key ^ (2 * (first + (uint64_t)e))));
}
