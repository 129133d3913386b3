/*
 * Seeded synthetic inputs: iid N(0, 1) values rounded to bf16.
 *
 * Counter-based, so any slice of a tensor can be produced independently and
 * in parallel, and every run on every machine sees the same bytes:
 *
 *   mix(z)       SplitMix64 output function (Steele, Lea and Flood,
 *                "Fast splittable pseudorandom number generators", 2014)
 *   base         mix(seed + G * (tensor_id + 1)),  G = 0x9E3779B97F4A7C15
 *   draw(i)      mix(base + G * (i + 1))
 *   u(i)         ((draw(i) >> 11) + 1) * 2^-53, in (0, 1]
 *   pair k       Box-Muller: r = sqrt(-2 ln u(2k)), t = 2 pi u(2k+1),
 *                x[2k] = r cos t, x[2k+1] = r sin t
 *   rounding     double -> float (round to nearest even) -> bf16 (round to
 *                nearest even on the float's bits)
 *
 * This file holds no attention arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static uint64_t mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static double unit(uint64_t base, uint64_t i)
{
    uint64_t d = mix(base + GOLDEN * (i + 1));
    return (double)((d >> 11) + 1) * (1.0 / 9007199254740992.0);
}

static uint16_t float_to_bf16_rne(float f)
{
    uint32_t b;
    memcpy(&b, &f, sizeof b);
    uint32_t lsb = (b >> 16) & 1u;
    b += 0x7FFFu + lsb;
    return (uint16_t)(b >> 16);
}

static const double TWO_PI = 6.283185307179586476925286766559;

/* out[e] for e in [start, start + n) of the tensor stream (seed, tensor_id). */
void synth_normal_bf16(uint64_t seed, uint64_t tensor_id, int64_t start, int64_t n, uint16_t *out)
{
    uint64_t base = mix(seed + GOLDEN * (tensor_id + 1));
#pragma omp parallel for schedule(static)
    for (int64_t e = start; e < start + n; e++) {
        int64_t k = e >> 1;
        double r = sqrt(-2.0 * log(unit(base, 2 * (uint64_t)k)));
        double t = TWO_PI * unit(base, 2 * (uint64_t)k + 1);
        double x = (e & 1) ? r * sin(t) : r * cos(t);
        out[e - start] = float_to_bf16_rne((float)x);
    }
}
