/*
 * synth_gen.c -- the counter-based random streams of the synthetic inputs and
 * their rounding to the working dtype.  Used through synth.py by the tests and
 * the benchmark; holds no Monarch attention arithmetic.
 *
 * SplitMix64 (Steele, Lea and Flood, OOPSLA 2014; Vigna's 64-bit finaliser):
 *   element i of the stream with key K is mix(K + (i + 1) * 0x9E3779B97F4A7C15),
 *   mix(z) = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
 *            z *= 0x94D049BB133111EB; z ^= z >> 31.
 * Uniform in (0, 1]: ((mix >> 11) + 1) * 2^-53.
 * Box-Muller (Box and Muller, 1958) on consecutive pairs (u1, u2):
 *   r = sqrt(-2 ln u1), z0 = r cos(2 pi u2), z1 = r sin(2 pi u2).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static double uniform_at(uint64_t key, int64_t i)
{
    uint64_t z = mix64(key + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ULL);
    return ((double)(z >> 11) + 1.0) * (1.0 / 9007199254740992.0);
}

uint64_t synth_mix64(uint64_t z) { return mix64(z); }

void synth_uniform53(uint64_t key, int64_t start, int64_t count, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++)
        out[i] = uniform_at(key, start + i);
}

void synth_normals(uint64_t key, int64_t count, double *out)
{
    const int64_t pairs = (count + 1) / 2;
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < pairs; p++) {
        double u1 = uniform_at(key, 2 * p), u2 = uniform_at(key, 2 * p + 1);
        double r = sqrt(-2.0 * log(u1)), th = two_pi * u2;
        out[2 * p] = r * cos(th);
        if (2 * p + 1 < count)
            out[2 * p + 1] = r * sin(th);
    }
}

/* Round to nearest bfloat16 (ties to even) straight from float64; writes the
 * rounded value (exact in float64) and/or its 16-bit storage. */
void synth_round_bf16(const double *x, int64_t n, double *rounded, uint16_t *bits)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        double v = x[i], r;
        if (fabs(v) >= 0x1p-126 || v == 0.0) {
            uint64_t b;
            memcpy(&b, &v, 8);
            const uint64_t drop = 45;                    /* 52 - 7 mantissa bits kept */
            uint64_t keep = b >> drop, rem = b & ((1ULL << drop) - 1), half = 1ULL << (drop - 1);
            if (rem > half || (rem == half && (keep & 1)))
                keep++;
            b = keep << drop;
            memcpy(&r, &b, 8);
        } else {                                         /* bf16 subnormal spacing 2^-133 */
            r = rint(v * 0x1p133) * 0x1p-133;
        }
        if (rounded)
            rounded[i] = r;
        if (bits) {
            float f = (float)r;
            uint32_t u;
            memcpy(&u, &f, 4);
            bits[i] = (uint16_t)(u >> 16);
        }
    }
}
