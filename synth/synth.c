/*
 * Seeded, counter-based generator of synthetic inputs (host side).
 *
 * This module holds no arithmetic of the method: it only draws the
 * numbers that both the oracle and the CUDA path consume (weights,
 * activations, router logits, per-expert sensitivities). The same
 * generator is implemented a second time for the device in
 * synth_dev.cu; the two use only IEEE-754 operations that are correctly
 * rounded on both processors (+, -, *, /, sqrt, exact frexp), evaluated
 * in the same order with no contraction, so they agree bit for bit.
 *
 * Published definitions used:
 *  - SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *    generators", OOPSLA 2014): state += 0x9E3779B97F4A7C15, then the
 *    variant-13 finaliser (shifts 30/27/31, multipliers 0xBF58476D1CE4E5B9
 *    and 0x94D049BB133111EB). Draw number c of stream key K is the
 *    finaliser applied to K + (c+1)*0x9E3779B97F4A7C15.
 *  - Marsaglia polar method (Marsaglia & Bray, SIAM Review 6(3), 1964) for
 *    N(0,1) pairs, with the natural log evaluated by the atanh series
 *    ln m = 2*(f + f^3/3 + f^5/5 + ...), f = (m-1)/(m+1), after reducing
 *    m to [sqrt(1/2), sqrt(2)) with frexp.
 *
 * Build with -ffp-contract=off so no multiply-add is fused.
 */
#include <stdint.h>
#include <math.h>

static inline uint64_t syn_fin(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t syn_stream_key(uint64_t seed, uint64_t stream)
{
    return syn_fin(seed ^ syn_fin(stream ^ 0xD1B54A32D192ED03ULL));
}

static inline uint64_t syn_draw(uint64_t key, uint64_t ctr)
{
    return syn_fin(key + (ctr + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

/* uniform on (-1, 1): (v + 0.5) * 2^-52 with v in [-2^52, 2^52) */
static inline double syn_sym_unit(uint64_t u)
{
    int64_t v = (int64_t)(u >> 11) - (int64_t)4503599627370496LL;
    return ((double)v + 0.5) * (1.0 / 4503599627370496.0);
}

static double syn_log(double s)
{
    int e;
    double m = frexp(s, &e);
    if (m < 0.70710678118654752440) {
        m = m * 2.0;
        e -= 1;
    }
    double f = (m - 1.0) / (m + 1.0);
    double f2 = f * f;
    double p = 1.0 / 25.0;
    for (int i = 11; i >= 0; --i)
        p = p * f2 + 1.0 / (double)(2 * i + 1);
    return (double)e * 0.69314718055994530942 + (2.0 * f) * p;
}

/* N(0,1) sample number idx of the stream: pair idx/2, member idx%2 */
static double syn_normal_at(uint64_t key, uint64_t idx)
{
    uint64_t pair = idx >> 1;
    for (int a = 0; a < 32; ++a) {
        double u = syn_sym_unit(syn_draw(key, pair * 64ULL + 2ULL * (uint64_t)a));
        double v = syn_sym_unit(syn_draw(key, pair * 64ULL + 2ULL * (uint64_t)a + 1ULL));
        double s = u * u + v * v;
        if (s >= 1.0 || s == 0.0)
            continue;
        double t = (-2.0 * syn_log(s)) / s;
        double r = sqrt(t);
        return (idx & 1ULL) ? v * r : u * r;
    }
    return 0.0;
}

static inline uint16_t syn_f32_to_bf16(float f)
{
    union { float f; uint32_t u; } c;
    c.f = f;
    uint32_t u = c.u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* out[i] = (float)(scale * z(start + i)) */
void syn_normal_f32(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
                    double scale, float *out)
{
    uint64_t key = syn_stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(scale * syn_normal_at(key, start + (uint64_t)i));
}

void syn_normal_f64(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
                    double scale, double *out)
{
    uint64_t key = syn_stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i)
        out[i] = scale * syn_normal_at(key, start + (uint64_t)i);
}

/* bf16 (round to nearest even) of (float)(scale * z(start + i)) */
void syn_normal_bf16(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
                     double scale, uint16_t *out)
{
    uint64_t key = syn_stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i)
        out[i] = syn_f32_to_bf16((float)(scale * syn_normal_at(key, start + (uint64_t)i)));
}

/* raw 64-bit draws, for permutations and other integer choices */
void syn_u64(uint64_t seed, uint64_t stream, uint64_t start, int64_t n, uint64_t *out)
{
    uint64_t key = syn_stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i)
        out[i] = syn_draw(key, start + (uint64_t)i);
}
