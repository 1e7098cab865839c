/*
 * counter_gen.c -- host implementation of the counter-based synthetic count
 * generator, in plain C for speed (the NumPy implementation in __init__.py is
 * the readable one; a CPU test checks that both agree bit for bit).
 *
 * Input generation only: no part of the resident's coding or queries.
 * z = SplitMix64 output number (s*P + p + 1) from `seed` (Steele, Lea &
 * Flood 2014; Vigna's splitmix64.c), u = z >> 11.  Per pixel class
 * (class_desc[c] = kind, offset, length, value):
 *   kind 0: Poisson by inverse CDF, count = min{k : u < thr[offset + k]};
 *   kind 1: uniform, count = z & dtype_max;
 *   kind 2: constant `value`;
 * then clipped to dtype_max.  out is [n_scans][P] of uint8 or uint16.
 */
#include <stddef.h>
#include <stdint.h>

static uint64_t mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

void wl_counter_counts(uint64_t seed, int64_t scan0, int64_t n_scans, int32_t P, const uint32_t *pixel_class,
                       const uint32_t *class_desc, const uint64_t *thr, int32_t dtype_bits, void *out)
{
    const uint32_t dmax = dtype_bits == 8 ? 0xFFu : 0xFFFFu;
    for (int64_t s = 0; s < n_scans; ++s) {
        for (int32_t p = 0; p < P; ++p) {
            const uint64_t idx = (uint64_t)(scan0 + s) * (uint64_t)P + (uint64_t)p + 1ull;
            const uint64_t z = mix(seed + idx * 0x9E3779B97F4A7C15ull);
            const uint32_t *d = class_desc + 4 * (size_t)pixel_class[p];
            uint32_t val;
            if (d[0] == 0) {
                const uint64_t u = z >> 11;
                int64_t lo = d[1], hi = (int64_t)d[1] + (d[2] > 0 ? d[2] : 1) - 1;
                while (lo < hi) {
                    const int64_t mid = (lo + hi) / 2;
                    if (u >= thr[mid])
                        lo = mid + 1;
                    else
                        hi = mid;
                }
                val = (uint32_t)(lo - (int64_t)d[1]);
            } else if (d[0] == 1) {
                val = (uint32_t)(z & dmax);
            } else {
                val = d[3];
            }
            if (val > dmax)
                val = dmax;
            if (dtype_bits == 8)
                ((uint8_t *)out)[s * (int64_t)P + p] = (uint8_t)val;
            else
                ((uint16_t *)out)[s * (int64_t)P + p] = (uint16_t)val;
        }
    }
}
