/*
 * Seeded synthetic inputs for the Sherry 3:4 ternary matmul workloads.
 *
 * This file holds NO arithmetic of the method (no ternarisation, packing,
 * quantisation or contraction).  It only draws the fp32 weight and activation
 * tensors that both the CPU oracle and the CUDA path consume, so that the two
 * sides see bit-identical inputs.
 *
 * Generator: splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used as a counter-based stream:
 *     key        = mix(seed)
 *     bits(j)    = mix(key + (j + 1) * 0x9E3779B97F4A7C15)
 * uniform in [0,1):   (bits >> 11) * 2^-53
 * uniform in (0,1]:   ((bits >> 11) + 1) * 2^-53
 * normal (Box-Muller, pair p gives elements 2p and 2p+1):
 *     r = sqrt(-2 ln u1),  z0 = r cos(2 pi u2),  z1 = r sin(2 pi u2)
 *     u1 = uniform(0,1] of bits(2p), u2 = uniform[0,1) of bits(2p+1)
 * computed in fp64 and rounded once to fp32 after scaling by sigma.
 * Element i of a tensor is a pure function of (seed, i), so any row of a
 * large tensor can be regenerated on its own.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed) { return mix64(seed + GOLDEN); }

static inline uint64_t stream_bits(uint64_t key, uint64_t j)
{
    return mix64(key + (j + 1) * GOLDEN);
}

static inline double u01_closed_open(uint64_t b) { return (double)(b >> 11) * 0x1.0p-53; }
static inline double u01_open_closed(uint64_t b) { return (double)((b >> 11) + 1) * 0x1.0p-53; }

static inline double normal_at(uint64_t key, uint64_t i)
{
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t p = i >> 1;
    double u1 = u01_open_closed(stream_bits(key, 2 * p));
    double u2 = u01_closed_open(stream_bits(key, 2 * p + 1));
    double r = sqrt(-2.0 * log(u1));
    return (i & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
}

/* out[i] = (float)(sigma * N(0,1)[seed, offset + i]) for i in [0, n). */
void synth_normal(uint64_t seed, uint64_t offset, int64_t n, double sigma, float* out)
{
    uint64_t key = stream_key(seed);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(sigma * normal_at(key, offset + (uint64_t)i));
}

/* Raw 64-bit stream words: out[i] = bits(seed, offset + i). */
void synth_bits(uint64_t seed, uint64_t offset, int64_t n, uint64_t* out)
{
    uint64_t key = stream_key(seed);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = stream_bits(key, offset + (uint64_t)i);
}

/*
 * Heavy-tailed weights: each element i (flat index offset + i) is, with
 * probability p, replaced by +-magnitude (equiprobable sign).  The decision
 * uses uniform[0,1) of bits(spike_seed, i) < p; the sign is bit 0 of the same
 * word (1 -> negative).  Applied in place to data[0, n).
 */
void synth_spikes(uint64_t spike_seed, uint64_t offset, int64_t n, double p,
                  float magnitude, float* data)
{
    uint64_t key = stream_key(spike_seed);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t b = stream_bits(key, offset + (uint64_t)i);
        if (u01_closed_open(b) < p) data[i] = (b & 1) ? -magnitude : magnitude;
    }
}
