/*
 * Seeded synthetic inputs for the MoE layer forward.
 *
 * This module is shared by the CPU oracle and by the GPU path's tests and
 * benchmark.  It holds no arithmetic of the MoE method itself: it only turns
 * (seed, tensor id, element index) into a normally distributed number and
 * rounds it to the storage type.
 *
 * Generator (counter based, so any slice of any tensor can be regenerated
 * without producing the elements before it):
 *   SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 *   generators", OOPSLA 2014; constants as in Vigna's public-domain
 *   splitmix64.c).  The n-th output (n >= 1) of a SplitMix64 stream started at
 *   state s is mix(s + n * 0x9E3779B97F4A7C15).
 *   Stream start for a tensor: s = mix(seed * 2^32 + tensor_id).
 *   Element pair p uses outputs n = 2p+1 and n = 2p+2:
 *     u1 = ((o1 >> 11) + 0.5) * 2^-53   in (0, 1)
 *     u2 =  (o2 >> 11)        * 2^-53   in [0, 1)
 *   Box-Muller (1958): r = sqrt(-2 ln u1), element 2p = r cos(2 pi u2),
 *   element 2p+1 = r sin(2 pi u2).
 *   The normal deviate is multiplied by `stddev` in double precision and
 *   rounded to nearest-even float; for bf16 storage the float is rounded to
 *   nearest-even bf16 (NaN cannot occur).
 */
#include <stdint.h>
#include <math.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_start(uint64_t seed, uint64_t tensor_id)
{
    return sm_mix((seed << 32) + tensor_id);
}

static inline double normal_at(uint64_t s0, uint64_t i)
{
    uint64_t p = i >> 1;
    uint64_t o1 = sm_mix(s0 + (2 * p + 1) * GOLDEN_GAMMA);
    uint64_t o2 = sm_mix(s0 + (2 * p + 2) * GOLDEN_GAMMA);
    double u1 = ((double)(o1 >> 11) + 0.5) * 0x1.0p-53;
    double u2 = (double)(o2 >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double a = 2.0 * M_PI * u2;
    return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Raw SplitMix64 output n (n >= 1) of the stream (seed, tensor_id). */
uint64_t synth_u64(uint64_t seed, uint64_t tensor_id, uint64_t n)
{
    return sm_mix(stream_start(seed, tensor_id) + n * GOLDEN_GAMMA);
}

/* Fill out[0..count) with elements [start, start+count) of the tensor
 * (seed, tensor_id), scaled by stddev, stored as float (dtype 0) or bf16 bits
 * (dtype 1).  Threads: OpenMP over elements. */
void synth_normal(uint64_t seed, uint64_t tensor_id, uint64_t start,
                  uint64_t count, double stddev, int dtype, void *out)
{
    uint64_t s0 = stream_start(seed, tensor_id);
    if (dtype == 0) {
        float *o = (float *)out;
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < (int64_t)count; ++j)
            o[j] = (float)(normal_at(s0, start + (uint64_t)j) * stddev);
    } else {
        uint16_t *o = (uint16_t *)out;
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < (int64_t)count; ++j)
            o[j] = f32_to_bf16_rne((float)(normal_at(s0, start + (uint64_t)j) * stddev));
    }
}

/* Uniform integers in [0, n) (used for synthetic expert assignments in the
 * dispatch tests): (o >> 11) * n >> 53 of SplitMix64 output index+1. */
void synth_uniform_int(uint64_t seed, uint64_t tensor_id, uint64_t start,
                       uint64_t count, uint32_t n, int32_t *out)
{
    uint64_t s0 = stream_start(seed, tensor_id);
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)count; ++j) {
        uint64_t o = sm_mix(s0 + (start + (uint64_t)j + 1) * GOLDEN_GAMMA);
        double u = (double)(o >> 11) * 0x1.0p-53;
        uint32_t v = (uint32_t)(u * (double)n);
        out[j] = (int32_t)(v < n ? v : n - 1);
    }
}
