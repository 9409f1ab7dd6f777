/*
 * Seeded synthetic inputs for the ragged 8-bit Adam bucket workloads.
 *
 * This file holds no arithmetic of the optimizer or of the layout planner:
 * it only turns (seed, stream, index) into numbers.  Both the CUDA path and
 * the CPU oracle receive the bytes it writes, so neither side generates its
 * own inputs.
 *
 * Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used in counter mode: value i of a stream
 * is mix(key + (i + 1) * 0x9E3779B97F4A7C15), so any element can be
 * regenerated on its own.  Normals use the Box-Muller transform
 * (Box & Muller, 1958) on two uniforms drawn at counters 2i and 2i+1.
 */
#include <math.h>
#include <stdint.h>

static const uint64_t GOLDEN = 0x9E3779B97F4A7C15ULL;

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Key of stream `stream` under `seed`: two mixing rounds so nearby seeds and
 * stream ids give unrelated keys. */
uint64_t synth_key(uint64_t seed, uint64_t stream) {
    return mix64(mix64(seed * GOLDEN + 0x632BE59BD9B4E019ULL) ^ (stream * 0xD1B54A32D192ED03ULL));
}

uint64_t synth_u64(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

/* Uniform double in [0, 1) with 53 random bits. */
static inline double unif(uint64_t key, uint64_t i) {
    return (double)(synth_u64(key, i) >> 11) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
    double u1 = 1.0 - unif(key, 2 * i);     /* (0, 1] so log() is finite */
    double u2 = unif(key, 2 * i + 1);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* out[j] = (float)(sigma * N(0,1)) for element indices first .. first+count-1. */
void synth_normal_f32(uint64_t key, uint64_t first, int64_t count, double sigma, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) out[j] = (float)(sigma * normal_at(key, first + (uint64_t)j));
}

/* Round a float to the nearest bfloat16, ties to even (inputs here are finite). */
static inline uint16_t to_bf16_bits(float f) {
    union { float f; uint32_t u; } v;
    v.f = f;
    uint32_t lsb = (v.u >> 16) & 1u;
    return (uint16_t)((v.u + 0x7FFFu + lsb) >> 16);
}

/* out[j] = bf16(sigma * N(0,1)) as raw bits, same element indexing. */
void synth_normal_bf16(uint64_t key, uint64_t first, int64_t count, double sigma, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j)
        out[j] = to_bf16_bits((float)(sigma * normal_at(key, first + (uint64_t)j)));
}

/* out[j] = uniform double in [0, 1), same element indexing. */
void synth_uniform_f64(uint64_t key, uint64_t first, int64_t count, double* out) {
    for (int64_t j = 0; j < count; ++j) out[j] = unif(key, first + (uint64_t)j);
}
