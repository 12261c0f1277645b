/* synth.c -- host implementation of the generator defined in synth.h. */
#include "synth.h"
#include <math.h>
#include <string.h>

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL
#define SYNTH_TWO_PI 6.283185307179586

static inline uint64_t mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}
static inline uint64_t base_of(uint64_t seed, uint64_t tid) { return mix(seed + SYNTH_GOLDEN * (tid + 1)); }
static inline uint64_t draw(uint64_t b, uint64_t i) { return mix(b + SYNTH_GOLDEN * (i + 1)); }
static inline double unit_open(uint64_t bits) { return ((double)(bits >> 11) + 0.5) * 0x1p-53; }

static inline double normal_at(uint64_t b, uint64_t i) {
    uint64_t p = i >> 1;
    double u1 = unit_open(draw(b, 2 * p));
    double u2 = unit_open(draw(b, 2 * p + 1));
    double r = sqrt(-2.0 * log(u1));
    double th = SYNTH_TWO_PI * u2;
    return (i & 1) ? r * sin(th) : r * cos(th);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

double synth_normal_f64(uint64_t seed, uint64_t tensor_id, uint64_t i) {
    return normal_at(base_of(seed, tensor_id), i);
}

double synth_uniform_f64(uint64_t seed, uint64_t tensor_id, uint64_t i, double lo, double hi) {
    return lo + (hi - lo) * unit_open(draw(base_of(seed, tensor_id), i));
}

void synth_fill_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                            double sigma, int64_t offset) {
    uint64_t b = base_of(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = f32_to_bf16_rne((float)(sigma * normal_at(b, (uint64_t)(offset + j))));
}

void synth_fill_normal_f32(float* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                           double sigma, int64_t offset) {
    uint64_t b = base_of(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (float)(sigma * normal_at(b, (uint64_t)(offset + j)));
}

void synth_fill_uniform_f32(float* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                            double lo, double hi, int64_t offset) {
    uint64_t b = base_of(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (float)(lo + (hi - lo) * unit_open(draw(b, (uint64_t)(offset + j))));
}
