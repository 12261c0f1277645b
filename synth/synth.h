/*
 * synth.h -- seeded, counter-based synthetic input generator (CPU side).
 *
 * This module only makes test and benchmark inputs. It holds none of the
 * LatentMoE arithmetic. Both the CPU oracle and the GPU harness draw their
 * inputs from the same definition, implemented twice (synth.c for the host,
 * synth_cuda.cu for the device):
 *
 *   mix(z)      = the splitmix64 output function (Steele, Lea and Flood,
 *                 "Fast splittable pseudorandom number generators", 2014):
 *                 z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                 z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
 *   base(s, t)  = mix(s + G * (t + 1))            G = 0x9E3779B97F4A7C15
 *   draw(b, i)  = mix(b + G * (i + 1))            (the i-th splitmix64 output)
 *   unit(bits)  = ((bits >> 11) + 0.5) * 2^-53    in the open interval (0, 1)
 *
 *   normal(s, t, i): Box-Muller on the pair p = floor(i / 2):
 *       u1 = unit(draw(b, 2p)), u2 = unit(draw(b, 2p + 1)),
 *       r = sqrt(-2 ln u1), th = 2 pi u2,
 *       value = r cos th for even i, r sin th for odd i          (fp64)
 *   uniform(s, t, i) = lo + (hi - lo) * unit(draw(b, i))           (fp64)
 *
 * Stored values: fp32 = the fp64 value rounded to nearest fp32; bf16 = that
 * fp32 value rounded to nearest-even bf16 (integer bit rounding, NaN-free).
 * `offset` selects the first element index, so any slice of a tensor can be
 * generated independently of the rest.
 */
#ifndef LMOE_SYNTH_H
#define LMOE_SYNTH_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

double synth_normal_f64(uint64_t seed, uint64_t tensor_id, uint64_t i);
double synth_uniform_f64(uint64_t seed, uint64_t tensor_id, uint64_t i, double lo, double hi);

/* out[j] = bf16(fp32(sigma * normal(seed, tensor_id, offset + j))), j < n */
void synth_fill_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                            double sigma, int64_t offset);
/* out[j] = fp32(sigma * normal(seed, tensor_id, offset + j)) */
void synth_fill_normal_f32(float* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                           double sigma, int64_t offset);
/* out[j] = fp32(uniform(seed, tensor_id, offset + j, lo, hi)) */
void synth_fill_uniform_f32(float* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                            double lo, double hi, int64_t offset);

#ifdef __cplusplus
}
#endif
#endif
