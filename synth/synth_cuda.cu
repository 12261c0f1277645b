// synth_cuda.cu -- device implementation of the generator defined in synth.h.
// Same definition as synth.c, evaluated per element on the GPU so that
// multi-GB weight sets are created directly in HBM. Not part of the layer.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {
constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ULL;
constexpr double kTwoPi = 6.283185307179586;

__device__ __forceinline__ uint64_t mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ uint64_t mix_h(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}
__device__ __forceinline__ double unit_open(uint64_t bits) {
    return ((double)(bits >> 11) + 0.5) * 0x1p-53;
}
__device__ __forceinline__ double normal_at(uint64_t b, uint64_t i) {
    uint64_t p = i >> 1;
    double u1 = unit_open(mix(b + kGolden * (2 * p + 1)));
    double u2 = unit_open(mix(b + kGolden * (2 * p + 2)));
    double r = sqrt(-2.0 * log(u1));
    double th = kTwoPi * u2;
    return (i & 1) ? r * sin(th) : r * cos(th);
}
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__global__ void k_normal_bf16(uint16_t* out, int64_t n, uint64_t b, double sigma, int64_t offset) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = f32_to_bf16_rne((float)(sigma * normal_at(b, (uint64_t)(offset + j))));
}
__global__ void k_normal_f32(float* out, int64_t n, uint64_t b, double sigma, int64_t offset) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = (float)(sigma * normal_at(b, (uint64_t)(offset + j)));
}
__global__ void k_uniform_f32(float* out, int64_t n, uint64_t b, double lo, double hi, int64_t offset) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = (float)(lo + (hi - lo) * unit_open(mix(b + kGolden * ((uint64_t)(offset + j) + 1))));
}

inline uint64_t base_of(uint64_t seed, uint64_t tid) { return mix_h(seed + kGolden * (tid + 1)); }
inline int grid_for(int64_t n) {
    int64_t g = (n + 255) / 256;
    return (int)(g < 148 * 64 ? (g < 1 ? 1 : g) : 148 * 64);
}
}  // namespace

extern "C" {
int synth_cuda_fill_normal_bf16(void* out, int64_t n, uint64_t seed, uint64_t tensor_id, double sigma,
                                int64_t offset, void* stream) {
    if (n <= 0) return 0;
    k_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t*)out, n, base_of(seed, tensor_id),
                                                                  sigma, offset);
    return (int)cudaGetLastError();
}
int synth_cuda_fill_normal_f32(void* out, int64_t n, uint64_t seed, uint64_t tensor_id, double sigma,
                               int64_t offset, void* stream) {
    if (n <= 0) return 0;
    k_normal_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((float*)out, n, base_of(seed, tensor_id), sigma,
                                                                 offset);
    return (int)cudaGetLastError();
}
int synth_cuda_fill_uniform_f32(void* out, int64_t n, uint64_t seed, uint64_t tensor_id, double lo, double hi,
                                int64_t offset, void* stream) {
    if (n <= 0) return 0;
    k_uniform_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((float*)out, n, base_of(seed, tensor_id), lo, hi,
                                                                  offset);
    return (int)cudaGetLastError();
}
}
