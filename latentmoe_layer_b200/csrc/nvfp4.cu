// nvfp4.cu -- NVFP4 quantisation of the routed experts' weights.
//
// The experts' up and down projections are the layers the pages keep in NVFP4
// ("Nemotron 3 Ultra 架构 QA", Q1.3 and Q8.1; the overview names NVFP4
// quantisation for inference). Format and recipe (stated in latentmoe.h):
// E2M1 elements, one E4M3 scale per 16 elements along K, one fp32 scale per
// matrix, written in tiles of 128 rows x 64 K that the expert GEMM's producer
// copies whole. Every decision is taken from correctly rounded fp32 operations
// (__fdiv_rn, __fmul_rn), so the codes do not depend on contraction or on the
// order of evaluation. Three launches: matrix amax (as float bits; max is
// order-independent), the codes and block scales, then g = amax / 2688.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lmoe_internal.h"

namespace lmoe {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float matrix_scale(uint32_t amax_bits) {
    const float amax = __uint_as_float(amax_bits);
    return amax > 0.f ? __fdiv_rn(amax, 2688.f) : 1.f;
}

// Nearest E4M3 byte to u >= 0, ties to the even mantissa, saturating at 448.
// Below 2^-6 the grid is m * 2^-9 (m = 8 is 2^-6, byte 0x08, the first normal
// value, so the subnormal branch needs no carry). Above, the 23-bit fp32
// mantissa is rounded to 3 bits; a carry into the exponent field is the next
// binade's first value.
__device__ __forceinline__ uint32_t e4m3_nearest(float u) {
    if (!(u > 0.f)) return 0u;
    if (u >= 448.f) return 0x7Eu;
    if (u < 0.015625f) return (uint32_t)__float2int_rn(__fmul_rn(u, 512.f));
    const uint32_t b = __float_as_uint(u);
    const int e = (int)((b >> 23) & 0xFFu) - 127;  // -6 .. 8
    const uint32_t mant = b & 0x7FFFFFu, rest = mant & 0xFFFFFu;
    uint32_t code = ((uint32_t)(e + 7) << 3) | (mant >> 20);
    if (rest > 0x80000u || (rest == 0x80000u && (code & 1u))) ++code;
    return code > 0x7Eu ? 0x7Eu : code;
}

__device__ __forceinline__ float e4m3_float(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
}

// Nearest E2M1 code to q: the midpoints of 0, 0.5, 1, 1.5, 2, 3, 4, 6 are
// 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5; a midpoint goes to the even code
// (0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4).
__device__ __forceinline__ uint32_t e2m1_nearest(float q) {
    const float a = fabsf(q);
    const uint32_t m = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
                     : a <= 2.5f  ? 4u : a < 3.5f  ? 5u : a <= 5.f   ? 6u : 7u;
    return (q < 0.f ? 8u : 0u) | m;
}

// amax of each matrix as float bits (|w| of bf16 values compares as unsigned).
__global__ void k_amax(const uint4* w, long long vec_per_mat, uint32_t* amax) {
    const int m = blockIdx.y;
    const uint4* p = w + (long long)m * vec_per_mat;
    uint32_t mx = 0;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < vec_per_mat;
         i += (long long)gridDim.x * blockDim.x) {
        const uint4 v = __ldg(p + i);
        const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) mx = max(mx, max((ws[j] & 0x7FFFu) << 16, ws[j] & 0x7FFF0000u));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    __shared__ uint32_t red[32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x < 32) {
        mx = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        if (threadIdx.x == 0) atomicMax(amax + m, mx);
    }
}

// One thread per 16-element block (global row gr, block b of the row).
__global__ void k_quantize(const uint4* w, long long n_blocks, int R, int K, const uint32_t* amax, uint8_t* codes,
                           uint8_t* sf) {
    const int bpr = K / 16;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_blocks;
         i += (long long)gridDim.x * blockDim.x) {
        const long long gr = i / bpr;
        const int b = (int)(i % bpr);
        const float g = matrix_scale(__ldg(amax + gr / R));
        const uint4 v0 = __ldg(w + 2 * i), v1 = __ldg(w + 2 * i + 1);
        const uint32_t ws[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float x[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            x[2 * j] = bf16_lo(ws[j]);
            x[2 * j + 1] = bf16_hi(ws[j]);
        }
        float bmax = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(x[j]));
        const uint32_t sb = e4m3_nearest(__fdiv_rn(__fdiv_rn(bmax, g), 6.f));
        const float S = e4m3_float(sb);
        uint32_t lo = 0, hi = 0;
        if (S != 0.f) {
            const float d = __fmul_rn(S, g);
#pragma unroll
            for (int j = 0; j < 8; ++j) lo |= e2m1_nearest(__fdiv_rn(x[j], d)) << (4 * j);
#pragma unroll
            for (int j = 0; j < 8; ++j) hi |= e2m1_nearest(__fdiv_rn(x[8 + j], d)) << (4 * j);
        }
        const int k0 = b * 16;
        const long long tile = (gr / 128) * (K / 64) + k0 / 64;
        const int rr = (int)(gr % 128);
        *reinterpret_cast<uint2*>(codes + tile * 4096 + rr * 32 + (k0 % 64) / 2) = make_uint2(lo, hi);
        sf[tile * 512 + rr * 4 + (k0 % 64) / 16] = (uint8_t)sb;
    }
}

__global__ void k_matrix_scale(float* gs, long long n_mat) {
    const long long m = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (m < n_mat) gs[m] = matrix_scale(__float_as_uint(gs[m]));
}

}  // namespace

cudaError_t launch_quantize_nvfp4(const uint16_t* w, long long n_mat, int R, int K, uint8_t* codes, uint8_t* sf,
                                  float* gs, cudaStream_t s) {
    if (n_mat <= 0) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(gs, 0, (size_t)n_mat * sizeof(float), s);
    if (e != cudaSuccess) return e;
    const long long vec_per_mat = (long long)R * K / 8;
    const int sms = tc_num_sms();
    long long bx = (vec_per_mat + 255) / 256;
    const long long cap = (4LL * sms + n_mat - 1) / n_mat;
    if (bx > cap) bx = cap;
    if (bx < 1) bx = 1;
    if (n_mat > 65535) return cudaErrorInvalidValue;
    k_amax<<<dim3((unsigned)bx, (unsigned)n_mat), 256, 0, s>>>(reinterpret_cast<const uint4*>(w), vec_per_mat,
                                                               reinterpret_cast<uint32_t*>(gs));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long n_blocks = n_mat * R * (long long)(K / 16);
    long long grid = (n_blocks + 255) / 256;
    if (grid > 32LL * sms) grid = 32LL * sms;
    k_quantize<<<(unsigned)grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(w), n_blocks, R, K,
                                              reinterpret_cast<const uint32_t*>(gs), codes, sf);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_matrix_scale<<<(unsigned)((n_mat + 255) / 256), 256, 0, s>>>(gs, n_mat);
    return cudaGetLastError();
}

}  // namespace lmoe
