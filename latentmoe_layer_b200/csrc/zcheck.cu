// zcheck.cu -- exact bf16 rounding of the latent z = bf16(x W_fc1^T).
//
// z is the layer's most sensitive rounding point: every routed expert of a
// token reads the same z row, so one z element that rounds to the other bf16
// neighbour than the exact dot product would moves all k expert outputs of
// that token. The tensor cores accumulate in fp32 (error ~1e-7 absolute at
// these shapes), so a small fraction of elements whose fp32 value lies next
// to a bf16 rounding midpoint can round the other way. Those elements are
// found and re-decided exactly, the same way the router re-decides tokens
// near its selection edge:
//   1. the fc1 GEMM writes z in fp32;
//   2. k_round_flag rounds every element to bf16 (nearest-even) and appends the
//      elements within `delta` of a rounding midpoint to a list;
//   3. k_recheck recomputes each listed element as an error-free sum of the
//      exact bf16 x bf16 products (each formed exactly in fp32) in double-fp32
//      arithmetic and stores the nearest-even bf16 rounding of that sum.
// The result equals the exactly rounded z whenever the fp32 error is below
// delta, and the set of listed elements, hence z, is deterministic.
#include <cuda_bf16.h>
#include <stdint.h>

#include "lmoe_internal.h"

namespace lmoe {
namespace {

// Distance test to the bf16 rounding midpoints around |v| (fp32 bit patterns
// are monotonic in the magnitude, so the midpoints are the truncated pattern
// +- 0x8000). Values whose truncation is 0 (|v| below the smallest normal
// bf16) are always listed.
__device__ __forceinline__ bool near_midpoint(float v, float delta) {
    const uint32_t u = __float_as_uint(v) & 0x7FFFFFFFu;
    const uint32_t t = u & 0xFFFF0000u;
    if (t == 0) return true;
    const float a = __uint_as_float(u);
    const float mid = __uint_as_float(t + 0x8000u);   // between t and the next bf16 value
    const float below = __uint_as_float(t - 0x8000u);  // between t and the previous bf16 value
    return fabsf(a - mid) < delta || a - below < delta;
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Error-free transformation of a sum (Knuth's TwoSum in round-to-nearest
// fp32): s + e == a + b exactly.
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
    s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// Nearest-even bf16 of hi + lo, where hi = fl32(hi + lo) and |lo| <= ulp(hi)/2.
// Every bf16 rounding midpoint is an fp32 number, so hi + lo lies on the same
// side of each midpoint as hi unless hi is a midpoint itself; then the sign of
// lo decides (lo == 0 is an exact tie: nearest even).
__device__ __forceinline__ uint16_t bf16_rn_of_pair(float hi, float lo) {
    const uint32_t u = __float_as_uint(hi);
    if ((u & 0xFFFFu) == 0x8000u && lo != 0.f) {
        const uint32_t t = u >> 16;  // hi truncated toward zero
        return (uint16_t)(((lo > 0.f) == (hi > 0.f)) ? t + 1u : t);
    }
    return (uint16_t)bf16_bits_rn(hi);
}

// One warp per row of z32 [rows, L] (L a multiple of 4): z = bf16(z32), and
// the near-midpoint elements appended to list (row, column) with one atomic
// per warp and 128-column step. Entries past `cap` are counted, not written.
__global__ void __launch_bounds__(256) k_round_flag(const float* __restrict__ z32, uint16_t* __restrict__ z,
                                                    int rows, int L, float delta, int2* __restrict__ list, int cap,
                                                    int* __restrict__ count) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int L4 = L / 4;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
        const float4* src = reinterpret_cast<const float4*>(z32 + (size_t)r * L);
        uint2* dst = reinterpret_cast<uint2*>(z + (size_t)r * L);
        for (int c0 = 0; c0 < L4; c0 += 32) {
            const int c4 = c0 + lane;
            uint32_t flags = 0;
            if (c4 < L4) {
                const float4 v = src[c4];
                dst[c4] = make_uint2(bf16_bits_rn(v.x) | (bf16_bits_rn(v.y) << 16),
                                     bf16_bits_rn(v.z) | (bf16_bits_rn(v.w) << 16));
                flags = (near_midpoint(v.x, delta) ? 1u : 0u) | (near_midpoint(v.y, delta) ? 2u : 0u) |
                        (near_midpoint(v.z, delta) ? 4u : 0u) | (near_midpoint(v.w, delta) ? 8u : 0u);
            }
            const int nf = __popc(flags);
            int incl = nf;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            int base = 0;
            if (lane == 31 && total > 0) base = atomicAdd(count, total);
            base = __shfl_sync(0xffffffffu, base, 31);
            int pos = base + incl - nf;
            for (int j = 0; j < 4; ++j)
                if ((flags >> j) & 1u) {
                    if (pos < cap) list[pos] = make_int2(r, 4 * c4 + j);
                    ++pos;
                }
        }
    }
}

// One warp per listed element: z[row, col] = bf16(sum_k x[row, k] w[col, k])
// (K a multiple of 8). Each product of two bf16 values has at most 16
// significant bits, so it is exact in fp32 (unless it falls below fp32's
// normal range, 2^-126); the products are summed without
// error into an unevaluated pair hi + lo (TwoSum per product, the error terms
// summed in lo), so no fp64 conversion is needed. The pair's relative error is
// about K * 2^-48 (lo's own rounding), far below the re-rounding margin.
__global__ void __launch_bounds__(256) k_recheck(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, int K,
                                                 int rows, int* err, const int2* __restrict__ list,
                                                 const int* __restrict__ count, int cap, uint16_t* __restrict__ z,
                                                 int L) {
    const int n = min(*count, cap);
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int K8 = K / 8;
    for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += nwarps) {
        const int2 e = list[i];
        if (!lmoe_check((unsigned)e.x < (unsigned)rows && (unsigned)e.y < (unsigned)L, err)) continue;
        const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)e.x * K);
        const uint4* wr = reinterpret_cast<const uint4*>(w + (size_t)e.y * K);
        float hi = 0.f, lo = 0.f;
        for (int k = lane; k < K8; k += 32) {
            const uint4 a = __ldg(xr + k), b = __ldg(wr + k);
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float err;
                two_sum(hi, __fmul_rn(__uint_as_float(av[j] << 16), __uint_as_float(bv[j] << 16)), hi, err);
                lo = __fadd_rn(lo, err);
                two_sum(hi, __fmul_rn(__uint_as_float(av[j] & 0xFFFF0000u), __uint_as_float(bv[j] & 0xFFFF0000u)),
                        hi, err);
                lo = __fadd_rn(lo, err);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float oh = __shfl_xor_sync(0xffffffffu, hi, o), ol = __shfl_xor_sync(0xffffffffu, lo, o);
            float err;
            two_sum(hi, oh, hi, err);
            lo = __fadd_rn(__fadd_rn(lo, ol), err);
        }
        float err;
        two_sum(hi, lo, hi, err);  // renormalise: hi = fl(hi + lo), err the exact remainder
        if (lane == 0) z[(size_t)e.x * L + e.y] = bf16_rn_of_pair(hi, err);
    }
}

int grid_for(long long warps_of_work, int cap_blocks) {
    long long g = (warps_of_work + 7) / 8;  // 8 warps per 256-thread block
    if (g < 1) g = 1;
    return (int)(g < cap_blocks ? g : cap_blocks);
}

}  // namespace

cudaError_t launch_z_round_flag(const float* z32, uint16_t* z, int rows, int L, float delta, int2* list, int cap,
                                int* count, int sms, cudaStream_t s) {
    k_round_flag<<<grid_for(rows, sms * 8), 256, 0, s>>>(z32, z, rows, L, delta, list, cap, count);
    return cudaGetLastError();
}

cudaError_t launch_z_recheck(const uint16_t* x, const uint16_t* w, int K, int rows, int* err, const int2* list,
                             const int* count, int cap, uint16_t* z, int L, int sms, cudaStream_t s) {
    k_recheck<<<sms * 8, 256, 0, s>>>(x, w, K, rows, err, list, count, cap, z, L);
    return cudaGetLastError();
}

}  // namespace lmoe
