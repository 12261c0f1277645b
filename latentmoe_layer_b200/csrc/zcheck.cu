// zcheck.cu -- exact bf16 rounding of the layer's GEMM outputs.
//
// z = bf16(x W_fc1^T) is the layer's most sensitive rounding point: every
// routed expert of a token reads the same z row, so one z element that rounds
// to the other bf16 neighbour than the exact dot product moves all k expert
// outputs of that token. The tensor cores accumulate in fp32 (error up to a few
// 1e-6 at these shapes), so the elements whose fp32 value lies next to a bf16
// rounding midpoint can round the other way. Those elements are found and
// re-decided exactly, the way the router re-decides tokens near its selection
// edge:
//   1. the fc1 GEMM writes z in fp32;
//   2. k_round_flag rounds every element to bf16 (nearest-even) and lists the
//      elements within the margin c0 + c1 |z| of a rounding midpoint;
//   3. k_recheck recomputes each listed element as an error-free sum of the
//      exact bf16 x bf16 products (each formed exactly in fp32) in double-fp32
//      arithmetic and stores the nearest-even bf16 rounding of that sum.
// The result equals the exactly rounded z whenever the fp32 error of an element
// is below its margin, and the set of listed elements, hence z, is
// deterministic.
//
// The relu2 activations (a_e of the experts, a_s of the shared expert) are the
// next rounding points. A flipped rounding of a = h^2 moves the output by about
// one bf16 step of a, which grows as h^2, so the flips that matter are those of
// the large activations: the GEMM epilogues list the activations with h above a
// threshold whose fp32 value lies within the accumulation-error margin of a
// midpoint, and k_recheck<relu2> recomputes them the same way.
#include <cuda_bf16.h>
#include <algorithm>
#include <stdint.h>

#include "lmoe_internal.h"

namespace lmoe {
namespace {

// Distance test to the bf16 rounding midpoints around |v| (fp32 bit patterns
// are monotonic in the magnitude, so the midpoints are the truncated pattern
// +- 0x8000), with the margin c0 + c1 |v|. Values whose truncation is 0 (|v|
// below the smallest normal bf16) are always listed.
__device__ __forceinline__ bool near_midpoint(float v, float c0, float c1) {
    const uint32_t u = __float_as_uint(v) & 0x7FFFFFFFu;
    const uint32_t t = u & 0xFFFF0000u;
    if (t == 0) return true;
    const float a = __uint_as_float(u);
    const float delta = c0 + c1 * a;
    const float mid = __uint_as_float(t + 0x8000u);   // between t and the next bf16 value
    const float below = __uint_as_float(t - 0x8000u);  // between t and the previous bf16 value
    return fabsf(a - mid) < delta || a - below < delta;
}

// Nearest-even bf16 of a double: round the 52-bit mantissa to 7 bits on the
// integer pattern (ties to even); the value, now of 8 significant bits, is
// exact as a float. (Normal range.)
__device__ __forceinline__ uint16_t bf16_rn_from_double(double v) {
    unsigned long long b = (unsigned long long)__double_as_longlong(v);
    b += 0x00000FFFFFFFFFFFull + ((b >> 45) & 1ull);
    b &= ~0x00001FFFFFFFFFFFull;
    return (uint16_t)(__float_as_uint((float)__longlong_as_double((long long)b)) >> 16);
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

// Error-free dot product of one lane's share of two bf16 rows (uint4 = 8 values,
// vectors k = lane, lane + 32, ... < K8): the exact products are summed into
// four independent hi + lo chains (one per bf16 pair of the vector, so the
// TwoSum dependency chains interleave), then merged without error. Returns the
// lane's pair; the caller reduces the warp.
template <typename LoadA>
__device__ __forceinline__ void dot_pairs(LoadA load_a, const uint4* __restrict__ wr, int K8, int lane, float& hi,
                                          float& lo) {
    float h[4] = {0.f, 0.f, 0.f, 0.f}, l[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int k = lane; k < K8; k += 32) {
        const uint4 a = load_a(k), b = __ldg(wr + k);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float e;
            two_sum(h[j], __fmul_rn(__uint_as_float(av[j] << 16), __uint_as_float(bv[j] << 16)), h[j], e);
            l[j] = __fadd_rn(l[j], e);
            two_sum(h[j], __fmul_rn(__uint_as_float(av[j] & 0xFFFF0000u), __uint_as_float(bv[j] & 0xFFFF0000u)), h[j],
                    e);
            l[j] = __fadd_rn(l[j], e);
        }
    }
    hi = h[0];
    lo = l[0];
#pragma unroll
    for (int j = 1; j < 4; ++j) {
        float e;
        two_sum(hi, h[j], hi, e);
        lo = __fadd_rn(__fadd_rn(lo, l[j]), e);
    }
}

// Warp reduction of the lanes' pairs (error-free merges), then the
// renormalised pair: hi = fl(hi + lo), lo the exact remainder.
__device__ __forceinline__ void warp_reduce_pair(float& hi, float& lo) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float oh = __shfl_xor_sync(0xffffffffu, hi, o), ol = __shfl_xor_sync(0xffffffffu, lo, o);
        float e;
        two_sum(hi, oh, hi, e);
        lo = __fadd_rn(__fadd_rn(lo, ol), e);
    }
    float rest;
    two_sum(hi, lo, hi, rest);
    lo = rest;
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

// One warp per segment of up to 2048 columns of a row of z32 [rows, L] (L a
// multiple of 4): z = bf16(z32), and the elements within m0 + m1 |z| of a
// rounding midpoint appended to list as (row, column), the segment's entries
// contiguous (one atomic per segment), with the segment recorded in rowtab as
// {row, first entry, entries}. Entries past `cap` are counted, not written.
constexpr int kSegCols = 2048;
__global__ void __launch_bounds__(256) k_round_flag(const float* __restrict__ z32, uint16_t* __restrict__ z,
                                                    int rows, int L, float m0, float m1, int2* __restrict__ list,
                                                    int cap, int* __restrict__ count, int4* __restrict__ rowtab,
                                                    int* __restrict__ nrowtab) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int L4 = L / 4, segs = (L + kSegCols - 1) / kSegCols;
    for (long long item = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; item < (long long)rows * segs;
         item += nwarps) {
        const int r = (int)(item / segs), c40 = (int)(item % segs) * (kSegCols / 4);
        const int c41 = min(L4, c40 + kSegCols / 4);
        const float4* src = reinterpret_cast<const float4*>(z32 + (size_t)r * L);
        uint2* dst = reinterpret_cast<uint2*>(z + (size_t)r * L);
        unsigned long long flags = 0;  // bit 4 s + j: element j of this lane's float4 at step s
        for (int s = 0; c40 + 32 * s < c41; ++s) {
            const int c4 = c40 + 32 * s + lane;
            if (c4 < c41) {
                const float4 v = src[c4];
                dst[c4] = make_uint2(bf16_bits_rn(v.x) | (bf16_bits_rn(v.y) << 16),
                                     bf16_bits_rn(v.z) | (bf16_bits_rn(v.w) << 16));
                const unsigned f = (near_midpoint(v.x, m0, m1) ? 1u : 0u) | (near_midpoint(v.y, m0, m1) ? 2u : 0u) |
                                   (near_midpoint(v.z, m0, m1) ? 4u : 0u) | (near_midpoint(v.w, m0, m1) ? 8u : 0u);
                flags |= (unsigned long long)f << (4 * s);
            }
        }
        const int nf = __popcll(flags);
        int incl = nf;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (total == 0) continue;
        int base = 0;
        if (lane == 31) {
            base = atomicAdd(count, total);
            const int t = atomicAdd(nrowtab, 1);  // rows * segs entries of room: never past the table
            rowtab[t] = make_int4(r, base, total, 0);
        }
        int pos = __shfl_sync(0xffffffffu, base, 31) + incl - nf;
        while (flags) {
            const int b = __ffsll((long long)flags) - 1;
            flags &= flags - 1ull;
            if (pos < cap) list[pos] = make_int2(r, 4 * (c40 + 32 * (b >> 2) + lane) + (b & 3));
            ++pos;
        }
    }
}

// Exact re-rounding of the listed z elements, `split` CTAs per segment of
// rowtab (more than one when there are few rows, so the entries spread over
// the SMs): the segment's row of x (K bf16, K a multiple of 8) is staged in
// shared memory, and each warp takes one listed element at a time, streaming
// its row of W (fc1_latent_proj, resident in L2 across the launch). The sum is
// the error-free double-fp32 sum of k_recheck.
__global__ void __launch_bounds__(256) k_recheck_rows(const uint16_t* __restrict__ A, int a_rows,
                                                      const uint16_t* __restrict__ W, int w_rows, int K, int* err,
                                                      const int2* __restrict__ list, int cap,
                                                      const int4* __restrict__ rowtab, const int* __restrict__ nrowtab,
                                                      uint16_t* __restrict__ out, int ldo, int split) {
    extern __shared__ uint4 xs[];  // K / 8 vectors
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int K8 = K / 8;
    const long long n = (long long)*nrowtab * split;
    for (long long item = blockIdx.x; item < n; item += gridDim.x) {
        const int part = (int)(item % split);  // this CTA's share of the segment's entries
        const int4 rt = rowtab[item / split];
        if (!lmoe_check((unsigned)rt.x < (unsigned)a_rows, err)) continue;  // uniform over the CTA
        __syncthreads();
        const uint4* xr = reinterpret_cast<const uint4*>(A + (size_t)rt.x * K);
        for (int k = threadIdx.x; k < K8; k += blockDim.x) xs[k] = __ldg(xr + k);
        __syncthreads();
        const int e1 = min(rt.y + rt.z, cap);
        for (int e = rt.y + part * nw + warp; e < e1; e += nw * split) {
            const int2 ent = list[e];
            if (!lmoe_check((unsigned)ent.y < (unsigned)w_rows, err)) continue;
            const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)ent.y * K);
            float hi, lo;
            dot_pairs([&](int k) { return xs[k]; }, wr, K8, lane, hi, lo);
            warp_reduce_pair(hi, lo);
            if (lane == 0) out[(size_t)rt.x * ldo + ent.y] = bf16_rn_of_pair(hi, lo);
        }
    }
}

// One warp per listed element (row, wrow): out[row, wrow % ldo] = the exact
// bf16 rounding of h = sum_k A[row, k] W[wrow, k] (kRelu2: of max(h, 0)^2),
// K a multiple of 8. Each product of two bf16 values has at most 16
// significant bits, so it is exact in fp32 (unless it falls below fp32's
// normal range, 2^-126); the products are summed without error into an
// unevaluated pair hi + lo (TwoSum per product, the error terms summed in lo),
// so no fp64 conversion is needed per product. The pair's relative error is
// about K * 2^-48 (lo's own rounding), far below any margin. kRelu2 squares
// hi + lo in fp64 (exact to 2^-53) before rounding.
template <bool kRelu2>
__global__ void __launch_bounds__(256) k_recheck(const uint16_t* __restrict__ A, int a_rows,
                                                 const uint16_t* __restrict__ W, int w_rows, int K, int* err,
                                                 const int2* __restrict__ list, const int* __restrict__ count, int cap,
                                                 uint16_t* __restrict__ out, int ldo) {
    const int n = min(*count, cap);
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int K8 = K / 8;
    for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += nwarps) {
        const int2 e = list[i];
        if (!lmoe_check((unsigned)e.x < (unsigned)a_rows && (unsigned)e.y < (unsigned)w_rows, err)) continue;
        const uint4* xr = reinterpret_cast<const uint4*>(A + (size_t)e.x * K);
        const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)e.y * K);
        float hi, lo;
        dot_pairs([&](int k) { return __ldg(xr + k); }, wr, K8, lane, hi, lo);
        warp_reduce_pair(hi, lo);
        if (lane == 0) {
            uint16_t r;
            if (kRelu2) {
                const double h = (double)hi + (double)lo;  // exact: 48 significant bits at most
                r = h > 0.0 ? bf16_rn_from_double(h * h) : (uint16_t)0;
            } else {
                r = bf16_rn_of_pair(hi, lo);
            }
            out[(size_t)e.x * ldo + (e.y % ldo)] = r;
        }
    }
}

int grid_for(long long warps_of_work, int cap_blocks) {
    long long g = (warps_of_work + 7) / 8;  // 8 warps per 256-thread block
    if (g < 1) g = 1;
    return (int)(g < cap_blocks ? g : cap_blocks);
}

}  // namespace

cudaError_t launch_z_round_flag(const float* z32, uint16_t* z, int rows, int L, float m0, float m1, int2* list, int cap,
                                int* count, int4* rowtab, int* nrowtab, int sms, cudaStream_t s) {
    const long long items = (long long)rows * ((L + kSegCols - 1) / kSegCols);
    k_round_flag<<<grid_for(items, sms * 8), 256, 0, s>>>(z32, z, rows, L, m0, m1, list, cap, count, rowtab, nrowtab);
    return cudaGetLastError();
}

cudaError_t launch_recheck_rows(const uint16_t* A, int a_rows, const uint16_t* W, int w_rows, int K, int* err,
                                const int2* list, int cap, const int4* rowtab, const int* nrowtab, uint16_t* out,
                                int ldo, int sms, cudaStream_t s) {
    const size_t smem = (size_t)K * 2;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_recheck_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    // rows (segments) below four CTAs per SM: split each segment's entries over up to 8 CTAs
    const long long segs = (long long)a_rows * ((w_rows + kSegCols - 1) / kSegCols);
    const int split = (int)std::max<long long>(1, std::min<long long>(8, (long long)sms * 4 / std::max(segs, 1LL)));
    k_recheck_rows<<<sms * 4, 256, smem, s>>>(A, a_rows, W, w_rows, K, err, list, cap, rowtab, nrowtab, out, ldo,
                                              split);
    return cudaGetLastError();
}

cudaError_t launch_recheck(bool relu2, const uint16_t* A, int a_rows, const uint16_t* W, int w_rows, int K, int* err,
                           const int2* list, const int* count, int cap, uint16_t* out, int ldo, int sms, cudaStream_t s) {
    if (relu2) k_recheck<true><<<sms * 8, 256, 0, s>>>(A, a_rows, W, w_rows, K, err, list, count, cap, out, ldo);
    else k_recheck<false><<<sms * 8, 256, 0, s>>>(A, a_rows, W, w_rows, K, err, list, count, cap, out, ldo);
    return cudaGetLastError();
}

}  // namespace lmoe
