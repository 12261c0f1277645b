// router.cu -- routing kernels of the LatentMoE layer.
//
// Router ("Nemotron 3 Ultra 架构 QA", Q5.2/Q5.3; "Nemotron-3-Labs-Ultra-Math-SFT"
// article, section 路由与共享专家): sigma = sigmoid(logits), choice = sigma +
// e_score_correction_bias (selection only), grouped top-k with the 1e-6 tie
// band in ascending id, weights = scale * sigma / sum(sigma of the selected).
//
// Two precisions of the same decision:
//  * k_select<float, true, .>: from fp32 tensor-core logits. The band rule only
//    departs from the plain top-k by value when the k-th and (k+1)-th
//    eligible choice scores are within 1e-6 (or the Gk-th and (Gk+1)-th group
//    scores are); the token is flagged when either gap is within a margin
//    `delta` of 1e-6, and flagged tokens are appended to a list.
//  * k_logits64 + k_select<double, false, .>: exact-product fp64 logits and the
//    decision in fp64, for the flagged tokens (or for all tokens when x is fp32
//    or in the fp32 validation mode).
// If every fp32 choice score is within delta/2 of its fp64 value, an
// unflagged token's expert gap exceeds 1e-6 in fp64 too, so both precisions
// select the top-k by value, and that set is the same in both because the gap
// exceeds the perturbation; group scores (sums of two) move by at most delta,
// which the 2*delta group margin covers.
#include <float.h>
#include <math.h>

#include "handle.h"
#include "lmoe_internal.h"

namespace lmoe {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float sigmoid_t(float v) { return 1.0f / (1.0f + expf(-v)); }
__device__ __forceinline__ double sigmoid_t(double v) { return 1.0 / (1.0 + exp(-v)); }

__device__ __forceinline__ unsigned first_n_bits(unsigned m, int n) {
    unsigned r = 0;
    for (int i = 0; i < n && m; ++i) {
        unsigned low = m & (0u - m);
        r |= low;
        m ^= low;
    }
    return r;
}

// Order-preserving integer keys of choice scores: key(a) > key(b) whenever
// a > b (-0 sorts just below +0), and every finite score has a key above 0,
// which marks an ineligible expert.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ unsigned long long order_key(double v) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(v);
    return (u >> 63) ? ~u : (u | (1ull << 63));
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ double key_value(unsigned long long k) {
    return __longlong_as_double((long long)((k >> 63) ? (k & ~(1ull << 63)) : ~k));
}

// tau = the k-th largest eligible choice score and next = the (k+1)-th (-inf
// when fewer than k+1 are eligible), equal scores counted once each, as k
// rounds of taking the largest would. Bisection on the keys: bit b of tau's key
// (from the top) is set when at least k eligible keys are >= the prefix with
// that bit set; one compare per element and one warp sum per bit. Lane l holds
// the keys of experts l + 32 i, i < kNI (bit i of elig: eligible).
template <typename F, int kNI>
__device__ __forceinline__ void kth_and_next(const F* c, unsigned elig, int nI, int k, F& tau, F& next) {
    using U = decltype(order_key(F(0)));
    const int lane = threadIdx.x & 31;
    U key[kNI];
#pragma unroll
    for (int i = 0; i < kNI; ++i) key[i] = (i < nI && ((elig >> i) & 1u)) ? order_key(c[lane + (i << 5)]) : (U)0;
    U res = 0;
    for (int b = 8 * (int)sizeof(U) - 1; b >= 0; --b) {
        const U cand = res | ((U)1 << b);
        int cnt = 0;
#pragma unroll
        for (int i = 0; i < kNI; ++i) cnt += key[i] >= cand ? 1 : 0;
        if (__reduce_add_sync(0xFFFFFFFFu, cnt) >= k) res = cand;
    }
    int at_or_above = 0;
    U below = 0;
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
        at_or_above += key[i] >= res ? 1 : 0;
        if (key[i] < res && key[i] > below) below = key[i];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const U o = __shfl_xor_sync(0xFFFFFFFFu, below, off);
        below = o > below ? o : below;
    }
    tau = key_value(res);
    if (__reduce_add_sync(0xFFFFFFFFu, at_or_above) > k) next = tau;
    else next = below == 0 ? -(F)INFINITY : key_value(below);
}

// Warp-cooperative grouped top-k for one token.// Warp-cooperative grouped top-k for one token. c[] and sig[] (length E) live
// in this warp's shared memory. Writes idx (ascending) and weights; returns
// true when the token must be re-decided in fp64 (kFlag only).
template <typename F, bool kFlag, int kNI>
__device__ bool warp_select(const F* c, const F* sig, int E, int G, int Gk, int k, float scale, F delta,
                            int32_t* idx_out, float* w_out) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    const F eps = (F)kBandEps;
    const F ninf = -(F)INFINITY;
    bool flag = false;
    unsigned keep = 0xFFFFFFFFu;
    const int per = E / G;
    if (G > 1) {
        F gs = ninf;
        if (per % 32 == 0) {
            // group g = i / m for every lane (m = per / 32): lane-local top-2, then warp top-2
            const int m = per >> 5;
            for (int g = 0; g < G; ++g) {
                F a = ninf, b = ninf;
                for (int i = g * m; i < (g + 1) * m; ++i) {
                    const F v = c[lane + (i << 5)];
                    if (v > a) {
                        b = a;
                        a = v;
                    } else if (v > b) {
                        b = v;
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const F oa = __shfl_xor_sync(0xFFFFFFFFu, a, off), ob = __shfl_xor_sync(0xFFFFFFFFu, b, off);
                    const F na = fmax(a, oa);
                    b = a >= oa ? fmax(b, oa) : fmax(a, ob);
                    a = na;
                }
                if (lane == g) gs = a + b;
            }
        } else if (32 % per == 0) {
            // each row of 32 lanes holds 32 / per whole groups, `per` consecutive lanes each
            const int gpr = 32 / per;
            for (int i = 0; i < ((E + 31) >> 5); ++i) {
                const int e = lane + (i << 5);
                F a = e < E ? c[e] : ninf, b = ninf;
                for (int off = per >> 1; off > 0; off >>= 1) {
                    const F oa = __shfl_xor_sync(0xFFFFFFFFu, a, off), ob = __shfl_xor_sync(0xFFFFFFFFu, b, off);
                    const F na = fmax(a, oa);
                    b = a >= oa ? fmax(b, oa) : fmax(a, ob);
                    a = na;
                }
                const F sum = __shfl_sync(0xFFFFFFFFu, a + b, (lane % gpr) * per);
                if (lane < G && lane / gpr == i) gs = sum;
            }
        } else if (lane < G) {
            F a = ninf, b = ninf;
            for (int e = lane * per; e < (lane + 1) * per; ++e) {
                F v = c[e];
                if (v > a) {
                    b = a;
                    a = v;
                } else if (v > b) {
                    b = v;
                }
            }
            gs = a + b;
        }
        int rank = 0;
        for (int g = 0; g < G; ++g) {
            F o = __shfl_sync(0xFFFFFFFFu, gs, g);
            if (o > gs || (o == gs && g < lane)) ++rank;
        }
        unsigned kth = __ballot_sync(0xFFFFFFFFu, lane < G && rank == Gk - 1);
        F tau = __shfl_sync(0xFFFFFFFFu, gs, __ffs(kth) - 1);
        bool inA = lane < G && gs > tau + eps;
        bool inB = lane < G && !inA && fabs(gs - tau) <= eps;
        unsigned mA = __ballot_sync(0xFFFFFFFFu, inA);
        unsigned mB = __ballot_sync(0xFFFFFFFFu, inB);
        keep = mA | first_n_bits(mB, Gk - __popc(mA));
        if (kFlag && Gk < G) {
            unsigned nxt = __ballot_sync(0xFFFFFFFFu, lane < G && rank == Gk);
            F below = __shfl_sync(0xFFFFFFFFu, gs, __ffs(nxt) - 1);
            flag |= (tau - below) <= eps + 2 * delta;
        }
    }
    // eligibility of this lane's experts e = lane + 32 i, one bit per i
    const int nI = (E + 31) >> 5;
    unsigned elig = 0;
    for (int i = 0; i < nI; ++i) {
        const int e = lane + (i << 5);
        if (e < E && ((keep >> (e / per)) & 1u)) elig |= 1u << i;
    }
    // tau = k-th largest eligible choice score, next = the (k+1)-th
    F tau, next;
    kth_and_next<F, kNI>(c, elig, nI, k, tau, next);
    if (kFlag) flag |= (tau - next) <= eps + delta;
    // A = {c > tau + eps}; the band |c - tau| <= eps fills the rest in ascending id.
    int nA = 0;
    for (int i = 0; i < nI; ++i) {
        const int e = lane + (i << 5);
        bool inA = ((elig >> i) & 1u) && c[e] > tau + eps;
        nA += __popc(__ballot_sync(0xFFFFFFFFu, inA));
    }
    const int need = k - nA;
    int nout = 0, nband = 0;
    for (int i = 0; i < nI; ++i) {
        const int e = lane + (i << 5);
        const bool el = (elig >> i) & 1u;
        F v = el ? c[e] : (F)0;
        bool inA = el && v > tau + eps;
        bool inB = el && !inA && fabs(v - tau) <= eps;
        unsigned mB = __ballot_sync(0xFFFFFFFFu, inB);
        bool take = inA || (inB && nband + __popc(mB & lt) < need);
        unsigned mT = __ballot_sync(0xFFFFFFFFu, take);
        if (take) idx_out[nout + __popc(mT & lt)] = e;
        nout += __popc(mT);
        nband += __popc(mB);
    }
    __syncwarp();
    // weights: scale * sigma_e / sum over the selected (fixed-order tree sum)
    F part = 0;
    for (int j = lane; j < k; j += 32) part += sig[idx_out[j]];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
    for (int j = lane; j < k; j += 32) w_out[j] = (float)((F)scale * sig[idx_out[j]] / part);
    return flag;
}

template <typename F, bool kFlag, int kNI>
__global__ void __launch_bounds__(kWarps * 32)
    k_select(const F* __restrict__ logits, const float* __restrict__ bias, int T, int E, int G, int Gk, int k,
             float scale, float delta, const int* __restrict__ list, const int* __restrict__ list_count,
             int32_t* __restrict__ idx, float* __restrict__ wgt, int* __restrict__ flaglist,
             int* __restrict__ flag_count, int* err) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    F* c = reinterpret_cast<F*>(smem_raw) + (size_t)warp * 2 * E;
    F* sig = c + E;
    const int n = list_count ? *list_count : T;
    for (int item = blockIdx.x * kWarps + warp; item < n; item += gridDim.x * kWarps) {
        const int t = list ? list[item] : item;
        if (!lmoe_check((unsigned)t < (unsigned)T, err)) continue;
        const F* lg = logits + (size_t)t * E;
        for (int e = lane; e < E; e += 32) {
            F s = sigmoid_t(lg[e]);
            sig[e] = s;
            c[e] = s + (F)bias[e];
        }
        __syncwarp();
        bool flag = warp_select<F, kFlag, kNI>(c, sig, E, G, Gk, k, scale, (F)delta, idx + (size_t)t * k,
                                               wgt + (size_t)t * k);
        if (kFlag && flag && lane == 0) {
            int pos = atomicAdd(flag_count, 1);
            flaglist[pos] = t;
        }
        __syncwarp();
    }
}

// fp64 logits: out[t, e] = sum_h x[t, h] * W_r[e, h]; the bf16 x bf16 (or
// fp32 x bf16) products are exact in fp64. One work item = one token and a
// chunk of 16 experts (each warp two of them, their rows streamed together);
// a block takes a contiguous run of items, so the items of one token follow
// each other and its row, staged in shared memory as fp64 and read as 16-byte
// vectors (conflict-free, each lane covering 8 consecutive h), is reused. Small
// chunks keep a few flagged tokens spread over many SMs.
constexpr int kERows = 2;                  // experts per warp and pass
constexpr int kEChunk = 8 * kERows;        // experts per work item (8 warps)
template <bool kXf32>
__global__ void __launch_bounds__(256)
    k_logits64(const void* __restrict__ x, const uint16_t* __restrict__ wr, int T, int E, int H,
               const int* __restrict__ list, const int* __restrict__ list_count, double* __restrict__ out, int* err) {
    extern __shared__ __align__(16) double xrow[];
    const int n = list_count ? *list_count : T;
    const int chunks = (E + kEChunk - 1) / kEChunk;
    const long long items = (long long)n * chunks;
    const long long per = (items + gridDim.x - 1) / gridDim.x;
    const long long i0 = (long long)blockIdx.x * per, i1 = min(items, i0 + per);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int cur = -1;
    for (long long item = i0; item < i1; ++item) {
        const int li = (int)(item / chunks), ch = (int)(item % chunks);
        const int t = list ? list[li] : li;
        if (!lmoe_check((unsigned)t < (unsigned)T, err)) continue;  // uniform over the block: no barrier skipped unevenly
        if (t != cur) {
            __syncthreads();
            for (int h = threadIdx.x; h < H; h += blockDim.x) {
                float v;
                if (kXf32) {
                    v = static_cast<const float*>(x)[(size_t)t * H + h];
                } else {
                    v = __uint_as_float((uint32_t) static_cast<const uint16_t*>(x)[(size_t)t * H + h] << 16);
                }
                xrow[h] = (double)v;
            }
            __syncthreads();
            cur = t;
        }
        const int e0 = ch * kEChunk + warp * kERows;
        if (e0 >= E) continue;
        const uint16_t* wrow[kERows];
#pragma unroll
        for (int j = 0; j < kERows; ++j) wrow[j] = wr + (size_t)min(e0 + j, E - 1) * H;
        double acc[kERows][2];
#pragma unroll
        for (int j = 0; j < kERows; ++j) acc[j][0] = acc[j][1] = 0.0;
        for (int h = lane * 8; h < H; h += 256) {
            uint4 pk[kERows];
#pragma unroll
            for (int j = 0; j < kERows; ++j) pk[j] = __ldg(reinterpret_cast<const uint4*>(wrow[j] + h));
            const double2* xv = reinterpret_cast<const double2*>(xrow + h);
            double2 xx[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) xx[q] = xv[q];
#pragma unroll
            for (int j = 0; j < kERows; ++j) {
                const uint32_t u[4] = {pk[j].x, pk[j].y, pk[j].z, pk[j].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[j][q & 1] = fma(xx[q].x, (double)__uint_as_float(u[q] << 16), acc[j][q & 1]);
                    acc[j][q & 1] = fma(xx[q].y, (double)__uint_as_float(u[q] & 0xFFFF0000u), acc[j][q & 1]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kERows; ++j) {
            double a = acc[j][0] + acc[j][1];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, off);
            if (lane == 0 && e0 + j < E) out[(size_t)t * E + e0 + j] = a;
        }
    }
}

}  // namespace

cudaError_t launch_router_select(const lmoe_handle* h, const Plan& p, char* ws, bool, cudaStream_t s) {
    const lmoe_config& c = h->cfg;
    int E = c.num_experts;
    int blocks = (p.T + kWarps - 1) / kWarps;
    if (blocks > 4 * h->num_sms) blocks = 4 * h->num_sms;
    size_t smem = (size_t)kWarps * 2 * E * sizeof(float);
    WsStats* st = reinterpret_cast<WsStats*>(ws + p.stats);
    // keys per lane: E / 32 rounded up to 16 or 32 (E <= kMaxE = 1024)
    auto kern = E <= 512 ? k_select<float, true, 16> : k_select<float, true, 32>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<blocks, kWarps * 32, smem, s>>>(
        reinterpret_cast<const float*>(ws + p.logits), h->w.e_bias, p.T, E, c.n_group, c.topk_group, c.top_k,
        c.routed_scaling_factor, h->flag_delta, nullptr, nullptr, reinterpret_cast<int32_t*>(ws + p.idx),
        reinterpret_cast<float*>(ws + p.wgt), reinterpret_cast<int*>(ws + p.flaglist), &st->flagged, &st->device_error);
    return cudaGetLastError();
}

cudaError_t launch_router_logits64(const lmoe_handle* h, const void* x, const Plan& p, char* ws, bool all,
                                   cudaStream_t s) {
    const lmoe_config& c = h->cfg;
    WsStats* st = reinterpret_cast<WsStats*>(ws + p.stats);
    const int* list = all ? nullptr : reinterpret_cast<const int*>(ws + p.flaglist);
    const int* cnt = all ? nullptr : &st->flagged;
    size_t smem = (size_t)c.hidden * sizeof(double);
    int blocks = 2 * h->num_sms;
    double* out = reinterpret_cast<double*>(ws + p.logits64);
    if (smem > 48 * 1024) {
        cudaError_t e = c.x_dtype == LMOE_FP32
                            ? cudaFuncSetAttribute(k_logits64<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem)
                            : cudaFuncSetAttribute(k_logits64<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem);
        if (e != cudaSuccess) return e;
    }
    if (c.x_dtype == LMOE_FP32)
        k_logits64<true><<<blocks, 256, smem, s>>>(x, static_cast<const uint16_t*>(h->w.router_w), p.T,
                                                   c.num_experts, c.hidden, list, cnt, out, &st->device_error);
    else
        k_logits64<false><<<blocks, 256, smem, s>>>(x, static_cast<const uint16_t*>(h->w.router_w), p.T,
                                                    c.num_experts, c.hidden, list, cnt, out, &st->device_error);
    return cudaGetLastError();
}

cudaError_t launch_router_select64(const lmoe_handle* h, const Plan& p, char* ws, bool all, cudaStream_t s) {
    const lmoe_config& c = h->cfg;
    WsStats* st = reinterpret_cast<WsStats*>(ws + p.stats);
    int E = c.num_experts;
    size_t smem = (size_t)kWarps * 2 * E * sizeof(double);
    auto kern = E <= 512 ? k_select<double, false, 16> : k_select<double, false, 32>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    int blocks = all ? (p.T + kWarps - 1) / kWarps : h->num_sms;
    if (blocks > 4 * h->num_sms) blocks = 4 * h->num_sms;
    if (blocks < 1) blocks = 1;
    kern<<<blocks, kWarps * 32, smem, s>>>(
        reinterpret_cast<const double*>(ws + p.logits64), h->w.e_bias, p.T, E, c.n_group, c.topk_group, c.top_k,
        c.routed_scaling_factor, 0.f, all ? nullptr : reinterpret_cast<const int*>(ws + p.flaglist),
        all ? nullptr : &st->flagged, reinterpret_cast<int32_t*>(ws + p.idx), reinterpret_cast<float*>(ws + p.wgt),
        nullptr, nullptr, &st->device_error);
    return cudaGetLastError();
}

}  // namespace lmoe
