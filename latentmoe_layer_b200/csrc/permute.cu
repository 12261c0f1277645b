// permute.cu -- token permutation, row gather, weighted combine and small
// conversion kernels of the LatentMoE layer.
//
// The permutation is a deterministic counting sort of the (token, expert)
// assignments by expert, stable in token id: permuted row
//   offsets[e] + (number of earlier tokens routed to e)
// holds token t's copy for expert e. It replaces the per-expert Python loop
// over `expert_hit` with index_add_ ("Nemotron 3 Ultra 架构 QA", Q5.1, Q5.6):
// expert e's rows are contiguous, so each expert's FFN is one GEMM over them,
// and the combine sums each token's k rows in ascending expert id.
#include <cuda_bf16.h>

#include "handle.h"
#include "lmoe_internal.h"
#include "ptx.cuh"

namespace lmoe {
namespace {

constexpr int kChunk = 256;  // tokens per counting block

__global__ void k_count(const int32_t* __restrict__ idx, int T, int k, int E, int* __restrict__ blockcounts,
                        int* err) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kChunk, t1 = min(T, t0 + kChunk);
    for (int i = t0 * k + threadIdx.x; i < t1 * k; i += blockDim.x)
        if (lmoe_check((unsigned)idx[i] < (unsigned)E, err)) atomicAdd(&hist[idx[i]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blockcounts[(size_t)blockIdx.x * E + e] = hist[e];
}

// Inclusive block scan of 4 integer lanes at once (blockDim.x == 1024).
__device__ void block_scan4(int4& v, int4* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int4 o;
        o.x = __shfl_up_sync(0xFFFFFFFFu, v.x, off);
        o.y = __shfl_up_sync(0xFFFFFFFFu, v.y, off);
        o.z = __shfl_up_sync(0xFFFFFFFFu, v.z, off);
        o.w = __shfl_up_sync(0xFFFFFFFFu, v.w, off);
        if (lane >= off) {
            v.x += o.x;
            v.y += o.y;
            v.z += o.z;
            v.w += o.w;
        }
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int4 t = warp_tot[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int4 o;
            o.x = __shfl_up_sync(0xFFFFFFFFu, t.x, off);
            o.y = __shfl_up_sync(0xFFFFFFFFu, t.y, off);
            o.z = __shfl_up_sync(0xFFFFFFFFu, t.z, off);
            o.w = __shfl_up_sync(0xFFFFFFFFu, t.w, off);
            if (lane >= off) {
                t.x += o.x;
                t.y += o.y;
                t.z += o.z;
                t.w += o.w;
            }
        }
        warp_tot[lane] = t;
    }
    __syncthreads();
    if (warp > 0) {
        int4 p = warp_tot[warp - 1];
        v.x += p.x;
        v.y += p.y;
        v.z += p.z;
        v.w += p.w;
    }
}

__global__ void __launch_bounds__(1024)
    k_scan(int* __restrict__ blockcounts, int nblk, int E, int* __restrict__ counts, int32_t* __restrict__ counts_out,
           int* __restrict__ offsets, int* __restrict__ pfx128, int* __restrict__ pfx64, int* __restrict__ pfxdec,
           int* __restrict__ pfx256, int4* __restrict__ rec32, int4* __restrict__ rec64, int4* __restrict__ rec128,
           int4* __restrict__ rec256, WsStats* __restrict__ st) {
    __shared__ int4 warp_tot[32];
    __shared__ int red[2];
    const int e = threadIdx.x;
    int run = 0;
    if (e < E) {
        for (int b0 = 0; b0 < nblk; b0 += 8) {  // 8 independent loads in flight
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = b0 + j < nblk ? blockcounts[(size_t)(b0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (b0 + j < nblk) blockcounts[(size_t)(b0 + j) * E + e] = run;
                run += v[j];
            }
        }
        counts[e] = run;
        if (counts_out) counts_out[e] = run;
    }
    if (e < 2) red[e] = 0;
    __syncthreads();
    if (e < E && run > 0) {
        atomicAdd(&red[0], 1);
        atomicMax(&red[1], run);
    }
    int4 v = make_int4(run, (run + 127) / 128, (run + 63) / 64, (run + kDecodeTN - 1) / kDecodeTN);
    int4 incl = v;
    block_scan4(incl, warp_tot);
    __syncthreads();
    int4 v2 = make_int4((run + 255) / 256, 0, 0, 0);
    int4 incl2 = v2;
    block_scan4(incl2, warp_tot);
    if (e < E) {
        pfx256[e] = incl2.x - v2.x;
        if (e == E - 1) pfx256[E] = incl2.x;
    }
    if (e < E) {
        offsets[e] = incl.x - v.x;
        pfx128[e] = incl.y - v.y;
        pfx64[e] = incl.z - v.z;
        pfxdec[e] = incl.w - v.w;
        if (e == E - 1) {
            offsets[E] = incl.x;
            pfx128[E] = incl.y;
            pfx64[E] = incl.z;
            pfxdec[E] = incl.w;
        }
    }
    // tile records: the j-th R-row tile of expert e starts at row offset + j R
    if (e < E) {
        const int off = incl.x - v.x;
        int4* recs[4] = {rec32 + (incl.w - v.w), rec64 + (incl.z - v.z), rec128 + (incl.y - v.y),
                         rec256 + (incl2.x - v2.x)};
        const int rows[4] = {kDecodeTN, 64, 128, 256};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            for (int j = 0; j * rows[q] < run; ++j)
                recs[q][j] = make_int4(e, off + j * rows[q], min(rows[q], run - j * rows[q]), 0);
    }
    __syncthreads();
    if (e == 0) {
        st->distinct = red[0];
        st->max_count = red[1];
    }
}

// One block per chunk of kChunk tokens, 8 warps of 32 tokens each. The
// chunk's expert ids are staged in shared memory; each warp counts its tokens
// per expert, a prefix over the warps gives each warp its start inside every
// expert's range, then each warp walks its 32 tokens in order (the k experts
// of a token are distinct, so its lanes never share a cursor). The result is
// the order of token id within every expert, as a sequential walk would give.
constexpr int kScatterWarps = 8;
__global__ void __launch_bounds__(kScatterWarps * 32)
    k_scatter(const int32_t* __restrict__ idx, const float* __restrict__ w, int T, int k, int E,
              const int* __restrict__ blockcounts, const int* __restrict__ offsets, int* __restrict__ perm,
              int* __restrict__ slot, float* __restrict__ wperm, int* err) {
    extern __shared__ int sm[];
    int* cur = sm;                        // [kScatterWarps][E] per-warp cursors
    int* sidx = sm + kScatterWarps * E;   // [kChunk * k]
    const int t0 = blockIdx.x * kChunk, t1 = min(T, t0 + kChunk);
    const int n = (t1 - t0) * k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) cur[i] = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) sidx[i] = idx[(size_t)t0 * k + i];
    __syncthreads();
    const int w0 = warp * (kChunk / kScatterWarps);
    const int w1 = min(t1 - t0, w0 + kChunk / kScatterWarps);
    for (int i = w0 * k + lane; i < w1 * k; i += 32)
        if (lmoe_check((unsigned)sidx[i] < (unsigned)E, err)) atomicAdd(&cur[warp * E + sidx[i]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {  // exclusive prefix over the warps
        int run = offsets[e] + blockcounts[(size_t)blockIdx.x * E + e];
        for (int q = 0; q < kScatterWarps; ++q) {
            const int c = cur[q * E + e];
            cur[q * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    int* mycur = cur + warp * E;
    for (int tl = w0; tl < w1; ++tl) {
        for (int j = lane; j < k; j += 32) {
            const int e = sidx[tl * k + j];
            if (!lmoe_check((unsigned)e < (unsigned)E, err)) {
                sidx[tl * k + j] = -1;
                continue;
            }
            const int pos = mycur[e];
            mycur[e] = pos + 1;
            sidx[tl * k + j] = pos;  // slot, written out below
        }
        __syncwarp();
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int pos = sidx[i];
        const size_t g = (size_t)t0 * k + i;
        if (!lmoe_check((unsigned)pos < (unsigned)(T * k), err)) continue;
        slot[g] = pos;
        perm[pos] = t0 + i / k;
        wperm[pos] = w[g];
    }
}

// dst[r, :] = src[perm[r], :] for r < *total (row_bytes multiple of 16). One
// warp per row: the source row index is read once, and each lane keeps up to
// eight 16-byte loads in flight before its stores.
__global__ void __launch_bounds__(256) k_gather(const uint4* __restrict__ src, int src_rows, int* err,
                                                uint4* __restrict__ dst, const int* __restrict__ perm,
                                                const int* __restrict__ total, int vec_per_row) {
    const int rows = *total;
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
        const int pr = __ldg(perm + r);
        if (!lmoe_check((unsigned)pr < (unsigned)src_rows, err)) continue;
        const uint4* s = src + (long long)pr * vec_per_row;
        uint4* d = dst + (long long)r * vec_per_row;
        int c = lane;
        for (; c + 7 * 32 < vec_per_row; c += 8 * 32) {
            uint4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = ld_global_nc_v4(s + c + 32 * j);
#pragma unroll
            for (int j = 0; j < 8; ++j) st_global_cs_v4(d + c + 32 * j, v[j]);  // rows far beyond L2
        }
        for (; c < vec_per_row; c += 32) st_global_cs_v4(d + c, ld_global_nc_v4(s + c));
    }
}

// comb[t, :] = sum_{j ascending} o[slot[t, j], :]   (o already carries w)
template <bool kBf16>
__global__ void __launch_bounds__(256)
    k_combine(const float4* __restrict__ o, int o_rows, int* err, const int* __restrict__ slot, void* __restrict__ comb,
              int T, int k, int L4) {
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const int* sl = slot + (size_t)t * k;
        for (int c = threadIdx.x; c < L4; c += blockDim.x) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < k; ++j) {
                if (!lmoe_check((unsigned)sl[j] < (unsigned)o_rows, err)) continue;
                float4 v = __ldcs(&o[(size_t)sl[j] * L4 + c]);  // o is read once: evict first
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            if (kBf16) {
                uint2 pk;
                pk.x = pack_bf16x2(acc.x, acc.y);
                pk.y = pack_bf16x2(acc.z, acc.w);
                reinterpret_cast<uint2*>(comb)[(size_t)t * L4 + c] = pk;
            } else {
                reinterpret_cast<float4*>(comb)[(size_t)t * L4 + c] = acc;
            }
        }
    }
}

__global__ void k_convert(const float4* __restrict__ x, uint2* __restrict__ xb, long long n4) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        float4 v = x[i];
        xb[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
}

__global__ void k_copy_routing(const int* __restrict__ idx, const float* __restrict__ w, int32_t* __restrict__ io,
                               float* __restrict__ wo, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        if (io) io[i] = idx[i];
        if (wo) wo[i] = w[i];
    }
}

// Load-balancing bias update ("Nemotron 3 Ultra 架构 QA", Q5.3) and MaxVio (Q5.4):
// one block; integer reductions are exact, and the fp64 update is written with
// explicit round-to-nearest multiply and subtract so no fused multiply-add
// changes its rounding.
__global__ void __launch_bounds__(1024)
    k_update_bias(const int32_t* __restrict__ counts, const float* __restrict__ bias_in, int E, double eta,
                  float* __restrict__ bias_out, double* __restrict__ maxvio) {
    __shared__ long long s_tot[32];
    __shared__ int s_max[32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const int c = e < E ? counts[e] : 0;
    long long t = c;
    int m = c;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        t += __shfl_xor_sync(0xFFFFFFFFu, t, off);
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    }
    if (lane == 0) {
        s_tot[warp] = t;
        s_max[warp] = m;
    }
    __syncthreads();
    if (warp == 0) {
        t = s_tot[lane];
        m = s_max[lane];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            t += __shfl_xor_sync(0xFFFFFFFFu, t, off);
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        }
        if (lane == 0) {
            s_tot[0] = t;
            s_max[0] = m;
        }
    }
    __syncthreads();
    const double mean = (double)s_tot[0] / (double)E;
    const float b = e < E ? bias_in[e] : 0.f;  // read before any write: bias_out may alias bias_in
    __syncthreads();
    if (e < E) bias_out[e] = (float)__dsub_rn((double)b, __dmul_rn(eta, __dsub_rn((double)c, mean)));
    if (e == 0 && maxvio) *maxvio = mean > 0.0 ? __ddiv_rn(__dsub_rn((double)s_max[0], mean), mean) : 0.0;
}

// Nearest-even bf16 of a double (normal range): keep 8 significant bits.
__device__ __forceinline__ double round_bf16_f64(double v) {
    unsigned long long u = (unsigned long long)__double_as_longlong(v);
    u += 0x00000FFFFFFFFFFFull + ((u >> 45) & 1ull);
    u &= ~0x00001FFFFFFFFFFFull;
    return __longlong_as_double((long long)u);
}
__device__ __forceinline__ uint16_t bf16_bits(double v) { return (uint16_t)(__float_as_uint((float)v) >> 16); }

// Pre-norm RMSNorm of the block ("Nemotron 3 Ultra 架构 QA", Q2.8): per token,
// r = 1 / sqrt(mean(x^2) + eps) in fp64 (squares of bf16 are exact, sqrt and
// division correctly rounded), xt = bf16(x r), out = bf16(gamma xt); explicit
// round-to-nearest operations keep every rounding the same as the definition.
__global__ void __launch_bounds__(256)
    k_rmsnorm(const uint16_t* __restrict__ x, const uint16_t* __restrict__ gamma, double eps, int T, int H,
              uint16_t* __restrict__ out) {
    __shared__ double red[8];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const uint16_t* xr = x + (size_t)t * H;
        double ss = 0.0;
        for (int h = threadIdx.x; h < H; h += blockDim.x) {
            const double v = (double)__uint_as_float((uint32_t)xr[h] << 16);
            ss = __dadd_rn(ss, __dmul_rn(v, v));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, off));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
        __syncthreads();
        double tot = 0.0;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot = __dadd_rn(tot, red[i]);
        __syncthreads();
        const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(tot, (double)H), eps)));
        for (int h = threadIdx.x; h < H; h += blockDim.x) {
            const double v = (double)__uint_as_float((uint32_t)xr[h] << 16);
            const double xt = round_bf16_f64(__dmul_rn(v, r));
            const double g = (double)__uint_as_float((uint32_t)gamma[h] << 16);
            out[(size_t)t * H + h] = bf16_bits(round_bf16_f64(__dmul_rn(g, xt)));
        }
    }
}

inline int grid_cap(long long work, int per_block, int cap) {
    long long g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    return (int)(g < cap ? g : cap);
}

}  // namespace

cudaError_t launch_permute(const lmoe_handle* h, const Plan& p, char* ws, int32_t* counts_out, cudaStream_t s) {
    const int E = h->cfg.num_experts, k = h->cfg.top_k;
    int* bc = reinterpret_cast<int*>(ws + p.blockcounts);
    const int32_t* idx = reinterpret_cast<const int32_t*>(ws + p.idx);
    int* err = &reinterpret_cast<WsStats*>(ws + p.stats)->device_error;
    k_count<<<p.nblk, 256, E * sizeof(int), s>>>(idx, p.T, k, E, bc, err);
    k_scan<<<1, 1024, 0, s>>>(bc, p.nblk, E, reinterpret_cast<int*>(ws + p.counts), counts_out,
                              reinterpret_cast<int*>(ws + p.offsets), reinterpret_cast<int*>(ws + p.pfx128),
                              reinterpret_cast<int*>(ws + p.pfx64), reinterpret_cast<int*>(ws + p.pfxdec),
                              reinterpret_cast<int*>(ws + p.pfx256), reinterpret_cast<int4*>(ws + p.rec32),
                              reinterpret_cast<int4*>(ws + p.rec64), reinterpret_cast<int4*>(ws + p.rec128),
                              reinterpret_cast<int4*>(ws + p.rec256), reinterpret_cast<WsStats*>(ws + p.stats));
    const size_t scatter_smem = (size_t)(kScatterWarps * E + kChunk * k) * sizeof(int);
    if (scatter_smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scatter_smem);
        if (e != cudaSuccess) return e;
    }
    k_scatter<<<p.nblk, 256, scatter_smem, s>>>(idx, reinterpret_cast<const float*>(ws + p.wgt), p.T, k, E, bc,
                                                   reinterpret_cast<const int*>(ws + p.offsets),
                                                   reinterpret_cast<int*>(ws + p.perm),
                                                   reinterpret_cast<int*>(ws + p.slot),
                                                   reinterpret_cast<float*>(ws + p.wperm), err);
    return cudaGetLastError();
}

// Rows received for expert parallelism: blockcounts holds the count of each
// (source rank, local expert) block (one "block row" of the scan); the scan
// gives its offsets, tile prefixes and tile records. If the counts do not add
// up to n_rows the tile prefixes are zeroed (no GEMM tile runs) and
// LMOE_ERR_INVALID_ARG is recorded.
__global__ void k_check_rows(const int* __restrict__ offsets, int nb, int n_rows, int* pfx128, int* pfx64, int* pfxdec,
                             int* pfx256, WsStats* st) {
    if (threadIdx.x == 0 && offsets[nb] != n_rows) {
        pfx128[nb] = pfx64[nb] = pfxdec[nb] = pfx256[nb] = 0;
        atomicCAS(&st->device_error, 0, (int)LMOE_ERR_INVALID_ARG);
    }
}

cudaError_t launch_group_scan(int* blockcounts, int nb, int n_rows, int* counts, int* offsets, int* pfx128, int* pfx64,
                              int* pfxdec, int* pfx256, int4* rec32, int4* rec64, int4* rec128, int4* rec256,
                              WsStats* st, cudaStream_t s) {
    k_scan<<<1, 1024, 0, s>>>(blockcounts, 1, nb, counts, nullptr, offsets, pfx128, pfx64, pfxdec, pfx256, rec32, rec64,
                              rec128, rec256, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_check_rows<<<1, 32, 0, s>>>(offsets, nb, n_rows, pfx128, pfx64, pfxdec, pfx256, st);
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, int src_rows, int* err, void* dst, const int* perm, int rows_total_max,
                               const int* total, int row_bytes, int sms, cudaStream_t s) {
    const int vpr = row_bytes / 16;
    int grid = grid_cap((long long)rows_total_max * 32, 256, sms * 8);  // one warp per row
    k_gather<<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), src_rows, err, static_cast<uint4*>(dst), perm, total,
                                  vpr);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float* o, int o_rows, int* err, const int* slot, void* comb, int T, int k, int L,
                           bool out_bf16, int sms, cudaStream_t s) {
    int grid = T < sms * 8 ? T : sms * 8;
    if (out_bf16)
        k_combine<true><<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(o), o_rows, err, slot, comb, T, k, L / 4);
    else
        k_combine<false><<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(o), o_rows, err, slot, comb, T, k, L / 4);
    return cudaGetLastError();
}

cudaError_t launch_convert_x(const float* x, uint16_t* xb, long long n, int sms, cudaStream_t s) {
    long long n4 = n / 4;
    k_convert<<<grid_cap(n4, 256, sms * 16), 256, 0, s>>>(reinterpret_cast<const float4*>(x),
                                                          reinterpret_cast<uint2*>(xb), n4);
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const uint16_t* x, const uint16_t* gamma, double eps, int T, int H, uint16_t* out, int sms,
                           cudaStream_t s) {
    k_rmsnorm<<<T < sms * 8 ? T : sms * 8, 256, 0, s>>>(x, gamma, eps, T, H, out);
    return cudaGetLastError();
}

cudaError_t launch_update_bias(const int32_t* counts, const float* bias_in, int E, double eta, float* bias_out,
                               double* maxvio, cudaStream_t s) {
    k_update_bias<<<1, 1024, 0, s>>>(counts, bias_in, E, eta, bias_out, maxvio);
    return cudaGetLastError();
}

cudaError_t launch_copy_routing(const int* idx, const float* w, int32_t* idx_out, float* w_out, long long n, int sms,
                                cudaStream_t s) {
    if (!idx_out && !w_out) return cudaSuccess;
    k_copy_routing<<<grid_cap(n, 256, sms * 8), 256, 0, s>>>(idx, w, idx_out, w_out, n);
    return cudaGetLastError();
}

}  // namespace lmoe
