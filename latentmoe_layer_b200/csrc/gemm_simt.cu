// gemm_simt.cu -- fp32 CUDA-core GEMMs of the fp32 validation mode.
//
// Same problem descriptors as the tensor-core engine (dense, grouped by
// expert, two concatenated K segments) and the same epilogues, computed with
// fp32 FMAs from fp32 (or bf16) activations and bf16 weights. This mode exists
// to check the layer's plumbing at 1e-5 relative error; it is not timed.
#include <cuda_bf16.h>

#include "lmoe_internal.h"
#include "ptx.cuh"

namespace lmoe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <bool kAf32>
__device__ __forceinline__ void load4(const void* base, long long off, float (&v)[4]) {
    if (kAf32) {
        float4 q = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
        v[0] = q.x, v[1] = q.y, v[2] = q.z, v[3] = q.w;
    } else {
        uint2 q = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + off);
        v[0] = __uint_as_float(q.x << 16), v[1] = __uint_as_float(q.x & 0xFFFF0000u);
        v[2] = __uint_as_float(q.y << 16), v[3] = __uint_as_float(q.y & 0xFFFF0000u);
    }
}

template <bool kAf32>
__global__ void __launch_bounds__(256) k_gemm_simt(const GemmProblem pr, const DeviceRouting r) {
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    int row0, rows, wrow0;
    const int col0 = blockIdx.y * TN;
    if (pr.grouped) {
        const int mt = blockIdx.x;
        if (mt >= r.pfx64[r.E]) return;
        int lo = 0, hi = r.E;
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (r.pfx64[mid] <= mt) lo = mid;
            else hi = mid;
        }
        row0 = r.offsets[lo] + (mt - r.pfx64[lo]) * TM;
        rows = min(TM, r.offsets[lo + 1] - row0);
        wrow0 = (pr.expert_mod ? lo % pr.expert_mod : lo) * pr.b_rows_per_expert + col0;
    } else {
        row0 = blockIdx.x * TM;
        rows = min(TM, pr.m_rows - row0);
        wrow0 = col0;
    }
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int lr = tid / 4, lk = (tid % 4) * 4;
    float acc[4][4] = {};
    for (int sg = 0; sg < pr.nseg; ++sg) {
        const int K = pr.kdim[sg];
        for (int k0 = 0; k0 < K; k0 += TK) {
            float av[4] = {0.f, 0.f, 0.f, 0.f}, bv[4];
            if (lr < rows) load4<kAf32>(pr.a_ptr[sg], (long long)(row0 + lr) * K + k0 + lk, av);
            load4<false>(pr.b_ptr[sg], (long long)(wrow0 + lr) * K + k0 + lk, bv);
            __syncthreads();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                As[lk + q][lr] = av[q];
                Bs[lk + q][lr] = bv[q];
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < TK; ++kk) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rr = ty * 4 + i;
        if (rr >= rows) continue;
        const long long row = row0 + rr;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float v = acc[i][j];
            if (pr.epi == EPI_RELU2_BF16 || pr.epi == EPI_RELU2_F32) {
                v = fmaxf(v, 0.f);
                v = v * v;
                // exact re-rounding list (bf16 mode): large activations near a rounding midpoint
                if (pr.epi == EPI_RELU2_BF16 && pr.rr_list && rr_flag(v, pr.rr_tau2_bits, pr.rr_ulps))
                    rr_append(pr, (int)row, wrow0 + tx * 4 + j);
            }
            if (pr.epi == EPI_SCALE_F32) v *= pr.row_scale[row];
            const long long o = row * pr.ldo + col0 + tx * 4 + j;
            if (pr.resid) v += __uint_as_float((uint32_t)pr.resid[o] << 16);
            if (pr.epi == EPI_BF16 || pr.epi == EPI_RELU2_BF16)
                static_cast<__nv_bfloat16*>(pr.out)[o] = __float2bfloat16_rn(v);
            else
                static_cast<float*>(pr.out)[o] = v;
        }
    }
}

}  // namespace

// Grouped problems launch enough row tiles for the worst case (every expert
// ragged: sum ceil(n_e / 64) <= max_rows / 64 + E); surplus blocks exit.
cudaError_t launch_gemm_simt(const GemmProblem* probs, int nprob, bool a_f32, const DeviceRouting& r, int max_rows,
                             cudaStream_t s) {
    for (int i = 0; i < nprob; ++i) {
        const GemmProblem& pr = probs[i];
        const int mt = pr.grouped ? (max_rows + TM - 1) / TM + r.E : (pr.m_rows + TM - 1) / TM;
        if (mt <= 0) continue;
        dim3 grid(mt, pr.n / TN);
        if (a_f32) k_gemm_simt<true><<<grid, 256, 0, s>>>(pr, r);
        else k_gemm_simt<false><<<grid, 256, 0, s>>>(pr, r);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lmoe
