// gemm_common.cuh -- pieces shared by the tcgen05 GEMM kernels (bf16 weights
// in gemm_tc.cu, NVFP4 weights in gemm_nvfp4.cu): launch parameters, tile
// shapes, the tile walk over dense and expert-grouped problems, and the
// epilogue that turns fp32 accumulators into the layer's outputs.
#pragma once
#include <cuda_bf16.h>
#include <string.h>

#include "lmoe_internal.h"
#include "ptx.cuh"

#ifndef LMOE_CHUNK_KB
#define LMOE_CHUNK_KB 8   // k-blocks (of 64) per TMEM accumulation chunk
#endif
#ifndef LMOE_PROMOTE_F64
#define LMOE_PROMOTE_F64 0  // 1: chunk partials are added into fp64 registers
#endif
#ifndef LMOE_MAX_BN
#define LMOE_MAX_BN 256
#endif


namespace lmoe {
namespace {

constexpr int kMaxMaps = kMaxTensorMaps;
constexpr int kMaxProb = kMaxProblems;
constexpr int kGroupM = 16;

struct alignas(64) TcParams {
    CUtensorMap maps[kMaxMaps];
    GemmProblem prob[kMaxProb];
    int nprob;
    int nmaps;
    int dense_tiles[kMaxProb];
    DeviceRouting r;
    int* err;
    unsigned spin;
};

struct TileInfo {
    int p;       // problem
    int row0;    // first activation row (permuted row for grouped problems)
    int rows;    // valid activation rows in this tile
    int wrow0;   // first weight row this CTA loads (row of B)
    int wcol0;   // weight row of the tile's first output column (differs from wrow0 in the second
                 // CTA of a 2-SM pair, which loads the upper half of the pair's B rows)
    int col0;    // first output column
    int e;       // expert of a grouped tile (-1 for dense problems)
    bool half;   // non-swapped tile with <= 64 valid rows: M = 64 MMAs (the expert's ragged tail)
};

// Appends the elements this thread marked in mask (bit i of word w = its
// accumulator column c0 + 32 w + i), n of them, to the problem's re-rounding
// list with one atomic per warp: an inclusive scan of the lanes' counts gives
// each lane its run of entries. Called by all 32 lanes of the warp.
template <int kW>
__device__ __forceinline__ void rr_append_warp(const GemmProblem& pr, int n, const uint32_t (&mask)[kW],
                                               const TileInfo& ti, int lane_row, int c0, bool swap) {
    const int lane = threadIdx.x & 31;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    int base = 0;
    if (lane == 31) base = atomicAdd(pr.rr_count, total);
    int pos = __shfl_sync(0xFFFFFFFFu, base, 31) + incl - n;
    for (int w = 0; w < kW; ++w) {
        uint32_t m = mask[w];
        while (m) {
            const int i = w * 32 + __ffs(m) - 1;
            m &= m - 1u;
            const int r = swap ? c0 + i : lane_row, col = swap ? lane_row : c0 + i;
            if (pos < pr.rr_cap) pr.rr_list[pos] = make_int2(ti.row0 + r, ti.wcol0 + col);
            ++pos;
        }
    }
}

template <int BN, bool kSwap>
struct Shape {
    static constexpr int XR = 128;            // rows of the MMA A operand tile
    static constexpr int YR = BN;             // rows of the MMA B operand tile
    static constexpr int kXBytes = XR * kBK * 2;
    static constexpr int kYBytes = YR * kBK * 2;
    static constexpr int kStageBytes = kXBytes + kYBytes;
    static constexpr int kActRows = kSwap ? BN : 128;   // activation rows per tile
    static constexpr int kOutCols = kSwap ? 128 : BN;   // output columns per tile
    // K is accumulated in chunks of kChunkKB k-blocks in TMEM; each chunk is
    // added into fp32 registers by the epilogue (see the file comment).
    static constexpr int kChunkKB = LMOE_CHUNK_KB;
    // TMEM chunk buffers: all 512 columns (one CTA per SM). Narrow tiles get
    // many buffers, so the MMA can run many chunks ahead of the epilogue's
    // drains: each chunk's round trip (commit, drain, release) is long next to
    // a 32-token chunk's tensor-core time.
#ifndef LMOE_TMEM_BUFS
    static constexpr int kBufs = 512 / BN;
#else
    static constexpr int kBufs = (LMOE_TMEM_BUFS * BN <= 512) ? LMOE_TMEM_BUFS : 512 / BN;
#endif
    static constexpr int kCols = kBufs * BN;
    static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128
                                        : kCols <= 256 ? 256 : 512;
    static constexpr int kEpiWarps = BN >= 128 ? 8 : 4;  // two warps per TMEM lane quarter for wide tiles
    static constexpr int kColsPerThread = BN / (kEpiWarps / 4);
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    // per epilogue warp: one 32-row x 128-byte output box, 128-byte swizzled, for bulk tensor stores
    static constexpr int kStageOutBytes = kSwap ? 0 : 4096;
};

// Per-expert tile prefix and tile records of a grouped problem for activation
// tiles of R rows.
template <int R>
__device__ __forceinline__ const int* grouped_prefix(const DeviceRouting& r) {
    static_assert(R == 32 || R == 64 || R == 128 || R == 256, "activation tile rows");
    return R == kDecodeTN ? r.pfxdec : R == 64 ? r.pfx64 : R == 128 ? r.pfx128 : r.pfx256;
}
template <int R>
__device__ __forceinline__ const int4* grouped_records(const DeviceRouting& r) {
    return R == kDecodeTN ? r.rec32 : R == 64 ? r.rec64 : R == 128 ? r.rec128 : r.rec256;
}

__device__ __forceinline__ int n_col_tiles(const GemmProblem& pr, int out_cols) { return pr.n / out_cols; }

// Tiles of the dense problems of a launch, and dense tile t -> its problem
// (t becomes the tile's index inside that problem).
static_assert(kMaxProb == 3, "dense_total / dense_problem are written out for three problems");
__device__ __forceinline__ int dense_total(const TcParams& P) {
    return P.dense_tiles[0] + (P.nprob > 1 ? P.dense_tiles[1] : 0) + (P.nprob > 2 ? P.dense_tiles[2] : 0);
}
__device__ __forceinline__ int dense_problem(const TcParams& P, int& t) {
    if (P.nprob < 2 || t < P.dense_tiles[0]) return 0;
    t -= P.dense_tiles[0];
    if (P.nprob < 3 || t < P.dense_tiles[1]) return 1;
    t -= P.dense_tiles[1];
    return 2;
}

template <int BN, bool kSwap>
__device__ __forceinline__ int total_tiles(const TcParams& P) {
    using S = Shape<BN, kSwap>;
    if (P.prob[0].grouped) {
        const int* pfx = grouped_prefix<S::kActRows>(P.r);
        return pfx[P.r.E] * n_col_tiles(P.prob[0], S::kOutCols);
    }
    return dense_total(P);
}

// Tile t -> coordinates. Dense problems are rasterised in groups of kGroupM
// row tiles (column tiles outer within a group) so that concurrently running
// CTAs share both operands in L2. Grouped problems walk experts in order,
// column tiles inner, so an expert's weights are read while its rows are hot;
// their row tiles come from the permutation's tile records (one 16-byte load,
// instead of a dependent search over the per-expert prefix at every tile).
template <int BN, bool kSwap>
__device__ __forceinline__ TileInfo decode_tile(const TcParams& P, int t) {
    using S = Shape<BN, kSwap>;
    TileInfo ti;
    if (P.prob[0].grouped) {
        const GemmProblem& pr = P.prob[0];
        const int nct = n_col_tiles(pr, S::kOutCols);
        const int mt = t / nct, ct = t % nct;
        int4 rc = __ldg(grouped_records<S::kActRows>(P.r) + mt);
#if LMOE_CHECKS
        // a tile record must name a group and a row range inside the permuted rows
        if (!lmoe_check((unsigned)rc.x < (unsigned)P.r.E && rc.y >= 0 && rc.z >= 1 && rc.z <= S::kActRows &&
                            rc.y + rc.z <= __ldg(P.r.offsets + P.r.E),
                        P.err))
            rc = make_int4(0, 0, 0, 0);  // a tile with no rows: loads stay in bounds, nothing is stored
#endif
        const int e = pr.expert_mod ? rc.x % pr.expert_mod : rc.x;
        ti.p = 0;
        ti.row0 = rc.y;
        ti.rows = rc.z;
        ti.col0 = ct * S::kOutCols;
        ti.wrow0 = e * pr.b_rows_per_expert + ti.col0;
        ti.wcol0 = ti.wrow0;
        ti.e = e;
        ti.half = !kSwap && ti.rows <= 64;
        return ti;
    }
    const int p = dense_problem(P, t);
    const GemmProblem& pr = P.prob[p];
    const int nct = n_col_tiles(pr, S::kOutCols);
    const int mtc = (pr.m_rows + S::kActRows - 1) / S::kActRows;
    int mt, ct;
    if (kSwap) {  // token tiles inner: the tiles that share a weight block run together
        ct = t / mtc;
        mt = t % mtc;
    } else {
        const int g = t / (kGroupM * nct), r = t % (kGroupM * nct);
        const int ms = min(kGroupM, mtc - g * kGroupM);
        mt = g * kGroupM + r % ms;
        ct = r / ms;
    }
    ti.p = p;
    ti.row0 = mt * S::kActRows;
    ti.rows = min(S::kActRows, pr.m_rows - ti.row0);
    ti.col0 = ct * S::kOutCols;
    ti.wrow0 = ti.col0;
    ti.wcol0 = ti.col0;
    ti.e = -1;
    ti.half = !kSwap && ti.rows <= 64;
    return ti;
}

// Epilogue of one tile from the thread's fp32 accumulators acc[CW], which
// hold accumulator columns c0 .. c0+CW-1 of TMEM lane `lane_row`.
// Non-swapped tiles with an output tensor map are written with bulk tensor
// stores: the warp stages its 32 rows x 128 bytes in shared memory with the
// 128-byte swizzle (conflict-free writes) and one lane issues the store. Rows
// past a dense problem's end are clipped by the tensor bounds; a grouped tile
// whose 32-row slab runs into the next expert's rows uses plain masked stores.
template <int BN, bool kSwap, int CW>
__device__ __forceinline__ void epilogue_store(const GemmProblem& pr, const TileInfo& ti, int lane_row, int c0,
                                               float (&acc)[CW], const CUtensorMap* omap, uint8_t* stage) {
    const int epi = pr.epi;
    const int lane = threadIdx.x & 31;
    if (pr.wscale) {  // NVFP4 experts: h = g_e * (sum of code * block scale * activation)
        const float g = __ldg(&pr.wscale[ti.e]);
#pragma unroll
        for (int i = 0; i < CW; ++i) acc[i] *= g;
    }
    if (epi == EPI_RELU2_BF16 || epi == EPI_RELU2_F32) {
#pragma unroll
        for (int i = 0; i < CW; ++i) {
            float a = fmaxf(acc[i], 0.f);
            acc[i] = a * a;
        }
        // exact re-rounding list (bf16 mode): large activations near a rounding midpoint, marked
        // in a bit mask first, then listed (a few per tile) with one atomic per warp. All 32
        // lanes of the warp are here.
        if (epi == EPI_RELU2_BF16 && pr.rr_list != nullptr) {
            constexpr int kW = (CW + 31) / 32;
            uint32_t mask[kW];
#pragma unroll
            for (int w = 0; w < kW; ++w) mask[w] = 0u;
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                // non-swapped: row lane_row of the tile, weight row c0 + i; swapped: the reverse
                const int r = kSwap ? c0 + i : lane_row;
                if (r < ti.rows && rr_flag(acc[i], pr.rr_tau2_bits, pr.rr_ulps)) mask[i >> 5] |= 1u << (i & 31);
            }
            int n = 0;
#pragma unroll
            for (int w = 0; w < kW; ++w) n += __popc(mask[w]);
            if (__any_sync(0xFFFFFFFFu, n != 0)) rr_append_warp<kW>(pr, n, mask, ti, lane_row, c0, kSwap);
        }
    }
    if (!kSwap && pr.resid && lane_row < ti.rows) {  // block residual: out = resid + acc (fp32)
        const uint4* rs = reinterpret_cast<const uint4*>(pr.resid + (size_t)(ti.row0 + lane_row) * pr.ldo + ti.col0 + c0);
#pragma unroll
        for (int q8 = 0; q8 < CW / 8; ++q8) {
            const uint4 u = __ldg(rs + q8);
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[q8 * 8 + 2 * j] += __uint_as_float(w4[j] << 16);
                acc[q8 * 8 + 2 * j + 1] += __uint_as_float(w4[j] & 0xFFFF0000u);
            }
        }
    }
    if (!kSwap) {
        const bool bf16_out = epi == EPI_BF16 || epi == EPI_RELU2_BF16;
        const int slab0 = lane_row - lane;  // first row of this warp's 32-row slab
        if (omap && (!pr.grouped || slab0 + 32 <= ti.rows)) {
            if (epi == EPI_SCALE_F32) {
                const float sc = __ldg(&pr.row_scale[ti.row0 + lane_row]);
#pragma unroll
                for (int i = 0; i < CW; ++i) acc[i] *= sc;
            }
            uint8_t* myrow = stage + lane * 128;
            constexpr int kGroupsF32 = CW / 32, kGroupsBf16 = CW / 64;
            const int ngroups = bf16_out ? kGroupsBf16 : kGroupsF32;
#pragma unroll
            for (int g = 0; g < (CW / 32); ++g) {
                if (g >= ngroups) break;
                if (lane == 0) bulk_wait_read_all();  // staging buffer free again
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v;
                    if (bf16_out) {
                        const int b = g * 64 + c * 8;
                        v = make_uint4(pack_bf16x2(acc[b], acc[b + 1]), pack_bf16x2(acc[b + 2], acc[b + 3]),
                                       pack_bf16x2(acc[b + 4], acc[b + 5]), pack_bf16x2(acc[b + 6], acc[b + 7]));
                    } else {
                        const int b = g * 32 + c * 4;
                        v = make_uint4(__float_as_uint(acc[b]), __float_as_uint(acc[b + 1]),
                                       __float_as_uint(acc[b + 2]), __float_as_uint(acc[b + 3]));
                    }
                    *reinterpret_cast<uint4*>(myrow + ((c ^ (lane & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int x = ti.col0 + c0 + g * (bf16_out ? 64 : 32);
                    tma_store_2d(omap, stage, x, ti.row0 + slab0);
                    bulk_commit();
                }
            }
            return;
        }
        // thread owns activation row (row0 + lane_row), output columns col0 + c0 ..
        if (lane_row >= ti.rows) return;
        const long long row = ti.row0 + lane_row;
        if (epi == EPI_SCALE_F32) {
            const float sc = __ldg(&pr.row_scale[row]);
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] *= sc;
        }
        if (bf16_out) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(pr.out) + row * pr.ldo + ti.col0 + c0);
#pragma unroll
            for (int q = 0; q < CW / 8; ++q)
                dst[q] = make_uint4(pack_bf16x2(acc[8 * q], acc[8 * q + 1]), pack_bf16x2(acc[8 * q + 2], acc[8 * q + 3]),
                                    pack_bf16x2(acc[8 * q + 4], acc[8 * q + 5]),
                                    pack_bf16x2(acc[8 * q + 6], acc[8 * q + 7]));
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(pr.out) + row * pr.ldo + ti.col0 + c0);
#pragma unroll
            for (int q = 0; q < CW / 4; ++q)
                dst[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        }
    } else {
        // thread owns output column (col0 + lane_row); accumulator columns are
        // the tile's tokens row0 + c0 + i. Lanes write consecutive columns.
        const long long col = ti.col0 + lane_row;
#pragma unroll
        for (int i = 0; i < CW; ++i) {
            const int tok = c0 + i;
            if (tok < ti.rows) {
                const long long row = ti.row0 + tok;
                float x = acc[i];
                if (epi == EPI_SCALE_F32) x *= __ldg(&pr.row_scale[row]);
                if (pr.resid) x += __uint_as_float((uint32_t)pr.resid[row * pr.ldo + col] << 16);
                if (epi == EPI_BF16 || epi == EPI_RELU2_BF16)
                    static_cast<__nv_bfloat16*>(pr.out)[row * pr.ldo + col] = __float2bfloat16_rn(x);
                else
                    static_cast<float*>(pr.out)[row * pr.ldo + col] = x;
            }
        }
    }
}

__device__ __forceinline__ int tile_kblocks(const GemmProblem& pr) {
    int n = pr.kdim[0] / kBK;
    if (pr.nseg > 1) n += pr.kdim[1] / kBK;
    return n;
}

inline void fill_params(TcParams& P, const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob,
                        const DeviceRouting& r, int* err, unsigned spin) {
    memset(&P, 0, sizeof(P));
    for (int i = 0; i < nmaps && i < kMaxMaps; ++i) P.maps[i] = maps[i];
    for (int i = 0; i < nprob; ++i) P.prob[i] = probs[i];
    P.nprob = nprob;
    P.nmaps = nmaps < kMaxMaps ? nmaps : kMaxMaps;
    P.r = r;
    P.err = err;
    P.spin = spin;
}

}  // namespace
}  // namespace lmoe
