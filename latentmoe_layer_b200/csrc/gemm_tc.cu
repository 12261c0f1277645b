// gemm_tc.cu -- persistent tcgen05 GEMM engine for sm_100a.
//
// Every dense contraction of the layer runs here: the router logits, fc1
// (fc1_latent_proj), the shared expert's up projection, each routed expert's
// up and down projection (grouped by expert over the permuted rows) and the
// output GEMM that fuses fc2_latent_proj with the shared expert's down
// projection by concatenating their K ranges into one accumulator
// (y = comb W_fc2^T + a_s W_sd^T; "Nemotron 3 Ultra 架构 QA", Q5.7).
//
// Structure of one CTA (one per SM, persistent over tiles):
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles into a ring of
//               shared-memory stages (mbarrier complete_tx), no multicast.
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma.cta_group::1.kind::f16,
//               128 x BN x 16 per instruction, fp32 accumulation in TMEM.
//   warps 2..   epilogue (4 or 8 warps; two per TMEM lane quarter for wide
//               tiles): tcgen05.ld, then the fused activation (relu2), row
//               weight or bf16 rounding, and the stores.
//
// Accumulation precision. The tensor core's fp32 accumulation over long K
// carries several times the error of round-to-nearest fp32, and that error
// grows with the accumulator's magnitude. Every GEMM output of the layer is
// rounded to bf16 before the next GEMM, so that error turns into flipped bf16
// roundings of large activations (one bf16 ulp at 64 is 0.5). K is therefore
// accumulated in chunks of 4 k-blocks (256) in a ring of TMEM buffers; the
// epilogue adds each chunk into fp32 registers, in order, while the MMA warp
// fills the next buffer. Partial sums stay small, so the tensor-core error
// no longer scales with the output, at the price of reading TMEM once per
// chunk instead of once per tile.
//
// Two tile shapes share the code:
//   kSwap = false  MMA M = 128 activation rows, N = BN weight rows.
//   kSwap = true   MMA M = 128 weight rows, N = BN tokens (decode batches,
//                  where each expert sees a handful of tokens: the weights sit
//                  on the 128-row side so no tensor-core work is padding).
// Every mbarrier wait is bounded; on running out the kernel records
// LMOE_ERR_TIMEOUT, drains its own TMA loads and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <string.h>

#include "lmoe_internal.h"
#include "ptx.cuh"

#ifndef LMOE_CHUNK_KB
#define LMOE_CHUNK_KB 4   // k-blocks (of 64) per TMEM accumulation chunk
#endif
#ifndef LMOE_PROMOTE_F64
#define LMOE_PROMOTE_F64 0  // 1: chunk partials are added into fp64 registers
#endif
#ifndef LMOE_MAX_BN
#define LMOE_MAX_BN 256
#endif

namespace lmoe {
namespace {

constexpr int kMaxMaps = 8;
constexpr int kGroupM = 16;

struct alignas(64) TcParams {
    CUtensorMap maps[kMaxMaps];
    GemmProblem prob[2];
    int nprob;
    int nmaps;
    int dense_tiles[2];
    DeviceRouting r;
    int* err;
    unsigned spin;
};

struct TileInfo {
    int p;       // problem
    int row0;    // first activation row (permuted row for grouped problems)
    int rows;    // valid activation rows in this tile
    int wrow0;   // first weight row (row of B)
    int col0;    // first output column
    int e;       // expert of a grouped tile (-1 for dense problems)
    bool half;   // non-swapped tile with <= 64 valid rows: M = 64 MMAs (the expert's ragged tail)
};

template <int BN, bool kSwap, bool kFp4 = false>
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
    static constexpr int kBufs = (4 * BN <= 512) ? 4 : 512 / BN;     // TMEM chunk buffers
    static constexpr int kCols = kBufs * BN;
    static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128
                                        : kCols <= 256 ? 256 : 512;
    static constexpr int kEpiWarps = BN >= 128 ? 8 : 4;  // two warps per TMEM lane quarter for wide tiles
    static constexpr int kColsPerThread = BN / (kEpiWarps / 4);
    // NVFP4 weights (swap tiles): the 128 x 64 weight tile arrives as 4096 bytes of
    // E2M1 codes and 512 bytes of E4M3 scales, and dequantisation warps write the
    // bf16 operand tile from them.
    static constexpr int kRawBytes = kFp4 ? 4096 + 512 : 0;
    static constexpr int kTxBytes = kFp4 ? kRawBytes + kYBytes : kStageBytes;  // bytes the producer's copies carry
    // Dequantisation warps, in groups that take alternate k-blocks so that
    // several stages convert at once: 8 groups of 1 warp for decode tiles,
    // 2 groups of 2 warps where the registers allow fewer warps.
    static constexpr int kDeqWarps = !kFp4 ? 0 : BN <= 64 ? 8 : 4;
    static constexpr int kDeqGroups = !kFp4 ? 1 : BN <= 64 ? 8 : 2;
    static constexpr int kDeqGroupWarps = kFp4 ? kDeqWarps / kDeqGroups : 1;
    static constexpr int kDeqItems = kFp4 ? 256 / (32 * kDeqGroupWarps) : 0;  // (row, half-row) items per thread
    static constexpr int kThreads = 64 + 32 * (kEpiWarps + kDeqWarps);
    // per epilogue warp: one 32-row x 128-byte output box, 128-byte swizzled, for bulk tensor stores
    static constexpr int kStageOutBytes = kSwap ? 0 : 4096;
    static constexpr int kBarBytes = 512;
    static constexpr int kLutBytes = kFp4 ? 256 * 4 : 0;
    static_assert(!kFp4 || kSwap, "NVFP4 weights sit on the MMA M side");
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

template <int BN, bool kSwap>
__device__ __forceinline__ int total_tiles(const TcParams& P) {
    using S = Shape<BN, kSwap>;
    if (P.prob[0].grouped) {
        const int* pfx = grouped_prefix<S::kActRows>(P.r);
        return pfx[P.r.E] * n_col_tiles(P.prob[0], S::kOutCols);
    }
    return P.dense_tiles[0] + (P.nprob > 1 ? P.dense_tiles[1] : 0);
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
        const int4 rc = __ldg(grouped_records<S::kActRows>(P.r) + mt);
        const int e = rc.x;
        ti.p = 0;
        ti.row0 = rc.y;
        ti.rows = rc.z;
        ti.col0 = ct * S::kOutCols;
        ti.wrow0 = e * pr.b_rows_per_expert + ti.col0;
        ti.e = e;
        ti.half = !kSwap && ti.rows <= 64;
        return ti;
    }
    int p = 0;
    if (P.nprob > 1 && t >= P.dense_tiles[0]) {
        t -= P.dense_tiles[0];
        p = 1;
    }
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

// ---------------------------------------------------------------- NVFP4
// E2M1 codes -> bf16. Eight codes (one 32-bit word, element i in nibble i) give
// four bf16 pairs. The three magnitude bits index two byte tables held in
// registers (high and low byte of the bf16 value of 0, 0.5, 1, 1.5, 2, 3, 4, 6)
// with byte permutes; the sign bits are moved to bit 7 of the high bytes; the
// block scale (bf16, both halves) multiplies the pair. code * scale has at most
// 6 significant bits and lies in [2^-10, 2688], so the product is exact.
__device__ __forceinline__ uint4 e2m1x8_to_bf16(uint32_t c, uint32_t scale2) {
    constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u;  // high bytes of magnitudes 0..3, 4..7
    constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;  // low bytes
    const uint32_t mag = c & 0x77777777u;
    const uint32_t d = c << 4;  // bit 7 of byte j = sign of element 2j; bit 7 of c's byte j = sign of 2j + 1
    const uint32_t mhi = mag >> 16;
    const uint32_t h0 = prmt(kHi0, kHi1, mag) | (prmt(d, c, 0x5140u) & 0x80808080u);
    const uint32_t l0 = prmt(kLo0, kLo1, mag);
    const uint32_t h1 = prmt(kHi0, kHi1, mhi) | (prmt(d, c, 0x7362u) & 0x80808080u);
    const uint32_t l1 = prmt(kLo0, kLo1, mhi);
    uint4 o;
    o.x = mul_bf16x2(prmt(l0, h0, 0x5140u), scale2);
    o.y = mul_bf16x2(prmt(l0, h0, 0x7362u), scale2);
    o.z = mul_bf16x2(prmt(l1, h1, 0x5140u), scale2);
    o.w = mul_bf16x2(prmt(l1, h1, 0x7362u), scale2);
    return o;
}

// bf16 value of an E4M3 byte (bias 7, 3 mantissa bits, subnormals m * 2^-9),
// duplicated in both halves. Exact: E4M3 values need 4 significant bits.
__device__ __forceinline__ uint32_t e4m3_to_bf16x2(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
    if (b & 0x80u) v = -v;
    const uint32_t h = __float_as_uint(v) >> 16;
    return h | (h << 16);
}

template <int BN, int STAGES, bool kSwap, bool kFp4 = false>
__global__ void __launch_bounds__(Shape<BN, kSwap, kFp4>::kThreads, 1) k_gemm_tc(const __grid_constant__ TcParams P) {
    using S = Shape<BN, kSwap, kFp4>;
    constexpr int NB = S::kBufs, CK = S::kChunkKB, CW = S::kColsPerThread;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((base_u32 + 1023u) & ~1023u) - base_u32);
    uint8_t* sX = smem;                                  // STAGES x kXBytes
    uint8_t* sY = smem + STAGES * S::kXBytes;            // STAGES x kYBytes
    uint8_t* sRaw = sY + STAGES * S::kYBytes;            // STAGES x kRawBytes (NVFP4 codes + scales)
    uint8_t* sOut = sRaw + STAGES * S::kRawBytes;        // kEpiWarps x kStageOutBytes
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + S::kEpiWarps * S::kStageOutBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* cfull = empty + STAGES;   // chunk accumulator ready (MMA -> epilogue)
    uint64_t* cempty = cfull + NB;      // chunk accumulator drained (epilogue -> MMA)
    uint64_t* done = cempty + NB;
    uint64_t* deq = done + 1;           // NVFP4: bf16 weight tile written (dequantisation -> MMA)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(deq + STAGES);
    uint32_t* scale_lut = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(full) + S::kBarBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&cfull[b], 1);
            mbar_init(&cempty[b], S::kEpiWarps);
        }
        mbar_init(done, 1);
        if (kFp4)
            for (int s = 0; s < STAGES; ++s) mbar_init(&deq[s], S::kDeqGroupWarps);
        fence_mbar_init();
    }
    if (kFp4 && warp >= 2 + S::kEpiWarps)
        for (int b = threadIdx.x - 32 * (2 + S::kEpiWarps); b < 256; b += 32 * S::kDeqWarps)
            scale_lut[b] = e4m3_to_bf16x2((uint32_t)b);
    if (warp == 0 && lane == 0)
        for (int i = 0; i < P.nmaps; ++i) prefetch_tmap(&P.maps[i]);
    if (warp == 1) {
        tmem_alloc(tmem_slot, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ntiles = total_tiles<BN, kSwap>(P);
    int* err = P.err;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, kSwap>(P, t);
            const GemmProblem& pr = P.prob[ti.p];
            for (int sg = 0; sg < pr.nseg && ok; ++sg) {
                const CUtensorMap* amap = &P.maps[pr.a_map[sg]];
                const CUtensorMap* bmap = &P.maps[pr.b_map[sg]];
                const int kb_n = pr.kdim[sg] / kBK;
                for (int kb = 0; kb < kb_n; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, P.spin, err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], S::kTxBytes);
                    if (kFp4) {
                        // weight tile (128 rows x 64 K) of NVFP4 codes and scales; tokens by TMA
                        const long long tile = (long long)(ti.wrow0 >> 7) * kb_n + kb;
                        uint8_t* raw = sRaw + stage * S::kRawBytes;
                        bulk_load(raw, pr.wq_codes + tile * 4096, 4096, &full[stage]);
                        bulk_load(raw + 4096, pr.wq_sf + tile * 512, 512, &full[stage]);
                        tma_load_2d(sY + stage * S::kYBytes, amap, &full[stage], kb * kBK, ti.row0);
                    } else if (!kSwap) {
                        tma_load_2d(sX + stage * S::kXBytes, amap, &full[stage], kb * kBK, ti.row0);
                        tma_load_2d(sY + stage * S::kYBytes, bmap, &full[stage], kb * kBK, ti.wrow0);
                    } else {
                        tma_load_2d(sX + stage * S::kXBytes, bmap, &full[stage], kb * kBK, ti.wrow0);
                        tma_load_2d(sY + stage * S::kYBytes, amap, &full[stage], kb * kBK, ti.row0);
                    }
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        // every load this thread issued has landed before the CTA can exit
        for (int s = 0; s < STAGES; ++s)
            if ((issued >> s) & 1u) mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, 1u << 26, err);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_full = idesc_bf16_f32(128, BN);
        constexpr uint32_t idesc_half = idesc_bf16_f32(64, BN);
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, kSwap>(P, t);
            const int kb_total = tile_kblocks(P.prob[ti.p]);
            // M = 64 puts D rows 16q..16q+15 in TMEM lanes 32q..32q+15 (q = lane quarter)
            const uint32_t idesc = ti.half ? idesc_half : idesc_full;
            for (int kb0 = 0; kb0 < kb_total && ok; kb0 += CK) {
                // next chunk accumulator must have been drained by the epilogue
                if (!mbar_wait_bounded(&cempty[buf], bphase ^ 1u, P.spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * BN);
                const int kb1 = min(kb_total, kb0 + CK);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(kFp4 ? &deq[stage] : &full[stage], phase, P.spin, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = sdesc_sw128(smem_u32(sX + stage * S::kXBytes));
                    const uint64_t bdesc = sdesc_sw128(smem_u32(sY + stage * S::kYBytes));
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        // +32 bytes per K step of 16 bf16 inside the 128-byte swizzled row
                        umma_bf16(d, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc,
                                  (kb > kb0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&cfull[buf]);
                if (++buf == NB) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
        }
        // all MMAs issued by this thread have completed before TMEM is freed
        umma_commit(done);
        mbar_wait_bounded(done, 0, 1u << 26, err);
    } else if (kFp4 && warp >= 2 + S::kEpiWarps) {
        // ------------------------------------------------ NVFP4 dequantisation
        // Each thread converts (row, half-row) items of the 128 x 64 weight tile:
        // 32 codes (16 bytes) and their two block scales -> four 16-byte chunks
        // of the 128-byte-swizzled bf16 operand row (chunk j at (j ^ (row & 7)) * 16).
        // Group g takes the k-blocks c with c % kDeqGroups == g (c counts the
        // CTA's k-blocks in the producer's order), so groups convert different
        // stages at the same time.
        const int dw = warp - (2 + S::kEpiWarps);
        const int grp = dw / S::kDeqGroupWarps;
        const int gt = (dw % S::kDeqGroupWarps) * 32 + lane;  // thread within the group
        uint32_t c = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, kSwap>(P, t);
            const int kb_total = tile_kblocks(P.prob[ti.p]);
            for (int kb = 0; kb < kb_total; ++kb, ++c) {
                if ((int)(c % S::kDeqGroups) != grp) continue;
                const int stage = (int)(c % STAGES);
                const uint32_t phase = (c / STAGES) & 1u;
                if (!mbar_wait_bounded(&full[stage], phase, P.spin, err)) {
                    ok = false;
                    break;
                }
                const uint8_t* raw = sRaw + stage * S::kRawBytes;
                uint8_t* dst = sX + stage * S::kXBytes;
                constexpr int NI = S::kDeqItems > 0 ? S::kDeqItems : 1;  // (the branch is dead without NVFP4)
#pragma unroll
                for (int i0 = 0; i0 < NI; i0 += 2) {  // two items' loads first, so their conversions overlap
                    constexpr int NJ = NI >= 2 ? 2 : 1;
                    uint4 cw[NJ];
                    uint32_t sA[NJ], sB[NJ];
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int it = gt + (i0 + j) * 32 * S::kDeqGroupWarps, r = it >> 1, hh = it & 1;
                        cw[j] = *reinterpret_cast<const uint4*>(raw + r * 32 + hh * 16);
                        const uint32_t sb = *reinterpret_cast<const uint16_t*>(raw + 4096 + r * 4 + hh * 2);
                        sA[j] = scale_lut[sb & 0xFFu];
                        sB[j] = scale_lut[sb >> 8];
                    }
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int it = gt + (i0 + j) * 32 * S::kDeqGroupWarps, r = it >> 1, hh = it & 1;
                        uint8_t* row = dst + r * 128;
                        const int sw = r & 7, j0 = 4 * hh;
                        const uint4 o0 = e2m1x8_to_bf16(cw[j].x, sA[j]), o1 = e2m1x8_to_bf16(cw[j].y, sA[j]);
                        const uint4 o2 = e2m1x8_to_bf16(cw[j].z, sB[j]), o3 = e2m1x8_to_bf16(cw[j].w, sB[j]);
                        st_shared_v4(row + (((j0 + 0) ^ sw) << 4), o0);
                        st_shared_v4(row + (((j0 + 1) ^ sw) << 4), o1);
                        st_shared_v4(row + (((j0 + 2) ^ sw) << 4), o2);
                        st_shared_v4(row + (((j0 + 3) ^ sw) << 4), o3);
                    }
                }
                fence_proxy_async_smem();  // generic-proxy writes visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(&deq[stage]);
            }
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int q = warp & 3;                // TMEM lane quarter this warp may access
        const int c0 = (ew >> 2) * CW;         // accumulator columns this warp owns
        const int lane_row = q * 32 + lane;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, kSwap>(P, t);
            const GemmProblem& pr = P.prob[ti.p];
            const int kb_total = tile_kblocks(pr);
#if LMOE_PROMOTE_F64
            double accd[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) accd[i] = 0.0;
#else
            float acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = 0.f;
#endif
            for (int kb0 = 0; kb0 < kb_total; kb0 += CK) {
                if (!mbar_wait_bounded(&cfull[buf], bphase, P.spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c0);
#pragma unroll
                for (int c = 0; c < CW; c += 32) {
                    uint32_t r0[16], r1[16];
                    tmem_ld16(taddr + (uint32_t)c, r0);
                    if (c + 16 < CW) tmem_ld16(taddr + (uint32_t)(c + 16), r1);
                    tmem_ld_wait();
#if LMOE_PROMOTE_F64
#pragma unroll
                    for (int i = 0; i < 16; ++i) accd[c + i] += (double)__uint_as_float(r0[i]);
                    if (c + 16 < CW) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) accd[c + 16 + i] += (double)__uint_as_float(r1[i]);
                    }
#else
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[c + i] += __uint_as_float(r0[i]);
                    if (c + 16 < CW) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc[c + 16 + i] += __uint_as_float(r1[i]);
                    }
#endif
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&cempty[buf]);
                if (++buf == NB) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
            if (!ok) break;
#if LMOE_PROMOTE_F64
            float acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = (float)accd[i];
#endif
            const CUtensorMap* omap = pr.out_map >= 0 && !ti.half ? &P.maps[pr.out_map] : nullptr;
            // half tiles: only lanes 0..15 of each quarter carry rows (row = 16q + lane)
            const int row_in_tile = ti.half ? (lane < 16 ? q * 16 + lane : 1 << 20) : lane_row;
            epilogue_store<BN, kSwap, CW>(pr, ti, row_in_tile, c0, acc, omap, sOut + ew * S::kStageOutBytes);
        }
        if (!kSwap && lane == 0) bulk_wait_all();  // this warp's bulk stores are complete
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, S::kTmemCols);
    }
}

// ---------------------------------------------------------------- 2-SM pairs
// (Selected with LMOE_OPT_GEMM_PATH = 4; measured no faster than the single-SM
// tiles on this layer, whose steady state is set by the 1 kW power cap.)
// A cluster of two CTAs on neighbouring SMs computes one 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256). Each CTA stages its own 128 A
// rows and its own half (128 rows) of B, 32 KB per k-block instead of the
// 48 KB a single CTA needs for 128 x 256, which keeps each SM's shared-memory
// traffic (TMA writes plus MMA operand reads) within its bandwidth and leaves
// room for 6 pipeline stages. The leader CTA (rank 0) issues the MMAs and
// commits them to barriers in both CTAs; each CTA drains its own 128 TMEM
// lanes, adds the K chunks in fp32 registers exactly as the single-CTA kernel
// does, and writes its own rows. Loads use the cta_group::2 form that counts
// completion on the leader's barrier; nothing is multicast.
struct PairShape {
    static constexpr int BN = 256;
    static constexpr int kXBytes = 128 * kBK * 2;   // this CTA's 128 A rows
    static constexpr int kYBytes = 128 * kBK * 2;   // this CTA's 128 rows of B
    static constexpr int kStageBytes = kXBytes + kYBytes;
    static constexpr int kChunkKB = LMOE_CHUNK_KB;
    static constexpr int kBufs = 2;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kEpiWarps = 8;
    static constexpr int kColsPerThread = 128;
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kStageOutBytes = 4096;
    static constexpr int kGroupM = 8;
};

__device__ __forceinline__ int pair_total_tiles(const TcParams& P) {
    if (P.prob[0].grouped) return P.r.pfx256[P.r.E] * (P.prob[0].n / PairShape::BN);
    return P.dense_tiles[0] + (P.nprob > 1 ? P.dense_tiles[1] : 0);
}

// Pair tile t -> this CTA's half: rows row0 .. row0+rows-1 (rows may be <= 0
// for the second CTA of a short tile), B rows wrow0 .. wrow0+127, output
// columns col0 .. col0+255.
__device__ __forceinline__ TileInfo pair_decode(const TcParams& P, int t, uint32_t rank) {
    int p = 0, prow0, prows, ct, wbase = 0, e = -1;
    if (P.prob[0].grouped) {
        const GemmProblem& pr = P.prob[0];
        const int nct = pr.n / PairShape::BN;
        const int mt = t / nct;
        ct = t % nct;
        const int4 rc = __ldg(P.r.rec256 + mt);
        prow0 = rc.y;
        prows = rc.z;
        wbase = rc.x * pr.b_rows_per_expert;
        e = rc.x;
    } else {
        if (P.nprob > 1 && t >= P.dense_tiles[0]) {
            t -= P.dense_tiles[0];
            p = 1;
        }
        const GemmProblem& pr = P.prob[p];
        const int nct = pr.n / PairShape::BN;
        const int mtc = (pr.m_rows + 255) / 256;
        const int g = t / (PairShape::kGroupM * nct), r = t % (PairShape::kGroupM * nct);
        const int ms = min(PairShape::kGroupM, mtc - g * PairShape::kGroupM);
        const int mt = g * PairShape::kGroupM + r % ms;
        ct = r / ms;
        prow0 = mt * 256;
        prows = min(256, pr.m_rows - prow0);
    }
    TileInfo ti;
    ti.p = p;
    ti.row0 = prow0 + (int)rank * 128;
    ti.rows = min(128, prows - (int)rank * 128);
    ti.col0 = ct * PairShape::BN;
    ti.wrow0 = wbase + ti.col0 + (int)rank * 128;
    ti.e = e;
    ti.half = false;
    return ti;
}

template <int STAGES>
__global__ void __launch_bounds__(PairShape::kThreads, 1) k_gemm_tc_pair(const __grid_constant__ TcParams P) {
    using S = PairShape;
    constexpr int NB = S::kBufs, CK = S::kChunkKB, CW = S::kColsPerThread, BN = S::BN;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((base_u32 + 1023u) & ~1023u) - base_u32);
    uint8_t* sX = smem;
    uint8_t* sY = smem + STAGES * S::kXBytes;
    uint8_t* sOut = sY + STAGES * S::kYBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + S::kEpiWarps * S::kStageOutBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* cfull = empty + STAGES;
    uint64_t* cempty = cfull + NB;
    uint64_t* done = cempty + NB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&cfull[b], 1);
            mbar_init(&cempty[b], 2 * S::kEpiWarps);  // both CTAs' epilogue warps
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0)
        for (int i = 0; i < P.nmaps; ++i) prefetch_tmap(&P.maps[i]);
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, S::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers and TMEM of both CTAs are ready
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ntiles = pair_total_tiles(P);
    int* err = P.err;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        for (int t = pair; t < ntiles && ok; t += npairs) {
            const TileInfo ti = pair_decode(P, t, rank);
            const GemmProblem& pr = P.prob[ti.p];
            for (int sg = 0; sg < pr.nseg && ok; ++sg) {
                const CUtensorMap* amap = &P.maps[pr.a_map[sg]];
                const CUtensorMap* bmap = &P.maps[pr.b_map[sg]];
                const int kb_n = pr.kdim[sg] / kBK;
                for (int kb = 0; kb < kb_n; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, P.spin, err)) {
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * S::kStageBytes);
                    const uint32_t lbar = mapa_shared(&full[stage], 0);
                    tma_load_2d_pair(sX + stage * S::kXBytes, amap, lbar, kb * kBK, ti.row0);
                    tma_load_2d_pair(sY + stage * S::kYBytes, bmap, lbar, kb * kBK, ti.wrow0);
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        // the leader's full barriers count both CTAs' bytes: waiting on them drains
        // every load of the pair before either CTA can pass the final cluster barrier
        if (leader)
            for (int s = 0; s < STAGES; ++s)
                if ((issued >> s) & 1u) mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, 1u << 26, err);
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------------------------ MMA issuer (leader only)
        constexpr uint32_t idesc = idesc_bf16_f32(256, BN);
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (int t = pair; t < ntiles && ok; t += npairs) {
            const TileInfo ti = pair_decode(P, t, rank);
            const int kb_total = tile_kblocks(P.prob[ti.p]);
            for (int kb0 = 0; kb0 < kb_total && ok; kb0 += CK) {
                if (!mbar_wait_bounded(&cempty[buf], bphase ^ 1u, P.spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * BN);
                const int kb1 = min(kb_total, kb0 + CK);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, P.spin, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = sdesc_sw128(smem_u32(sX + stage * S::kXBytes));
                    const uint64_t bdesc = sdesc_sw128(smem_u32(sY + stage * S::kYBytes));
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16_pair(d, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc,
                                       (kb > kb0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair_both(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair_both(&cfull[buf]);
                if (++buf == NB) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
        }
        umma_commit_pair_self(done);
        mbar_wait_bounded(done, 0, 1u << 26, err);
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2;
        const int q = warp & 3;
        const int c0 = (ew >> 2) * CW;
        const int lane_row = q * 32 + lane;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        for (int t = pair; t < ntiles && ok; t += npairs) {
            const TileInfo ti = pair_decode(P, t, rank);
            const GemmProblem& pr = P.prob[ti.p];
            const int kb_total = tile_kblocks(pr);
            float acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = 0.f;
            for (int kb0 = 0; kb0 < kb_total; kb0 += CK) {
                if (!mbar_wait_bounded(&cfull[buf], bphase, P.spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c0);
#pragma unroll
                for (int c = 0; c < CW; c += 32) {
                    uint32_t r0[16], r1[16];
                    tmem_ld16(taddr + (uint32_t)c, r0);
                    tmem_ld16(taddr + (uint32_t)(c + 16), r1);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[c + i] += __uint_as_float(r0[i]);
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[c + 16 + i] += __uint_as_float(r1[i]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(&cempty[buf], 0));
                if (++buf == NB) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
            if (!ok) break;
            const CUtensorMap* omap = pr.out_map >= 0 ? &P.maps[pr.out_map] : nullptr;
            epilogue_store<BN, false, CW>(pr, ti, lane_row, c0, acc, omap, sOut + ew * S::kStageOutBytes);
        }
        if (lane == 0) bulk_wait_all();
    }
    __syncthreads();
    tc_fence_before();
    cluster_sync_all();  // both CTAs done with TMEM; the leader's MMAs have completed
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, S::kTmemCols);
}

template <int BN, int STAGES, bool kSwap, bool kFp4>
constexpr size_t smem_bytes() {
    using S = Shape<BN, kSwap, kFp4>;
    return 1024 + (size_t)STAGES * (S::kStageBytes + S::kRawBytes) + (size_t)S::kEpiWarps * S::kStageOutBytes +
           S::kBarBytes + S::kLutBytes;
}

template <int BN, int STAGES, bool kSwap, bool kFp4 = false>
cudaError_t launch_impl(const TcParams& P, int grid, cudaStream_t s) {
    using S = Shape<BN, kSwap, kFp4>;
    constexpr size_t smem = smem_bytes<BN, STAGES, kSwap, kFp4>();
    static_assert(smem <= 232448, "shared memory");
    static_assert((3 * STAGES + 2 * S::kBufs + 1) * 8 + 4 <= S::kBarBytes, "barrier area");
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<BN, STAGES, kSwap, kFp4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_gemm_tc<BN, STAGES, kSwap, kFp4><<<grid, S::kThreads, smem, s>>>(P);
    return cudaGetLastError();
}

int g_num_sms = 0;

}  // namespace

int tc_num_sms() {
    if (g_num_sms == 0) {
        int dev = 0, n = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_num_sms = n > 0 ? n : 148;
    }
    return g_num_sms;
}

static void fill_params(TcParams& P, const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob,
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

// Dense tile counts (host side) and a grid no larger than the work.
template <int BN, bool kSwap>
static int dense_tile_count(const GemmProblem& pr) {
    using S = Shape<BN, kSwap>;
    return ((pr.m_rows + S::kActRows - 1) / S::kActRows) * (pr.n / S::kOutCols);
}

cudaError_t launch_gemm_tc(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                           const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s) {
    TcParams P;
    fill_params(P, maps, nmaps, probs, nprob, r, err, spin_limit);
    const int sms = tc_num_sms();
    int grid = sms;
    if (!probs[0].grouped) {
        long long tiles = 0;
        for (int i = 0; i < nprob; ++i) {
            P.dense_tiles[i] = bn == 256   ? dense_tile_count<256, false>(probs[i])
                               : bn == 128 ? dense_tile_count<128, false>(probs[i])
                                           : dense_tile_count<64, false>(probs[i]);
            tiles += P.dense_tiles[i];
        }
        if (tiles < grid) grid = (int)tiles;
        if (grid < 1) return cudaSuccess;
    }
    switch (bn) {
        case 256: return launch_impl<256, 4, false>(P, grid, s);
        case 128: return launch_impl<128, 6, false>(P, grid, s);
        case 64: return launch_impl<64, 8, false>(P, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_tc_pair(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob,
                                const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s) {
    constexpr int STAGES = 6;
    using S = PairShape;
    constexpr size_t smem = 1024 + (size_t)STAGES * S::kStageBytes + (size_t)S::kEpiWarps * S::kStageOutBytes + 256;
    static_assert(smem <= 232448, "shared memory");
    static_assert((2 * STAGES + 2 * S::kBufs + 1) * 8 + 4 <= 256, "barrier area");
    TcParams P;
    fill_params(P, maps, nmaps, probs, nprob, r, err, spin_limit);
    int pairs = tc_num_sms() / 2;
    if (!probs[0].grouped) {
        long long tiles = 0;
        for (int i = 0; i < nprob; ++i) {
            P.dense_tiles[i] = ((probs[i].m_rows + 255) / 256) * (probs[i].n / S::BN);
            tiles += P.dense_tiles[i];
        }
        if (tiles < pairs) pairs = (int)tiles;
        if (pairs < 1) return cudaSuccess;
    }
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tc_pair<STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(S::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_gemm_tc_pair<STAGES>, P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_gemm_tc_decode(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob,
                                  const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s) {
    TcParams P;
    fill_params(P, maps, nmaps, probs, nprob, r, err, spin_limit);
    int grid = tc_num_sms();
    if (!probs[0].grouped) {
        long long tiles = 0;
        for (int i = 0; i < nprob; ++i) {
            P.dense_tiles[i] = dense_tile_count<kDecodeTN, true>(probs[i]);
            tiles += P.dense_tiles[i];
        }
        if (tiles < grid) grid = (int)tiles;
        if (grid < 1) return cudaSuccess;
    }
    return launch_impl<kDecodeTN, 10, true>(P, grid, s);
}

// Grouped expert GEMMs with NVFP4 weights: weight-stationary tiles (128 weight
// rows on the MMA M side), bn = 32 tokens per tile (decode) or 128 (prefill).
cudaError_t launch_gemm_tc_nvfp4(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                                 const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s) {
    if (nprob != 1 || !probs[0].grouped || probs[0].nseg != 1 || !probs[0].wq_codes || !probs[0].wq_sf)
        return cudaErrorInvalidValue;
    TcParams P;
    fill_params(P, maps, nmaps, probs, nprob, r, err, spin_limit);
    const int grid = tc_num_sms();
    switch (bn) {
        case kDecodeTN: return launch_impl<kDecodeTN, 8, true, true>(P, grid, s);
        case 128: return launch_impl<128, 6, true, true>(P, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

// ---------------------------------------------------------------- self-test
__global__ void k_selftest_wait(int* err, unsigned spin) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, spin, err);  // nothing ever arrives
}

cudaError_t launch_selftest_wait(int* err, unsigned spin_limit, cudaStream_t s) {
    k_selftest_wait<<<1, 32, 0, s>>>(err, spin_limit);
    return cudaGetLastError();
}

}  // namespace lmoe
