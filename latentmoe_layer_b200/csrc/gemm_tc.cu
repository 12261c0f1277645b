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
// accumulated in chunks of 8 k-blocks (512) in a ring of TMEM buffers; the
// epilogue adds each chunk into fp32 registers, in order, while the MMA warp
// fills the next buffer. Partial sums stay small, so the tensor-core error
// no longer scales with the output, at the price of reading TMEM once per
// chunk instead of once per tile. (Chunks of 4 flip half as many roundings
// but, with only two 256-column buffers for the widest tiles, stall the MMA
// often enough to cost ~8% of a 16384-token Ultra forward; 8 costs ~1%.)
//
// Two tile shapes share the code:
//   kSwap = false  MMA M = 128 activation rows, N = BN weight rows.
//   kSwap = true   MMA M = 128 weight rows, N = BN tokens (decode batches,
//                  where each expert sees a handful of tokens: the weights sit
//                  on the 128-row side so no tensor-core work is padding).
// Every mbarrier wait is bounded; on running out the kernel records
// LMOE_ERR_TIMEOUT, drains its own TMA loads and MMAs, frees TMEM and returns.
#include "gemm_common.cuh"

namespace lmoe {
namespace {

// CG: shared-memory stages released per MMA commit. A tcgen05.commit holds the
// issuing thread's MMAs for about an MMA's latency (~230 cycles measured,
// against 130 for a 128 x 256 x 16 MMA), so one commit per 4-MMA stage costs
// ~30% of the MMA rate; a commit per two stages halves that but also halves the
// refill units of the ring, which costs more than it saves when K is long (the
// operands then stream from HBM for many k-blocks per tile). A second issuing
// thread hides much of it too (two threads committing every 4 MMAs: 156 cycles
// per MMA against 189.6 for one).
//
// NIS: MMA-issuing threads. With two (lane 0 of warp 1 and of an extra warp
// after the epilogue warps), issuer i takes the k-blocks of parity i into its
// own TMEM accumulator (buffer i), so each commits after every stage it used
// while the other's MMAs keep the tensor pipe busy. A chunk then spans 2 * ck
// k-blocks, ck in each accumulator, and the epilogue adds buffer 0, then
// buffer 1, into its registers: the partial sums have the single-issuer
// chunk's length. Needs an even k-block count in every tile (the parity then
// carries across tiles) and an even stage count (a stage keeps its issuer).
template <int BN, int STAGES, bool kSwap, int CG, int NIS>
__global__ void __launch_bounds__(Shape<BN, kSwap>::kThreads + (NIS - 1) * 32, 1)
    k_gemm_tc(const __grid_constant__ TcParams P) {
    using S = Shape<BN, kSwap>;
    constexpr int NB = S::kBufs, CK = S::kChunkKB, CW = S::kColsPerThread;
    static_assert(STAGES % CG == 0, "stage groups");
    static_assert(NIS == 1 || (NIS == 2 && NB == 2 && CG == 1 && STAGES % 2 == 0 && !kSwap), "two issuers");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((base_u32 + 1023u) & ~1023u) - base_u32);
    uint8_t* sX = smem;                                  // STAGES x kXBytes
    uint8_t* sY = smem + STAGES * S::kXBytes;            // STAGES x kYBytes
    uint8_t* sOut = sY + STAGES * S::kYBytes;            // kEpiWarps x kStageOutBytes
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + S::kEpiWarps * S::kStageOutBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* cfull = empty + STAGES;   // chunk accumulator ready (MMA -> epilogue)
    uint64_t* cempty = cfull + NB;      // chunk accumulator drained (epilogue -> MMA)
    uint64_t* done = cempty + NB;       // one per issuer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + NIS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kIssuer2Warp = S::kThreads / 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&cfull[b], 1);
            mbar_init(&cempty[b], S::kEpiWarps);
        }
        for (int i = 0; i < NIS; ++i) mbar_init(&done[i], 1);
        fence_mbar_init();
    }
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
                    // a group of CG stages is released by one commit: wait for it at the group's first stage
                    if (stage % CG == 0 && !mbar_wait_bounded(&empty[stage / CG], phase ^ 1u, P.spin, err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
                    if (!kSwap) {
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
    } else if (lane == 0 && (warp == 1 || (NIS == 2 && warp == kIssuer2Warp))) {
        // ------------------------------------------------ MMA issuer(s)
        constexpr uint32_t idesc_full = idesc_bf16_f32(128, BN);
        constexpr uint32_t idesc_half = idesc_bf16_f32(64, BN);
        const int ii = warp == 1 ? 0 : 1;  // this issuer's k-block parity (NIS == 2)
        int stage = NIS == 2 ? ii : 0, buf = NIS == 2 ? ii : 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, kSwap>(P, t);
            const int kb_total = tile_kblocks(P.prob[ti.p]);
            const int ck = (P.prob[ti.p].chunk_kb ? P.prob[ti.p].chunk_kb : CK) * NIS;
            // M = 64 puts D rows 16q..16q+15 in TMEM lanes 32q..32q+15 (q = lane quarter)
            const uint32_t idesc = ti.half ? idesc_half : idesc_full;
            for (int kb0 = 0; kb0 < kb_total && ok; kb0 += ck) {
                // next chunk accumulator must have been drained by the epilogue
                if (!mbar_wait_bounded(&cempty[buf], bphase ^ 1u, P.spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * BN);
                const int kb1 = min(kb_total, kb0 + ck);
                const int kbs = kb0 + (NIS == 2 ? ii : 0);
                for (int kb = kbs; kb < kb1; kb += NIS) {
                    if (!mbar_wait_bounded(&full[stage], phase, P.spin, err)) {
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
                                  (kb > kbs || kk > 0) ? 1u : 0u);
                    }
                    if (stage % CG == CG - 1) umma_commit(&empty[stage / CG]);
                    stage += NIS;
                    if (stage >= STAGES) {
                        stage -= STAGES;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&cfull[buf]);
                if (NIS == 2) {
                    bphase ^= 1u;  // this issuer's one buffer, once per chunk
                } else if (++buf == NB) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
        }
        // all MMAs issued by this thread have completed before TMEM is freed
        umma_commit(&done[ii]);
        mbar_wait_bounded(&done[ii], 0, 1u << 26, err);
    } else if (warp >= 2 && warp < 2 + S::kEpiWarps) {
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
            const int ck = pr.chunk_kb ? pr.chunk_kb : CK;
#if LMOE_PROMOTE_F64
            double accd[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) accd[i] = 0.0;
#else
            float acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = 0.f;
#endif
            // NIS == 2: chunks of 2 ck k-blocks, one partial in each buffer, added in buffer order
            const int nparts = NIS * ((kb_total + ck * NIS - 1) / (ck * NIS));
            for (int part = 0; part < nparts; ++part) {
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
// (Selected with LMOE_OPT_GEMM_PATH = 4. Slower than the single-SM tiles on
// this layer at its power-capped steady state: 25.7 against 23.4-23.9 ms per
// 16384-token Ultra forward, each path timed in its own process.)
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
    return dense_total(P);
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
        e = pr.expert_mod ? rc.x % pr.expert_mod : rc.x;
        wbase = e * pr.b_rows_per_expert;
    } else {
        p = dense_problem(P, t);
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
    ti.wrow0 = wbase + ti.col0 + (int)rank * 128;  // this CTA's half of the pair's B rows
    ti.wcol0 = wbase + ti.col0;                      // the output columns span both halves
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
            const int ck = P.prob[ti.p].chunk_kb ? P.prob[ti.p].chunk_kb : CK;
            for (int kb0 = 0; kb0 < kb_total && ok; kb0 += ck) {
                if (!mbar_wait_bounded(&cempty[buf], bphase ^ 1u, P.spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * BN);
                const int kb1 = min(kb_total, kb0 + ck);
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
            const int ck = pr.chunk_kb ? pr.chunk_kb : CK;
            float acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = 0.f;
            for (int kb0 = 0; kb0 < kb_total; kb0 += ck) {
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

template <int BN, int STAGES, bool kSwap>
constexpr size_t smem_bytes() {
    using S = Shape<BN, kSwap>;
    return 1024 + (size_t)STAGES * S::kStageBytes + (size_t)S::kEpiWarps * S::kStageOutBytes + 512;
}

template <int BN, int STAGES, bool kSwap, int CG = 1, int NIS = 1>
cudaError_t launch_impl(const TcParams& P, int grid, cudaStream_t s) {
    using S = Shape<BN, kSwap>;
    constexpr size_t smem = smem_bytes<BN, STAGES, kSwap>();
    static_assert(smem <= 232448, "shared memory");
    static_assert((2 * STAGES + 2 * S::kBufs + NIS) * 8 + 4 <= 512, "barrier area");
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<BN, STAGES, kSwap, CG, NIS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_gemm_tc<BN, STAGES, kSwap, CG, NIS><<<grid, S::kThreads + (NIS - 1) * 32, smem, s>>>(P);
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

// Dense tile counts (host side) and a grid no larger than the work.
template <int BN, bool kSwap>
static int dense_tile_count(const GemmProblem& pr) {
    using S = Shape<BN, kSwap>;
    return ((pr.m_rows + S::kActRows - 1) / S::kActRows) * (pr.n / S::kOutCols);
}

cudaError_t launch_gemm_tc(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                           const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s) {
    if (nprob < 1 || nprob > kMaxProb || nmaps > kMaxMaps) return cudaErrorInvalidValue;
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
    bool short_k = true, even_k = true;
    for (int i = 0; i < nprob; ++i) {
        const int kbt = probs[i].kdim[0] / kBK + (probs[i].nseg > 1 ? probs[i].kdim[1] / kBK : 0);
        short_k = short_k && kbt <= 32;
        even_k = even_k && kbt % 2 == 0;
    }
    // short tiles (at most 32 k-blocks: the expert up GEMM at L = 2048): two MMA issuers, or one
    // commit per two stages when a tile's k-block count is odd. Long-K tiles keep one issuer
    // with a commit per stage: both other forms cost them 3-10% (with two issuers interleaved in
    // the tensor pipe each stage is released later; stage pairs halve the ring's refill units),
    // which matters where the operands stream from HBM.
    if (short_k && bn == 256) {
        if (even_k) return launch_impl<256, 4, false, 1, 2>(P, grid, s);
        return launch_impl<256, 4, false, 2>(P, grid, s);
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
    if (nprob < 1 || nprob > kMaxProb || nmaps > kMaxMaps) return cudaErrorInvalidValue;
    constexpr int STAGES = 6;
    using S = PairShape;
    constexpr size_t smem = 1024 + (size_t)STAGES * S::kStageBytes + (size_t)S::kEpiWarps * S::kStageOutBytes + 256;
    static_assert(smem <= 232448, "shared memory");
    static_assert((2 * STAGES + 2 * S::kBufs + 1) * 8 + 4 <= 512, "barrier area");
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

cudaError_t launch_gemm_tc_decode(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                                  const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s) {
    if (nprob < 1 || nprob > kMaxProb || nmaps > kMaxMaps) return cudaErrorInvalidValue;
    if (bn != kDecodeTN && (bn != 64 || probs[0].grouped)) return cudaErrorInvalidValue;
    TcParams P;
    fill_params(P, maps, nmaps, probs, nprob, r, err, spin_limit);
    int grid = tc_num_sms();
    if (!probs[0].grouped) {
        long long tiles = 0;
        for (int i = 0; i < nprob; ++i) {
            P.dense_tiles[i] = bn == 64 ? dense_tile_count<64, true>(probs[i]) : dense_tile_count<kDecodeTN, true>(probs[i]);
            tiles += P.dense_tiles[i];
        }
        if (tiles < grid) grid = (int)tiles;
        if (grid < 1) return cudaSuccess;
    }
    // 64-token tiles: every token of a short batch in one tile, one pass over each weight tile
    if (bn == 64) return launch_impl<64, 8, true>(P, grid, s);
    return launch_impl<kDecodeTN, 10, true>(P, grid, s);
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
