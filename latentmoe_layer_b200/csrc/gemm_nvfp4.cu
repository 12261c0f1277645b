// gemm_nvfp4.cu -- grouped expert GEMMs whose weights are NVFP4.
//
// The routed experts' up and down projections are the NVFP4 layers of the
// pages' model ("Nemotron 3 Ultra 架构 QA", Q1.3 and Q8.1). Weights are E2M1
// codes with one E4M3 scale per 16 along K and one fp32 scale per matrix
// (layout in latentmoe.h), activations stay bf16: each 128 x 64 weight tile is
// expanded exactly into bf16 in shared memory and multiplied on the tensor
// cores (tcgen05.mma kind::f16, fp32 accumulation in TMEM), so the arithmetic
// is that of the bf16 path applied to the dequantised weights.
//
// Weight-stationary tiles: MMA M = 128 weight rows, N = BN tokens of one
// expert (BN = 32 at decode sizes, 128 otherwise). A ring of shared-memory
// stages, each holding KB k-blocks of 64 (token tiles by TMA with the 128-byte
// swizzle, codes and scales by bulk copy), feeds dequantisation warps that
// write the bf16 weight rows into TMEM slots; the MMA reads A from TMEM and B
// (tokens) from shared memory. Every barrier wait and commit sits on the path
// of a 32-token tile, whose tensor-core work per k-block is short, so a stage
// carries several k-blocks to spread that cost.
// Roles: warp 0 producer, warp 1 MMA issuer and TMEM owner, then the epilogue
// warps (TMEM chunk drains, as in the bf16 kernel), then the dequantisation
// warps.
#include "gemm_common.cuh"

namespace lmoe {
namespace {

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

// The same conversion with the block scale folded into the byte tables: t
// holds, for one E4M3 scale s, the high bytes (t.x: magnitudes 0..3, t.y:
// 4..7) and low bytes (t.z, t.w) of the bf16 values of s * {0, 0.5, 1, 1.5,
// 2, 3, 4, 6}. Those products are exact in bf16 (at most 6 significant bits),
// so the result equals e2m1x8_to_bf16(c, s) bit for bit, signs and zeros
// included, without the four multiplies.
__device__ __forceinline__ uint4 e2m1x8_to_bf16_scaled(uint32_t c, const uint4& t) {
    const uint32_t mag = c & 0x77777777u;
    const uint32_t d = c << 4;
    const uint32_t mhi = mag >> 16;
    const uint32_t h0 = prmt(t.x, t.y, mag) ^ (prmt(d, c, 0x5140u) & 0x80808080u);
    const uint32_t l0 = prmt(t.z, t.w, mag);
    const uint32_t h1 = prmt(t.x, t.y, mhi) ^ (prmt(d, c, 0x7362u) & 0x80808080u);
    const uint32_t l1 = prmt(t.z, t.w, mhi);
    uint4 o;
    o.x = prmt(l0, h0, 0x5140u);
    o.y = prmt(l0, h0, 0x7362u);
    o.z = prmt(l1, h1, 0x5140u);
    o.w = prmt(l1, h1, 0x7362u);
    return o;
}

// Byte tables of e2m1x8_to_bf16_scaled for the E4M3 scale byte b: the bf16
// products s * m of the eight magnitudes m, signs included (0 * s is -0 for a
// negative s). A code's sign bit flips its product's sign (xor), which is
// what the multiply by s gives for every code, -0 and negative scales
// included.
__device__ __forceinline__ uint4 e4m3_scaled_table(uint32_t b) {
    const uint32_t s2 = e4m3_to_bf16x2(b);
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        constexpr uint32_t kMag[8] = {0x0000u, 0x3F00u, 0x3F80u, 0x3FC0u, 0x4000u, 0x4040u, 0x4080u, 0x40C0u};
        const uint32_t v = mul_bf16x2(kMag[j] | (kMag[j] << 16), s2) & 0xFFFFu;
        hi[j] = v >> 8;
        lo[j] = v & 0xFFu;
    }
    uint4 t;
    t.x = hi[0] | (hi[1] << 8) | (hi[2] << 16) | (hi[3] << 24);
    t.y = hi[4] | (hi[5] << 8) | (hi[6] << 16) | (hi[7] << 24);
    t.z = lo[0] | (lo[1] << 8) | (lo[2] << 16) | (lo[3] << 24);
    t.w = lo[4] | (lo[5] << 8) | (lo[6] << 16) | (lo[7] << 24);
    return t;
}

// ------------------------------------------------------------------------------
// The dequantised weights live in TMEM: the tensor core takes its A operand
// (128 weight rows x K) from TMEM, so the bf16 weight tile never passes through
// shared memory (with it in shared memory, the codes read, the bf16 tile
// written and read back, and the copies made ~49 KB of shared-memory traffic
// per k-block; now ~17 KB). Each
// dequantisation thread owns one weight row = one TMEM lane: it reads the row's
// 32 code bytes and 4 scale bytes and stores 32 columns (64 bf16) with
// tcgen05.st. A warp may only touch its own TMEM lane quarter, so the
// dequantisation warps form G groups of four (one per quarter); every group
// works on every stage, group g converting the stage's k-blocks j with
// j % G == g, so a stage's conversion is spread over all G x 4 warps (one
// group per stage made each stage a long serial chain per thread).
// TMEM columns: [0, NB * NI * BN) accumulator chunk buffers (one accumulator
// per MMA issuer), then AS slots of KB bf16 weight tiles (32 columns each).
// The shared-memory ring (codes, scales, token tiles) is deeper than the slot
// ring, so copies run far ahead of the conversions: before it overwrites slot
// c % AS, the conversion of stage c waits for the MMA of stage c - AS, the
// slot's last reader, on that stage's `empty` barrier (no barrier is added to
// the MMA's path).
// Template parameters: BN tokens per tile, STAGES shared-memory stages of KB
// k-blocks, G dequantisation warp groups, AS TMEM weight slots, NB accumulator
// chunk buffers, NI MMA-issuing warps (issuer i takes the k-blocks j % NI == i
// of a stage), SL conversion through per-scale byte tables.
// At decode sizes a 128 x 32 x 16 MMA occupies the tensor core ~48 cycles
// whatever its N (up to 64), so a stage of four k-blocks has ~780 cycles of
// tensor time; the measured stage takes ~2000, spent on the conversion
// (~1300 cycles of ALU work per warp), the MMA issuer's barrier round trips
// and its slower issue next to the converting warps.
template <int BN, int STAGES, int KB, int G, int AS, int NB, int NI, bool SL>
struct Fp4TmShape {
    using T = Shape<BN, true>;
    static constexpr int kTokBytes = BN * kBK * 2;
    static constexpr int kOffCodes = KB * kTokBytes;
    static constexpr int kOffSf = kOffCodes + KB * 4096;
    static constexpr int kStageBytes = (kOffSf + KB * 512 + 1023) & ~1023;
    static constexpr int kTxBytes = KB * (kTokBytes + 4096 + 512);
    static constexpr int kBufs = NB;                 // accumulator chunk buffers, one accumulator per MMA issuer
    static constexpr uint32_t kColA = NB * NI * BN;  // first column of the weight tiles
    static constexpr int kDeqWarps = 4 * G;
    static constexpr int kThreads = 32 * (1 + NI + T::kEpiWarps + kDeqWarps);
    static constexpr int kBarBytes = 1024;
    static constexpr int kBars = 3 * STAGES + 2 * kBufs + 1;
    static constexpr int kLutBytes = SL ? 256 * 16 : 256 * 4;  // per-scale byte tables, or bf16 scales
    static constexpr size_t kSmem = 1024 + (size_t)STAGES * kStageBytes + kBarBytes + kLutBytes;
    static_assert(kColA + AS * KB * 32 <= 512 && AS <= STAGES, "accumulators and weight tiles fit TMEM");
    static_assert(kBars * 8 + 4 <= kBarBytes, "barrier area");
    static_assert(KB % G == 0 && KB % NI == 0 && T::kChunkKB % KB == 0 && (NI == 1 || NI == 2), "groups / chunks");
    static_assert(kSmem <= 232448 && STAGES <= 32, "shared memory");
};

template <int BN, int STAGES, int KB, int G, int AS, int NB, int NI, bool SL>
__global__ void __launch_bounds__(Fp4TmShape<BN, STAGES, KB, G, AS, NB, NI, SL>::kThreads, 1)
    k_gemm_nvfp4_tm(const __grid_constant__ TcParams P) {
    using F = Fp4TmShape<BN, STAGES, KB, G, AS, NB, NI, SL>;
    using S = typename F::T;
    constexpr int CK = S::kChunkKB, CW = S::kColsPerThread;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((base_u32 + 1023u) & ~1023u) - base_u32);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * F::kStageBytes);  // copies landed (producer)
    uint64_t* deq = full + STAGES;         // weight tiles stored in TMEM (dequantisation -> MMA)
    uint64_t* empty = deq + STAGES;        // MMA done with the stage (MMA -> producer)
    uint64_t* cfull = empty + STAGES;      // chunk accumulator ready (MMA -> epilogue)
    uint64_t* cempty = cfull + NB;         // chunk accumulator drained (epilogue -> MMA)
    uint64_t* done = cempty + NB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    uint32_t* scale_lut = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(full) + F::kBarBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&deq[s], 4 * G);
            mbar_init(&empty[s], NI);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&cfull[b], NI);
            mbar_init(&cempty[b], S::kEpiWarps);
        }
        mbar_init(done, NI);
        fence_mbar_init();
    }
    const int dq0 = 1 + NI + S::kEpiWarps;  // first dequantisation warp
    if (warp >= dq0)
        for (int b = threadIdx.x - 32 * dq0; b < 256; b += 32 * F::kDeqWarps) {
            if constexpr (SL)
                reinterpret_cast<uint4*>(scale_lut)[b] = e4m3_scaled_table((uint32_t)b);
            else
                scale_lut[b] = e4m3_to_bf16x2((uint32_t)b);
        }
    if (warp == 0 && lane == 0)
        for (int i = 0; i < P.nmaps; ++i) prefetch_tmap(&P.maps[i]);
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ntiles = total_tiles<BN, true>(P);
    const int kb_n = P.prob[0].kdim[0] / kBK;   // a multiple of KB (K is a multiple of 128)
    const unsigned spin = P.spin;
    int* err = P.err;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ producer
        const CUtensorMap* amap = &P.maps[P.prob[0].a_map[0]];
        const uint8_t* codes_g = P.prob[0].wq_codes;
        const uint8_t* sf_g = P.prob[0].wq_sf;
        uint32_t c = 0, issued = 0, issued_par = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, true>(P, t);
            const long long tile0 = (long long)(ti.wrow0 >> 7) * kb_n;
            for (int kb = 0; kb < kb_n; kb += KB, ++c) {
                const int s = (int)(c % STAGES);
                const uint32_t ph = (c / STAGES) & 1u;
                if (!mbar_wait_bounded(&empty[s], ph ^ 1u, spin, err)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + s * F::kStageBytes;
                mbar_arrive_expect_tx(&full[s], F::kTxBytes);
#pragma unroll
                for (int j = 0; j < KB; ++j) tma_load_2d(st + j * F::kTokBytes, amap, &full[s], (kb + j) * kBK, ti.row0);
                bulk_load(st + F::kOffCodes, codes_g + (tile0 + kb) * 4096, KB * 4096, &full[s]);
                bulk_load(st + F::kOffSf, sf_g + (tile0 + kb) * 512, KB * 512, &full[s]);
                issued |= 1u << s;
                issued_par = (issued_par & ~(1u << s)) | (ph << s);
            }
        }
        for (int s = 0; s < STAGES; ++s)
            if ((issued >> s) & 1u) mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, 1u << 26, err);
    } else if (warp >= 1 && warp <= NI && lane == 0) {
        // ------------------------------------------------ MMA issuers: issuer i takes the k-blocks
        // j % NI == i of every stage into its own accumulator of the chunk buffer
        constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
        const int iss = warp - 1;
        uint32_t c = 0, bphase = 0;
        int buf = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            for (int kb0 = 0; kb0 < kb_n && ok; kb0 += CK) {
                if (!mbar_wait_bounded(&cempty[buf], bphase ^ 1u, spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)((buf * NI + iss) * BN);
                const int kb1 = min(kb_n, kb0 + CK);
                for (int kb = kb0; kb < kb1; kb += KB, ++c) {
                    const int s = (int)(c % STAGES);
                    // deq[s] completes only after every dequantisation warp has seen full[s]
                    // complete, so the stage's copies (the token tiles included) have landed
                    if (!mbar_wait_bounded(&deq[s], (c / STAGES) & 1u, spin, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* st = smem + s * F::kStageBytes;
#pragma unroll
                    for (int jj = 0; jj < KB / NI; ++jj) {
                        const int j = jj * NI + iss;
                        const uint32_t a = tmem_base + F::kColA + (uint32_t)(((c % AS) * KB + j) * 32);
                        const uint64_t bdesc = sdesc_sw128(smem_u32(st + j * F::kTokBytes));
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)
                            umma_bf16_tmem_a(d, a + (uint32_t)(kk * 8), bdesc + (uint64_t)(kk * 2), idesc,
                                             (kb + j - iss > kb0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&cfull[buf]);
                if (++buf == NB) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
        }
        umma_commit(done);
        mbar_wait_bounded(done, 0, 1u << 26, err);
    } else if (warp >= dq0) {
        // ------------------------------------------------ dequantisation into TMEM
        const int dw = warp - dq0;
        const int grp = dw >> 2;
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int row = q * 32 + lane;          // weight row = TMEM lane
        uint32_t c = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < kb_n; kb += KB, ++c) {
                const int s = (int)(c % STAGES);
                const uint32_t slot = c % AS;
                if (c >= (uint32_t)AS) {  // the slot's last reader, the MMA of stage c - AS, has completed
                    const uint32_t p = c - AS;
                    if (!mbar_wait_bounded(&empty[p % STAGES], (p / STAGES) & 1u, spin, err)) {
                        ok = false;
                        break;
                    }
                }
                if (!mbar_wait_bounded(&full[s], (c / STAGES) & 1u, spin, err)) {
                    ok = false;
                    break;
                }
                const uint8_t* st = smem + s * F::kStageBytes;
                // every shared-memory load of this warp's k-blocks of the stage first (codes and
                // scale bytes), then the conversions and TMEM stores
                constexpr int NJ = KB / G;
                uint4 cw[NJ][2];
                uint32_t sbw[NJ];
#pragma unroll
                for (int u = 0; u < NJ; ++u) {
                    const int j = grp + u * G;
                    const uint8_t* codes = st + F::kOffCodes + j * 4096 + row * 32;
                    cw[u][0] = ld_shared_v4(codes);
                    cw[u][1] = ld_shared_v4(codes + 16);
                    sbw[u] = ld_shared_u32(st + F::kOffSf + j * 512 + row * 4);
                }
#pragma unroll
                for (int u = 0; u < NJ; ++u) {
                    const int j = grp + u * G;
                    const uint4 c0 = cw[u][0], c1 = cw[u][1];
                    const uint32_t sb = sbw[u];
                    uint4 os[8];
                    if constexpr (SL) {
                        const uint4* tl = reinterpret_cast<const uint4*>(scale_lut);
                        const uint4 t0 = ld_shared_v4(tl + (sb & 0xFFu)), t1 = ld_shared_v4(tl + ((sb >> 8) & 0xFFu));
                        const uint4 t2 = ld_shared_v4(tl + ((sb >> 16) & 0xFFu)), t3 = ld_shared_v4(tl + (sb >> 24));
                        os[0] = e2m1x8_to_bf16_scaled(c0.x, t0), os[1] = e2m1x8_to_bf16_scaled(c0.y, t0);
                        os[2] = e2m1x8_to_bf16_scaled(c0.z, t1), os[3] = e2m1x8_to_bf16_scaled(c0.w, t1);
                        os[4] = e2m1x8_to_bf16_scaled(c1.x, t2), os[5] = e2m1x8_to_bf16_scaled(c1.y, t2);
                        os[6] = e2m1x8_to_bf16_scaled(c1.z, t3), os[7] = e2m1x8_to_bf16_scaled(c1.w, t3);
                    } else {
                        const uint32_t s0 = ld_shared_u32(scale_lut + (sb & 0xFFu));
                        const uint32_t s1 = ld_shared_u32(scale_lut + ((sb >> 8) & 0xFFu));
                        const uint32_t s2 = ld_shared_u32(scale_lut + ((sb >> 16) & 0xFFu));
                        const uint32_t s3 = ld_shared_u32(scale_lut + (sb >> 24));
                        os[0] = e2m1x8_to_bf16(c0.x, s0), os[1] = e2m1x8_to_bf16(c0.y, s0);
                        os[2] = e2m1x8_to_bf16(c0.z, s1), os[3] = e2m1x8_to_bf16(c0.w, s1);
                        os[4] = e2m1x8_to_bf16(c1.x, s2), os[5] = e2m1x8_to_bf16(c1.y, s2);
                        os[6] = e2m1x8_to_bf16(c1.z, s3), os[7] = e2m1x8_to_bf16(c1.w, s3);
                    }
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        w[4 * i] = os[i].x;
                        w[4 * i + 1] = os[i].y;
                        w[4 * i + 2] = os[i].z;
                        w[4 * i + 3] = os[i].w;
                    }
                    tmem_st32(tmem_base + ((uint32_t)(q * 32) << 16) + F::kColA + (slot * KB + j) * 32u, w);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&deq[s]);
            }
        }
    } else if (warp > NI) {
        // ------------------------------------------------ epilogue (as the bf16 swap tiles)
        const GemmProblem& pr = P.prob[0];
        const int ew = warp - 1 - NI;
        const int q = warp & 3;
        const int c0 = (ew >> 2) * CW;
        const int lane_row = q * 32 + lane;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<BN, true>(P, t);
            float acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = 0.f;
            for (int kb0 = 0; kb0 < kb_n; kb0 += CK) {
                if (!mbar_wait_bounded(&cfull[buf], bphase, spin, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * NI * BN + c0);
#pragma unroll
                for (int na = 0; na < NI; ++na) {
#pragma unroll
                    for (int cc = 0; cc < CW; cc += 32) {
                        uint32_t r0[16], r1[16];
                        tmem_ld16(taddr + (uint32_t)(na * BN + cc), r0);
                        if (cc + 16 < CW) tmem_ld16(taddr + (uint32_t)(na * BN + cc + 16), r1);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc[cc + i] += __uint_as_float(r0[i]);
                        if (cc + 16 < CW) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) acc[cc + 16 + i] += __uint_as_float(r1[i]);
                        }
                    }
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
            epilogue_store<BN, true, CW>(pr, ti, lane_row, c0, acc, nullptr, nullptr);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <int BN, int STAGES, int KB, int G, int AS, int NB, int NI, bool SL>
cudaError_t launch_nvfp4_tm(const TcParams& P, int grid, cudaStream_t s) {
    using F = Fp4TmShape<BN, STAGES, KB, G, AS, NB, NI, SL>;
    cudaError_t e = cudaFuncSetAttribute(k_gemm_nvfp4_tm<BN, STAGES, KB, G, AS, NB, NI, SL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)F::kSmem);
    if (e != cudaSuccess) return e;
    k_gemm_nvfp4_tm<BN, STAGES, KB, G, AS, NB, NI, SL><<<grid, F::kThreads, F::kSmem, s>>>(P);
    return cudaGetLastError();
}

}  // namespace

// Grouped expert GEMMs with NVFP4 weights, bn = 32 tokens per tile (decode) or 128.
cudaError_t launch_gemm_tc_nvfp4(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                                 const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s) {
    if (nprob != 1 || !probs[0].grouped || probs[0].nseg != 1 || !probs[0].wq_codes || !probs[0].wq_sf)
        return cudaErrorInvalidValue;
    TcParams P;
    fill_params(P, maps, nmaps, probs, nprob, r, err, spin_limit);
    const int grid = tc_num_sms();
    switch (bn) {
        case kDecodeTN:
            // four k-blocks per stage where K allows (a multiple of 256), else two; the decode
            // tiles read the conversion's per-scale byte tables
            // (stages of four: two MMA issuers, each taking two k-blocks of every stage into its own
            // accumulator, 2.6% faster than one issuer for all four)
            if ((probs[0].kdim[0] / kBK) % 4 == 0) return launch_nvfp4_tm<kDecodeTN, 5, 4, 2, 2, 4, 2, true>(P, grid, s);
            return launch_nvfp4_tm<kDecodeTN, 8, 2, 2, 4, 8, 1, true>(P, grid, s);
        case 128: return launch_nvfp4_tm<128, 5, 2, 1, 4, 2, 1, false>(P, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lmoe
