// api.cu -- the C ABI of the LatentMoE layer forward (include/latentmoe.h):
// argument validation, workspace carving, TMA descriptor encoding and the
// launch sequence. Every launch goes to the caller's stream or to the handle's
// second stream, forked from and joined back into the caller's stream within
// the call; nothing here synchronises except the diagnostic entry points that
// say so.
//
// Launch sequence of latentmoe_forward (bf16 mode):
//   1 input GEMM        logits = x W_r^T (fp32), z = x W_fc1^T (fp32 when z is
//                       re-rounded) and a_s = relu2(x W_su^T) (bf16): one launch,
//                       three problems (the router in a launch of its own where
//                       the tile shapes differ)
//   -- fork: on the second stream, steps 2-4; on the caller's stream, step 5
//   2 select            sigmoid, +bias, grouped top-k, weights; near-edge flags
//   3 fp64 re-check     flagged tokens: exact-product fp64 logits and decision
//   4 permutation       counts, offsets, tile prefixes, perm, slot, row weights
//   5 exact re-rounding z = bf16 of the exact sum for the elements near a
//                       rounding midpoint; the same for the large a_s
//   -- join
//   6 gather            z rows into expert order
//   7 expert up GEMM    a = relu2(z_e W_up[e]^T) (bf16), grouped by expert,
//                       then the exact re-rounding of its large activations
//   8 expert down GEMM  o = w * (a_e W_down[e]^T) (fp32), grouped by expert
//   9 combine           comb[t] = bf16(sum over the token's k rows, ascending id)
//  10 output GEMM       y = comb W_fc2^T + a_s W_sd^T (fp32), one K-concatenated GEMM
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <new>

#include "handle.h"
#include "lmoe_internal.h"

using namespace lmoe;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode = nullptr;

bool get_encoder() {
    if (g_encode) return true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return false;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return true;
}

// Row-major [rows, cols] (cols contiguous), 128-byte-swizzled boxes of
// 128 bytes x box_rows rows.
bool encode_2d(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows, bool f32) {
    const int esz = f32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * esz};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// bf16 operand tiles: 64 columns (one 128-byte swizzle row) x box_rows rows.
bool encode_bf16(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows) {
    return encode_2d(m, base, rows, cols, box_rows, false);
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

bool plan_of(const lmoe_config& c, int T, Plan& p) {
    const size_t E = c.num_experts, k = c.top_k, H = c.hidden, L = c.latent, I = c.expert_inter,
                 Is = c.shared_inter;
    const size_t A = (size_t)T * k;
    const size_t act = c.mode == LMOE_MODE_BF16 ? 2 : 4;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += al256(bytes);
        return o;
    };
    p.T = T;
    p.A = (int)A;
    p.nblk = (T + 255) / 256;
    p.stats = take(sizeof(WsStats));
    p.logits = take((size_t)T * E * 4);
    p.logits64 = take((size_t)T * E * 8);
    p.flaglist = take((size_t)T * 4);
    p.idx = take(A * 4);
    p.wgt = take(A * 4);
    p.counts = take(E * 4);
    p.offsets = take((E + 1) * 4);
    p.pfx128 = take((E + 1) * 4);
    p.pfx64 = take((E + 1) * 4);
    p.pfxdec = take((E + 1) * 4);
    p.pfx256 = take((E + 1) * 4);
    p.rec32 = take((A / 32 + E) * 16);
    p.rec64 = take((A / 64 + E) * 16);
    p.rec128 = take((A / 128 + E) * 16);
    p.rec256 = take((A / 256 + E) * 16);
    p.blockcounts = take((size_t)p.nblk * E * 4);
    p.perm = take(A * 4);
    p.slot = take(A * 4);
    p.wperm = take(A * 4);
    p.xbf = (c.mode == LMOE_MODE_BF16 && c.x_dtype == LMOE_FP32) ? take((size_t)T * H * 2) : 0;
    p.xnorm = c.x_dtype == LMOE_BF16 ? take((size_t)T * H * 2) : 0;  // latentmoe_forward_block
    p.z = take((size_t)T * L * act);
    p.zperm = take(A * L * act);
    p.aperm = take(A * I * act);
    p.o = take(A * L * 4);
    p.comb = take((size_t)T * L * act);
    p.as = take((size_t)T * Is * act);
    // near-midpoint list of the exact z re-rounding, room for every element of z: it
    // shares the expert activation buffer (free until the expert up GEMM) when that
    // is large enough (top_k * I >= 4 L), else it has its own
    p.zlist = (A * I * act >= (size_t)T * L * 8) ? p.aperm : take((size_t)T * L * 8);
    // activation re-rounding list (the shared expert's, then the experts': one at a time), room
    // for every activation the flag test can list at any accepted tau (~0.5% of the larger set;
    // ~0.02% is listed at the default tau on the synthetic workloads)
    p.alist_cap = (int)std::min<size_t>(act_list_room(std::max((size_t)T * Is, A * I)), 0x7FFFFFFF);
    p.alist = take((size_t)p.alist_cap * 8);
    p.zrowtab = take((size_t)T * ((L + 2047) / 2048) * 16);  // one {row, first, entries} per 2048-column segment
    p.total = off;
    return true;
}

lmoe_status check_config(const lmoe_config* c) {
    if (!c) return LMOE_ERR_INVALID_ARG;
    if (c->hidden <= 0 || c->latent <= 0 || c->num_experts <= 0 || c->top_k <= 0 || c->n_group <= 0 ||
        c->topk_group <= 0 || c->expert_inter <= 0 || c->shared_inter <= 0 || c->max_tokens <= 0)
        return LMOE_ERR_INVALID_ARG;
    if (c->hidden % 64 || c->latent % 64 || c->expert_inter % 64 || c->shared_inter % 64)
        return LMOE_ERR_INVALID_ARG;
    if (c->num_experts % c->n_group || c->topk_group > c->n_group) return LMOE_ERR_INVALID_ARG;
    if (c->top_k > c->topk_group * (c->num_experts / c->n_group)) return LMOE_ERR_INVALID_ARG;
    if (!(c->routed_scaling_factor == c->routed_scaling_factor) || isinf(c->routed_scaling_factor))
        return LMOE_ERR_INVALID_ARG;
    if ((c->x_dtype != LMOE_BF16 && c->x_dtype != LMOE_FP32) ||
        (c->mode != LMOE_MODE_BF16 && c->mode != LMOE_MODE_FP32))
        return LMOE_ERR_INVALID_ARG;
    if (c->expert_format != LMOE_EXPERTS_BF16 && c->expert_format != LMOE_EXPERTS_NVFP4) return LMOE_ERR_INVALID_ARG;
    if (c->expert_format == LMOE_EXPERTS_NVFP4 &&
        (c->mode != LMOE_MODE_BF16 || c->expert_inter % 128 || c->latent % 128))
        return LMOE_ERR_UNSUPPORTED;  // weight tiles of 128 rows; tensor-core path only
    if (c->local_experts < 0 || c->expert_base < 0 || c->local_experts > c->num_experts ||
        (long long)c->expert_base + (c->local_experts ? c->local_experts : c->num_experts) > c->num_experts)
        return LMOE_ERR_INVALID_ARG;
    if (c->num_experts > kMaxE || c->n_group > kMaxG || c->top_k > kMaxK) return LMOE_ERR_UNSUPPORTED;
    if (c->n_group > 1 && c->num_experts / c->n_group < 2) return LMOE_ERR_UNSUPPORTED;
    if (c->hidden > 16384) return LMOE_ERR_UNSUPPORTED;  // fp64 router stages one x row in shared memory
    if ((long long)c->max_tokens * c->top_k > (1LL << 30)) return LMOE_ERR_UNSUPPORTED;
    if ((long long)c->max_tokens * c->latent > 0x7FFFFFFFLL) return LMOE_ERR_UNSUPPORTED;  // z element list index
    return LMOE_OK;
}

lmoe_status check_weights(const lmoe_config& c, const lmoe_weights* w) {
    if (!w) return LMOE_ERR_INVALID_ARG;
    const void* ps[8] = {w->router_w, w->e_bias, w->fc1_w, w->fc2_w, w->up_w, w->down_w, w->shared_up_w,
                         w->shared_down_w};
    for (const void* p : ps)
        if (!p || !aligned(p, 16)) return LMOE_ERR_INVALID_ARG;
    if (c.expert_format == LMOE_EXPERTS_NVFP4) {
        if (!w->up_sf || !w->down_sf || !aligned(w->up_sf, 16) || !aligned(w->down_sf, 16)) return LMOE_ERR_INVALID_ARG;
        if (!w->up_gs || !w->down_gs || !aligned(w->up_gs, 4) || !aligned(w->down_gs, 4)) return LMOE_ERR_INVALID_ARG;
    }
    return LMOE_OK;
}

// Tensor-core tile choice for a set of problem widths.
#ifndef LMOE_MAX_BN
#define LMOE_MAX_BN 256
#endif
int pick_bn(const int* ns, int cnt) {
    for (int bn : {256, 128, 64}) {
        if (bn > LMOE_MAX_BN) continue;
        bool ok = true;
        for (int i = 0; i < cnt; ++i) ok = ok && ns[i] % bn == 0;
        if (ok) return bn;
    }
    return 0;
}

// Tokens per tile of a swap-AB (decode) launch: 64 where every problem is dense
// and 64-token tiles take fewer waves over the SMs than 32-token ones (each
// token tile streams the same weight tiles again; at equal waves more tiles in a
// wave keep more SMs streaming), else kDecodeTN.
int decode_bn(const GemmProblem* probs, int nprob, int sms) {
    long long t32 = 0, t64 = 0;
    for (int i = 0; i < nprob; ++i) {
        if (probs[i].grouped) return kDecodeTN;
        t32 += (long long)((probs[i].m_rows + kDecodeTN - 1) / kDecodeTN) * (probs[i].n / 128);
        t64 += (long long)((probs[i].m_rows + 63) / 64) * (probs[i].n / 128);
    }
    return (t64 + sms - 1) / sms < (t32 + sms - 1) / sms ? 64 : kDecodeTN;
}

struct Ctx {
    lmoe_handle* h;
    const Plan* p;
    char* ws;
    cudaStream_t s;
    DeviceRouting r;
    int* err;
    WsStats* st;          // the call's statistics block
    int2* alist;          // activation re-rounding list and its room
    int alist_cap;
    bool decode;  // swap-AB tiles for the expert GEMMs and the dense GEMMs
    bool simt;
};

// Runs one GEMM launch (1 or 2 problems sharing the tile path). Operands are
// given as (pointer, rows, K) and encoded here for the chosen tile shape.
struct Operand {
    const void* ptr;
    long long rows;
};

cudaError_t run_gemm(Ctx& c, GemmProblem* probs, int nprob, const Operand (*a)[2], const Operand (*b)[2],
                     bool a_f32_simt) {
    if (c.simt) return launch_gemm_simt(probs, nprob, a_f32_simt, c.r, c.p->A, c.s);
    if (nprob < 1 || nprob > kMaxProblems) return cudaErrorInvalidValue;
    int ns[kMaxProblems];
    bool swap = c.decode;
    for (int i = 0; i < nprob; ++i) {
        ns[i] = probs[i].n;
        swap = swap && probs[i].n % 128 == 0;
    }
    const int bn = swap ? decode_bn(probs, nprob, c.h->num_sms) : pick_bn(ns, nprob);
    if (bn == 0) return cudaErrorInvalidValue;
    // 256 x 256 tiles on 2-SM pairs (option 4): each CTA of the pair loads 128 rows of B
    const bool pair = !swap && bn == 256 && c.h->gemm_path == 4;
    CUtensorMap maps[kMaxTensorMaps];
    int nm = 0;
    for (int i = 0; i < nprob; ++i)
        for (int sg = 0; sg < probs[i].nseg; ++sg) {
            const int K = probs[i].kdim[sg];
            // problems that read the same activation matrix share its map
            int am = -1;
            for (int j = 0; j < i && am < 0; ++j)
                if (probs[j].nseg == 1 && a[j][0].ptr == a[i][sg].ptr && a[j][0].rows == a[i][sg].rows &&
                    probs[j].kdim[0] == K)
                    am = probs[j].a_map[0];
            if (am < 0) {
                if (nm >= kMaxTensorMaps ||
                    !encode_bf16(&maps[nm], a[i][sg].ptr, a[i][sg].rows, K, swap ? bn : kBM))
                    return cudaErrorInvalidValue;
                am = nm++;
            }
            probs[i].a_map[sg] = am;
            if (nm >= kMaxTensorMaps ||
                !encode_bf16(&maps[nm], b[i][sg].ptr, b[i][sg].rows, K, swap ? kBM : pair ? 128 : bn))
                return cudaErrorInvalidValue;
            probs[i].b_map[sg] = nm++;
        }
    // output maps for the bulk tensor stores of non-swapped tiles (32-row slabs)
    for (int i = 0; i < nprob && !swap; ++i) {
        const bool f32_out = probs[i].epi == EPI_F32 || probs[i].epi == EPI_SCALE_F32 || probs[i].epi == EPI_RELU2_F32;
        const long long rows = probs[i].grouped ? (long long)c.p->A : probs[i].m_rows;
        if (nm >= kMaxTensorMaps || probs[i].ldo != probs[i].n ||
            !encode_2d(&maps[nm], probs[i].out, rows, probs[i].n, 32, f32_out)) {
            probs[i].out_map = -1;
            continue;
        }
        probs[i].out_map = nm++;
    }
    if (swap) return launch_gemm_tc_decode(maps, nm, probs, nprob, bn, c.r, c.err, c.h->spin_limit, c.s);
    if (pair) return launch_gemm_tc_pair(maps, nm, probs, nprob, c.r, c.err, c.h->spin_limit, c.s);
    return launch_gemm_tc(maps, nm, probs, nprob, bn, c.r, c.err, c.h->spin_limit, c.s);
}

// Grouped expert GEMM with NVFP4 weights: only the activation operand goes
// through a tensor map (box rows = the token tile); the weight tiles are
// copied from the tiled code / scale arrays.
cudaError_t run_gemm_nvfp4(Ctx& c, GemmProblem* pr, const Operand& act) {
    const int bn = c.decode ? kDecodeTN : 128;
    CUtensorMap map;
    if (!encode_bf16(&map, act.ptr, act.rows, pr->kdim[0], bn)) return cudaErrorInvalidValue;
    pr->a_map[0] = 0;
    pr->b_map[0] = -1;
    return launch_gemm_tc_nvfp4(&map, 1, pr, 1, bn, c.r, c.err, c.h->spin_limit, c.s);
}

// TMEM accumulation chunks (k-blocks of 64) per GEMM: a chunk bounds the size of
// the partial sums the tensor core accumulates, which matters where the output
// is rounded to bf16 (0: the engine's default of 8 k-blocks, also taken by the
// fp32 outputs of the expert down and output GEMMs).
#ifndef LMOE_CHUNK_UP
#define LMOE_CHUNK_UP 0      // expert up (a_e, re-rounded): the engine's default
#endif
#ifndef LMOE_CHUNK_DOWN
#define LMOE_CHUNK_DOWN 0
#endif
#ifndef LMOE_CHUNK_OUT
#define LMOE_CHUNK_OUT 0
#endif
#ifndef LMOE_CHUNK_FC1
#define LMOE_CHUNK_FC1 4     // fc1 when z is re-rounded: smaller partial sums, a smaller margin
#endif
#ifndef LMOE_CHUNK_SHARED_UP
#define LMOE_CHUNK_SHARED_UP 4  // shared up (a_s, K = H) when its activations are re-rounded
#endif

// The exact re-rounding list of a relu2 activation problem (see rr_flag).
void set_act_recheck(const Ctx& c, GemmProblem& pr, int* count) {
    const double tau = c.h->act_tau, c0 = c.h->act_c0, c1 = c.h->act_c1;
    pr.rr_list = c.alist;
    pr.rr_count = count;
    pr.rr_cap = c.alist_cap;
    const float tau2 = (float)(tau * tau);
    memcpy(&pr.rr_tau2_bits, &tau2, 4);
    // margin of a = h^2 over an fp32 ulp of a (>= a 2^-24), at its largest (a = tau^2)
    pr.rr_ulps = act_margin_ulps(tau, c0, c1);
}

GemmProblem make_problem(int grouped, int m_rows, int n, int epi, void* out, long long ldo) {
    GemmProblem p;
    memset(&p, 0, sizeof(p));
    p.grouped = grouped;
    p.m_rows = m_rows;
    p.n = n;
    p.nseg = 1;
    p.epi = epi;
    p.out = out;
    p.ldo = ldo;
    p.out_map = -1;
    return p;
}

lmoe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA; }

#define LMOE_TRY(expr)                                   \
    do {                                                 \
        cudaError_t _e = (expr);                         \
        if (_e != cudaSuccess) {                         \
            c.h->last_cuda_error = (int)_e;              \
            return LMOE_ERR_CUDA;                        \
        }                                                \
    } while (0)

// Launch `expr`, which starts `n` kernels, and count them.
#define LMOE_LAUNCH(n, expr)          \
    do {                              \
        LMOE_TRY(expr);               \
        c.h->launches += (n);         \
    } while (0)

// Stage marker (latentmoe_set_profile_events). A failed record must not leave
// a pending runtime error for the next launch check to report, so it is
// consumed here: a marker never fails the call it times.
void mark(const Ctx& c, int i) {
    if (c.h->prof_events && i < c.h->prof_n &&
        cudaEventRecord(static_cast<cudaEvent_t>(c.h->prof_events[i]), c.s) != cudaSuccess)
        (void)cudaGetLastError();
}

__attribute__((unused)) lmoe_status take_device_error(lmoe_handle* h) {
    volatile int* he = h->herr;
    int v = *he;
    if (v != 0) {
        *he = 0;
        return (lmoe_status)v;
    }
    return LMOE_OK;
}

lmoe_status validate_call(lmoe_handle* h, const void* x, int T, void* ws, size_t ws_bytes, Plan& p) {
    if (!h || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
    if (T == 0) return LMOE_OK;
    if (!x || !aligned(x, 16)) return LMOE_ERR_INVALID_ARG;
    plan_of(h->cfg, T, p);
    if (!ws || !aligned(ws, 256) || ws_bytes < p.total) return LMOE_ERR_WORKSPACE;
    return LMOE_OK;
}

// Routing, first part: the statistics reset and, with router_gemm, the fp32
// router logits (tensor cores), unless every token is decided in fp64.
bool route_fp64_all(const Ctx& c) {
    const lmoe_config& cf = c.h->cfg;
    return c.h->fp64_all || cf.mode == LMOE_MODE_FP32 || cf.x_dtype == LMOE_FP32 || cf.num_experts % 64 != 0 ||
           c.simt;
}

// Whether a forward computes the router logits as the first problem of the
// input GEMM launch (fc1 + shared up, which read the same x) instead of in a
// launch of their own: only where that leaves the launch's tiles as they are
// (the same tile width, the same swap-AB choice at decode sizes).
bool router_in_input_gemm(const Ctx& c) {
    const lmoe_config& cf = c.h->cfg;
    if (route_fp64_all(c)) return false;
    const int E = cf.num_experts, L = cf.latent, Is = cf.shared_inter;
    const bool swap2 = c.decode && L % 128 == 0 && Is % 128 == 0;
    if (swap2) return E % 128 == 0;
    const int ns2[2] = {L, Is}, ns3[3] = {E, L, Is};
    return pick_bn(ns3, 3) == pick_bn(ns2, 2);
}

lmoe_status route_head(Ctx& c, const void* x, bool router_gemm) {
    lmoe_handle* h = c.h;
    const lmoe_config& cf = h->cfg;
    const Plan& p = *c.p;
    char* ws = c.ws;
    LMOE_TRY(cudaMemsetAsync(ws + p.stats, 0, sizeof(WsStats), c.s));
    if (router_gemm && !route_fp64_all(c)) {
        GemmProblem pr = make_problem(0, p.T, cf.num_experts, EPI_F32, ws + p.logits, cf.num_experts);
        pr.kdim[0] = cf.hidden;
        Operand a[1][2] = {{{x, p.T}, {nullptr, 0}}};
        Operand b[1][2] = {{{h->w.router_w, cf.num_experts}, {nullptr, 0}}};
        Ctx rc = c;
        rc.decode = c.decode && cf.num_experts % 128 == 0;
        LMOE_LAUNCH(1, run_gemm(rc, &pr, 1, a, b, false));
    }
    return LMOE_OK;
}

// Routing, second part: selection with the near-edge flags, the fp64
// re-decision of the flagged tokens (or of every token), the counting sort.
// Writes idx/w/counts into the workspace and, if given, the caller's outputs.
lmoe_status route_tail(Ctx& c, const void* x, int32_t* idx_out, float* w_out, int32_t* counts_out) {
    lmoe_handle* h = c.h;
    const lmoe_config& cf = h->cfg;
    const Plan& p = *c.p;
    char* ws = c.ws;
    if (!route_fp64_all(c)) {
        LMOE_LAUNCH(1, launch_router_select(h, p, ws, false, c.s));
        LMOE_LAUNCH(1, launch_router_logits64(h, x, p, ws, false, c.s));
        LMOE_LAUNCH(1, launch_router_select64(h, p, ws, false, c.s));
    } else {
        LMOE_LAUNCH(1, launch_router_logits64(h, x, p, ws, true, c.s));
        LMOE_LAUNCH(1, launch_router_select64(h, p, ws, true, c.s));
    }
    LMOE_LAUNCH(3, launch_permute(h, p, ws, counts_out, c.s));
    LMOE_LAUNCH((idx_out || w_out) ? 1 : 0,
                launch_copy_routing(reinterpret_cast<const int*>(ws + p.idx), reinterpret_cast<const float*>(ws + p.wgt),
                                    idx_out, w_out, (long long)p.T * cf.top_k, h->num_sms, c.s));
    return LMOE_OK;
}

// Routing in order on the call's stream (latentmoe_route): the router GEMM,
// then steps 2-4 of the file comment.
lmoe_status do_route(Ctx& c, const void* x, int32_t* idx_out, float* w_out, int32_t* counts_out) {
    lmoe_status s = route_head(c, x, true);
    if (s != LMOE_OK) return s;
    return route_tail(c, x, idx_out, w_out, counts_out);
}

// Where the routing tail of a forward writes the caller's copies of its outputs.
struct RouteOut {
    int32_t* idx;
    float* w;
    int32_t* counts;
};

Ctx make_ctx(lmoe_handle* h, const Plan& p, void* ws, void* stream) {
    Ctx c;
    c.h = h;
    c.p = &p;
    c.ws = static_cast<char*>(ws);
    c.s = static_cast<cudaStream_t>(stream);
    c.r.offsets = reinterpret_cast<const int*>(c.ws + p.offsets);
    c.r.pfx128 = reinterpret_cast<const int*>(c.ws + p.pfx128);
    c.r.pfx64 = reinterpret_cast<const int*>(c.ws + p.pfx64);
    c.r.pfxdec = reinterpret_cast<const int*>(c.ws + p.pfxdec);
    c.r.pfx256 = reinterpret_cast<const int*>(c.ws + p.pfx256);
    c.r.rec32 = reinterpret_cast<const int4*>(c.ws + p.rec32);
    c.r.rec64 = reinterpret_cast<const int4*>(c.ws + p.rec64);
    c.r.rec128 = reinterpret_cast<const int4*>(c.ws + p.rec128);
    c.r.rec256 = reinterpret_cast<const int4*>(c.ws + p.rec256);
    c.r.E = h->cfg.num_experts;
    c.err = &reinterpret_cast<WsStats*>(c.ws + p.stats)->device_error;
    c.st = reinterpret_cast<WsStats*>(c.ws + p.stats);
    c.alist = reinterpret_cast<int2*>(c.ws + p.alist);
    c.alist_cap = p.alist_cap;
    const lmoe_config& cf = h->cfg;
    c.simt = h->gemm_path == 3 || cf.mode == LMOE_MODE_FP32;
    if (h->gemm_path == 1 || h->gemm_path == 4) c.decode = false;
    else if (h->gemm_path == 2) c.decode = true;
    else c.decode = (long long)p.T * cf.top_k <= 64LL * cf.num_experts;  // <= 64 rows per expert on average
    return c;
}

__global__ void k_publish_error(const int* derr, int* herr) {
    int v = *derr;
    if (v != 0) *(volatile int*)herr = v;
}

// Experts whose weights the handle holds (a shard of them for expert parallelism).
int experts_held(const lmoe_config& c) { return c.local_experts > 0 ? c.local_experts : c.num_experts; }

lmoe_status rerounding(Ctx& c, const void* xa, bool zcheck, bool act_rr);

// Steps 1-6 of the file comment: the input GEMM (z = x W_fc1^T and
// a_s = relu2(x W_su^T), with the router logits as a first problem when
// with_router), then the rows of z in expert order into zdst. The routing tail
// (route_tail, after route_head on the call's stream) runs here on the handle's
// second stream, next to the exact re-roundings of z and a_s, which do not read
// its outputs; the gather, the first reader of the permutation, waits for it.
lmoe_status stage_front(Ctx& c, const void* x, void* zdst, const RouteOut& ro, bool with_router) {
    lmoe_handle* h = c.h;
    const lmoe_config& cf = h->cfg;
    const Plan& p = *c.p;
    char* ws_c = c.ws;
    const bool bf16 = cf.mode == LMOE_MODE_BF16;
    const int act = bf16 ? 2 : 4;
    const int H = cf.hidden, L = cf.latent, Is = cf.shared_inter, E = cf.num_experts;
    const int gemm_kernels = c.simt ? 2 : 1;  // SIMT launches one kernel per problem
    // exact re-rounding of z (bf16 mode, every GEMM path): fc1 writes fp32 z into the expert
    // output buffer, which is free until the expert down GEMM, and the near-midpoint list goes
    // into the plan's list buffer (room for all of z, so no element can be left out)
    const bool zcheck = bf16 && h->zcheck_delta > 0.f;
    // GEMM operand x: bf16 x as given, fp32 x rounded to bf16 (bf16 mode) or fp32 x (validation mode).
    const void* xa = x;
    bool xa_f32 = cf.x_dtype == LMOE_FP32;
    if (bf16 && cf.x_dtype == LMOE_FP32) {
        LMOE_LAUNCH(1, launch_convert_x(static_cast<const float*>(x), reinterpret_cast<uint16_t*>(ws_c + p.xbf),
                                        (long long)p.T * H, h->num_sms, c.s));
        xa = ws_c + p.xbf;
        xa_f32 = false;
    }
    const bool act_rr = bf16 && h->act_tau > 0.f;
    {
        // problems: [router logits (fp32), when merged,] fc1, shared up; all read x
        GemmProblem pr[3];
        Operand a[3][2], b[3][2];
        int np = 0;
        auto add = [&](GemmProblem q, const void* w, int n) {
            q.kdim[0] = H;
            q.a_ptr[0] = xa;
            q.b_ptr[0] = w;
            a[np][0] = {xa, p.T};
            a[np][1] = {nullptr, 0};
            b[np][0] = {w, n};
            b[np][1] = {nullptr, 0};
            pr[np] = q;
            return np++;
        };
        if (with_router) add(make_problem(0, p.T, E, EPI_F32, ws_c + p.logits, E), h->w.router_w, E);
        const int i_fc1 = add(make_problem(0, p.T, L, bf16 && !zcheck ? EPI_BF16 : EPI_F32,
                                           ws_c + (zcheck ? p.o : p.z), L),
                              h->w.fc1_w, L);
        const int i_su = add(make_problem(0, p.T, Is, bf16 ? EPI_RELU2_BF16 : EPI_RELU2_F32, ws_c + p.as, Is),
                             h->w.shared_up_w, Is);
        // fc1 in short chunks when z is re-rounded: a smaller fp32 error, a shorter list
        if (zcheck) pr[i_fc1].chunk_kb = LMOE_CHUNK_FC1;
        if (act_rr) {
            set_act_recheck(c, pr[i_su], &c.st->asflagged);
            pr[i_su].chunk_kb = LMOE_CHUNK_SHARED_UP;
        }
        LMOE_LAUNCH(gemm_kernels, run_gemm(c, pr, np, a, b, xa_f32));
    }
    // fork: the routing tail on the second stream once the input GEMM is done (the GEMM keeps
    // every SM; the tail's kernels share them with the re-roundings)
    LMOE_TRY(cudaEventRecord(h->ev_fork, c.s));
    LMOE_TRY(cudaStreamWaitEvent(h->aux, h->ev_fork, 0));
    Ctx ca = c;
    ca.s = h->aux;
    const lmoe_status rs = route_tail(ca, x, ro.idx, ro.w, ro.counts);
    cudaError_t je = cudaEventRecord(h->ev_join, h->aux);
    lmoe_status s = rs != LMOE_OK ? rs : rerounding(c, xa, zcheck, act_rr);
    // join (also after a failure, so that no work of this call is left on the second stream)
    if (je == cudaSuccess) je = cudaStreamWaitEvent(c.s, h->ev_join, 0);
    if (s != LMOE_OK) return s;
    if (je != cudaSuccess) {
        h->last_cuda_error = (int)je;
        return LMOE_ERR_CUDA;
    }
    mark(c, 2);
    LMOE_LAUNCH(1, launch_gather_rows(ws_c + p.z, p.T, c.err, zdst, reinterpret_cast<const int*>(ws_c + p.perm), p.A,
                                      reinterpret_cast<const int*>(ws_c + p.offsets) + E, L * act, h->num_sms, c.s));
    mark(c, 3);
    return LMOE_OK;
}

// The exact re-roundings of the input stage: z (round, list, re-check by row
// segments) and the shared-expert activations a_s.
lmoe_status rerounding(Ctx& c, const void* xa, bool zcheck, bool act_rr) {
    lmoe_handle* h = c.h;
    const lmoe_config& cf = h->cfg;
    const Plan& p = *c.p;
    char* ws_c = c.ws;
    const int H = cf.hidden, L = cf.latent, Is = cf.shared_inter;
    if (zcheck) {
        const int cap = (int)std::min<long long>((long long)p.T * L, 0x7FFFFFFF);  // T * L < 2^31 (create)
        int2* list = reinterpret_cast<int2*>(ws_c + p.zlist);
        int* count = &c.st->zflagged;
        uint16_t* z = reinterpret_cast<uint16_t*>(ws_c + p.z);
        int4* rowtab = reinterpret_cast<int4*>(ws_c + p.zrowtab);
        LMOE_LAUNCH(1, launch_z_round_flag(reinterpret_cast<const float*>(ws_c + p.o), z, p.T, L, h->zcheck_delta,
                                           0.4f * h->zcheck_delta, list, cap, count, rowtab, &c.st->zrows, h->num_sms,
                                           c.s));
        LMOE_LAUNCH(1, launch_recheck_rows(static_cast<const uint16_t*>(xa), p.T,
                                           static_cast<const uint16_t*>(h->w.fc1_w), L, H, c.err, list, cap, rowtab,
                                           &c.st->zrows, z, L, h->num_sms, c.s));
    }
    if (act_rr)
        LMOE_LAUNCH(1, launch_recheck(true, static_cast<const uint16_t*>(xa), p.T,
                                      static_cast<const uint16_t*>(h->w.shared_up_w), Is, H, c.err, c.alist,
                                      &c.st->asflagged, c.alist_cap, reinterpret_cast<uint16_t*>(ws_c + p.as), Is,
                                      h->num_sms, c.s));
    return LMOE_OK;
}

// Steps 7-8 on n rows grouped as c.r describes: a = relu2(rows W_up[e]^T) into
// a_buf, o = w * (a W_down[e]^T) (NVFP4: the matrix scales before relu2 and w).
// Group g takes expert g % expert_mod's weights when expert_mod is non-zero.
lmoe_status stage_experts(Ctx& c, const void* rows, long long n, const float* row_w, void* a_buf, float* o,
                          int expert_mod) {
    lmoe_handle* h = c.h;
    const lmoe_config& cf = h->cfg;
    const bool bf16 = cf.mode == LMOE_MODE_BF16;
    const bool fp4 = cf.expert_format == LMOE_EXPERTS_NVFP4;
    const int L = cf.latent, I = cf.expert_inter, Ew = experts_held(cf);
    const bool act_rr = bf16 && !fp4 && h->act_tau > 0.f;
    {
        GemmProblem pr = make_problem(1, 0, I, bf16 ? EPI_RELU2_BF16 : EPI_RELU2_F32, a_buf, I);
        pr.kdim[0] = L;
        pr.b_rows_per_expert = I;
        pr.expert_mod = expert_mod;
        pr.chunk_kb = LMOE_CHUNK_UP;
        if (act_rr) set_act_recheck(c, pr, &c.st->aeflagged);
        pr.a_ptr[0] = rows;
        pr.b_ptr[0] = h->w.up_w;
        Operand a[1][2] = {{{rows, n}, {nullptr, 0}}};
        Operand b[1][2] = {{{h->w.up_w, (long long)Ew * I}, {nullptr, 0}}};
        if (fp4) {
            pr.wq_codes = static_cast<const uint8_t*>(h->w.up_w);
            pr.wq_sf = static_cast<const uint8_t*>(h->w.up_sf);
            pr.wscale = h->w.up_gs;
            LMOE_LAUNCH(1, run_gemm_nvfp4(c, &pr, a[0][0]));
        } else {
            LMOE_LAUNCH(1, run_gemm(c, &pr, 1, a, b, !bf16));
        }
    }
    if (act_rr)
        LMOE_LAUNCH(1, launch_recheck(true, static_cast<const uint16_t*>(rows), (int)n,
                                      static_cast<const uint16_t*>(h->w.up_w), Ew * I, L, c.err, c.alist,
                                      &c.st->aeflagged, c.alist_cap, static_cast<uint16_t*>(a_buf), I, h->num_sms,
                                      c.s));
    mark(c, 4);
    {
        GemmProblem pr = make_problem(1, 0, L, EPI_SCALE_F32, o, L);
        pr.kdim[0] = I;
        pr.b_rows_per_expert = L;
        pr.expert_mod = expert_mod;
        pr.chunk_kb = LMOE_CHUNK_DOWN;
        pr.row_scale = row_w;
        pr.a_ptr[0] = a_buf;
        pr.b_ptr[0] = h->w.down_w;
        Operand a[1][2] = {{{a_buf, n}, {nullptr, 0}}};
        Operand b[1][2] = {{{h->w.down_w, (long long)Ew * L}, {nullptr, 0}}};
        if (fp4) {
            pr.wq_codes = static_cast<const uint8_t*>(h->w.down_w);
            pr.wq_sf = static_cast<const uint8_t*>(h->w.down_sf);
            pr.wscale = h->w.down_gs;
            LMOE_LAUNCH(1, run_gemm_nvfp4(c, &pr, a[0][0]));
        } else {
            LMOE_LAUNCH(1, run_gemm(c, &pr, 1, a, b, !bf16));
        }
    }
    mark(c, 5);
    return LMOE_OK;
}

// Steps 9-10: comb[t] = bf16(sum of the token's k rows of o, ascending expert
// id) via the slot map of do_route, then y = comb W_fc2^T + a_s W_sd^T
// (+ resid), one K-concatenated GEMM.
lmoe_status stage_back(Ctx& c, const float* o, float* y, const uint16_t* resid) {
    lmoe_handle* h = c.h;
    const lmoe_config& cf = h->cfg;
    const Plan& p = *c.p;
    char* ws_c = c.ws;
    const bool bf16 = cf.mode == LMOE_MODE_BF16;
    const int H = cf.hidden, L = cf.latent, Is = cf.shared_inter;
    LMOE_LAUNCH(1, launch_combine(o, p.A, c.err, reinterpret_cast<const int*>(ws_c + p.slot), ws_c + p.comb, p.T,
                                  cf.top_k, L, bf16, h->num_sms, c.s));
    mark(c, 6);
    {
        GemmProblem pr = make_problem(0, p.T, H, EPI_F32, y, H);
        pr.chunk_kb = LMOE_CHUNK_OUT;
        pr.nseg = 2;
        pr.kdim[0] = L;
        pr.kdim[1] = Is;
        pr.a_ptr[0] = ws_c + p.comb;
        pr.b_ptr[0] = h->w.fc2_w;
        pr.a_ptr[1] = ws_c + p.as;
        pr.b_ptr[1] = h->w.shared_down_w;
        pr.resid = resid;
        Operand a[1][2] = {{{ws_c + p.comb, p.T}, {ws_c + p.as, p.T}}};
        Operand b[1][2] = {{{h->w.fc2_w, H}, {h->w.shared_down_w, H}}};
        LMOE_LAUNCH(1, run_gemm(c, &pr, 1, a, b, !bf16));
    }
    mark(c, 7);
    return LMOE_OK;
}

// The layer on x (steps 1-10 of the file comment). With norm_src the pre-norm
// runs first and x is its output; with `resid` (bf16 [T, H]) the output GEMM
// adds it: y = resid + layer(x).
lmoe_status forward_impl(lmoe_handle* h, const Plan& p, const void* x, float* y, void* ws, void* stream,
                         int32_t* topk_idx, float* topk_w, int32_t* expert_counts, const uint16_t* resid,
                         const uint16_t* norm_src, const uint16_t* norm_w, double norm_eps) {
    lmoe_status s;
    const lmoe_config& cf = h->cfg;
    Ctx c = make_ctx(h, p, ws, stream);
    char* ws_c = c.ws;
    h->launches = 0;
    mark(c, 0);
    if (norm_src) LMOE_LAUNCH(1, launch_rmsnorm(norm_src, norm_w, norm_eps, p.T, cf.hidden,
                                                reinterpret_cast<uint16_t*>(const_cast<void*>(x)), h->num_sms, c.s));
    const bool merged = router_in_input_gemm(c);
    s = route_head(c, x, !merged);
    if (s != LMOE_OK) return s;
    mark(c, 1);
    s = stage_front(c, x, ws_c + p.zperm, RouteOut{topk_idx, topk_w, expert_counts}, merged);
    if (s != LMOE_OK) return s;
    s = stage_experts(c, ws_c + p.zperm, p.A, reinterpret_cast<const float*>(ws_c + p.wperm), ws_c + p.aperm,
                      reinterpret_cast<float*>(ws_c + p.o), 0);
    if (s != LMOE_OK) return s;
    s = stage_back(c, reinterpret_cast<const float*>(ws_c + p.o), y, resid);
    if (s != LMOE_OK) return s;
    k_publish_error<<<1, 1, 0, c.s>>>(c.err, h->derr);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

// Workspace of latentmoe_ep_experts: the scan of the received blocks and the
// expert activations of the received rows.
struct EpPlan {
    size_t total, stats, bcounts, counts, offsets, pfx128, pfx64, pfxdec, pfx256, rec32, rec64, rec128, rec256, a, alist;
    int alist_cap;
};

void ep_plan_of(const lmoe_config& c, int n_rows, int nb, EpPlan& p) {
    const size_t n = n_rows;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += al256(bytes);
        return o;
    };
    p.stats = take(sizeof(WsStats));
    p.bcounts = take((size_t)nb * 4);
    p.counts = take((size_t)nb * 4);
    p.offsets = take((size_t)(nb + 1) * 4);
    p.pfx128 = take((size_t)(nb + 1) * 4);
    p.pfx64 = take((size_t)(nb + 1) * 4);
    p.pfxdec = take((size_t)(nb + 1) * 4);
    p.pfx256 = take((size_t)(nb + 1) * 4);
    p.rec32 = take((n / 32 + nb) * 16);
    p.rec64 = take((n / 64 + nb) * 16);
    p.rec128 = take((n / 128 + nb) * 16);
    p.rec256 = take((n / 256 + nb) * 16);
    p.a = take(n * c.expert_inter * (c.mode == LMOE_MODE_BF16 ? 2 : 4));
    p.alist_cap = (int)std::min<size_t>(n * c.expert_inter / 256 + 64, 0x7FFFFFFF);
    p.alist = take((size_t)p.alist_cap * 8);
    p.total = off;
}

lmoe_status check_outputs(float* y, int32_t* topk_idx, float* topk_w, int32_t* expert_counts) {
    if (!y || !aligned(y, 16)) return LMOE_ERR_INVALID_ARG;
    if ((topk_idx && !aligned(topk_idx, 4)) || (topk_w && !aligned(topk_w, 4)) ||
        (expert_counts && !aligned(expert_counts, 4)))
        return LMOE_ERR_INVALID_ARG;
    return LMOE_OK;
}

}  // namespace

extern "C" {

lmoe_status latentmoe_forward(lmoe_handle* h, const void* x, int T, float* y, void* ws, size_t ws_bytes,
                                         void* stream, int32_t* topk_idx, float* topk_w, int32_t* expert_counts) {
    Plan p;
    lmoe_status s = validate_call(h, x, T, ws, ws_bytes, p);
    if (s != LMOE_OK || T == 0) return s;
    if (experts_held(h->cfg) != h->cfg.num_experts) return LMOE_ERR_UNSUPPORTED;  // a shard: use the ep_ calls
    s = check_outputs(y, topk_idx, topk_w, expert_counts);
    if (s != LMOE_OK) return s;
    s = take_device_error(h);
    if (s != LMOE_OK) return s;
    return forward_impl(h, p, x, y, ws, stream, topk_idx, topk_w, expert_counts, nullptr, nullptr, nullptr, 0.0);
}

lmoe_status latentmoe_forward_block(lmoe_handle* h, const void* x, int T, const void* norm_w,
                                               float norm_eps, float* y, void* ws, size_t ws_bytes, void* stream,
                                               int32_t* topk_idx, float* topk_w, int32_t* expert_counts) {
    Plan p;
    lmoe_status s = validate_call(h, x, T, ws, ws_bytes, p);
    if (s != LMOE_OK || T == 0) return s;
    if (h->cfg.x_dtype != LMOE_BF16 || experts_held(h->cfg) != h->cfg.num_experts) return LMOE_ERR_UNSUPPORTED;
    if (!norm_w || !aligned(norm_w, 16) || !(norm_eps >= 0.f) || isinf(norm_eps)) return LMOE_ERR_INVALID_ARG;
    s = check_outputs(y, topk_idx, topk_w, expert_counts);
    if (s != LMOE_OK) return s;
    s = take_device_error(h);
    if (s != LMOE_OK) return s;
    char* xn = static_cast<char*>(ws) + p.xnorm;
    return forward_impl(h, p, xn, y, ws, stream, topk_idx, topk_w, expert_counts, static_cast<const uint16_t*>(x),
                        static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(norm_w), (double)norm_eps);
}


lmoe_status latentmoe_create(const lmoe_config* cfg, const lmoe_weights* w, lmoe_handle** out) {
    if (!out) return LMOE_ERR_INVALID_ARG;
    lmoe_status s = check_config(cfg);
    if (s != LMOE_OK) return s;
    s = check_weights(*cfg, w);
    if (s != LMOE_OK) return s;
    if (!get_encoder()) return LMOE_ERR_CUDA;
    lmoe_handle* h = new (std::nothrow) lmoe_handle();
    if (!h) return LMOE_ERR_INTERNAL;
    h->cfg = *cfg;
    h->w = *w;
    if (cudaHostAlloc(reinterpret_cast<void**>(&h->herr), 64, cudaHostAllocMapped) != cudaSuccess) {
        delete h;
        return LMOE_ERR_CUDA;
    }
    *h->herr = 0;
    if (cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->derr), h->herr, 0) != cudaSuccess) {
        cudaFreeHost(h->herr);
        delete h;
        return LMOE_ERR_CUDA;
    }
    h->num_sms = tc_num_sms();
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess ||
        cudaStreamCreateWithPriority(&h->aux, cudaStreamNonBlocking, hi) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess) {
        latentmoe_destroy(h);
        return LMOE_ERR_CUDA;
    }
    *out = h;
    return LMOE_OK;
}

lmoe_status latentmoe_workspace_size(const lmoe_handle* h, int T, size_t* bytes) {
    if (!h || !bytes || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
    Plan p;
    plan_of(h->cfg, T, p);
    *bytes = T == 0 ? 0 : p.total;
    return LMOE_OK;
}

lmoe_status latentmoe_route(lmoe_handle* h, const void* x, int T, int32_t* topk_idx, float* topk_w,
                            int32_t* expert_counts, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    lmoe_status s = validate_call(h, x, T, ws, ws_bytes, p);
    if (s != LMOE_OK || T == 0) return s;
    if ((topk_idx && !aligned(topk_idx, 4)) || (topk_w && !aligned(topk_w, 4)) ||
        (expert_counts && !aligned(expert_counts, 4)))
        return LMOE_ERR_INVALID_ARG;
    s = take_device_error(h);
    if (s != LMOE_OK) return s;
    Ctx c = make_ctx(h, p, ws, stream);
    h->launches = 0;
    s = do_route(c, x, topk_idx, topk_w, expert_counts);
    if (s != LMOE_OK) return s;
    k_publish_error<<<1, 1, 0, c.s>>>(c.err, h->derr);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

void latentmoe_destroy(lmoe_handle* h) {
    if (!h) return;
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->aux) cudaStreamDestroy(h->aux);
    if (h->herr) cudaFreeHost(h->herr);
    delete h;
}

const char* latentmoe_status_string(lmoe_status s) {
    switch (s) {
        case LMOE_OK: return "ok";
        case LMOE_ERR_INVALID_ARG: return "invalid argument";
        case LMOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case LMOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case LMOE_ERR_CUDA: return "CUDA error";
        case LMOE_ERR_TIMEOUT: return "bounded device wait timed out";
        case LMOE_ERR_INTERNAL: return "internal error";
    }
    return "unknown status";
}

lmoe_status latentmoe_set_option(lmoe_handle* h, lmoe_option opt, long long v) {
    if (!h) return LMOE_ERR_INVALID_ARG;
    switch (opt) {
        case LMOE_OPT_GEMM_PATH:
            if (v < 0 || v > 4) return LMOE_ERR_INVALID_ARG;
            if (v == 3 && h->cfg.expert_format == LMOE_EXPERTS_NVFP4) return LMOE_ERR_UNSUPPORTED;
            h->gemm_path = (int)v;
            return LMOE_OK;
        case LMOE_OPT_ROUTER_FP64_ALL:
            h->fp64_all = v != 0;
            return LMOE_OK;
        case LMOE_OPT_FLAG_DELTA:
            if (v < 0 || v > 100000000) return LMOE_ERR_INVALID_ARG;
            h->flag_delta = (float)(v * 1e-9);
            return LMOE_OK;
        case LMOE_OPT_Z_RECHECK_DELTA:
            if (v < 0 || v > 100000000) return LMOE_ERR_INVALID_ARG;
            h->zcheck_delta = (float)(v * 1e-9);
            return LMOE_OK;
        case LMOE_OPT_SPIN_LIMIT:
            if (v < 1 || v > 0xFFFFFFFFLL) return LMOE_ERR_INVALID_ARG;
            h->spin_limit = (unsigned)v;
            return LMOE_OK;
        case LMOE_OPT_ACT_RECHECK_TAU:
            // 0 disables; below kActTauMin the list could not hold every flagged activation
            if (v < 0 || v > 1000000 || (v > 0 && v * 1e-3 < kActTauMin)) return LMOE_ERR_INVALID_ARG;
            h->act_tau = (float)(v * 1e-3);
            return LMOE_OK;
    }
    return LMOE_ERR_INVALID_ARG;
}

lmoe_status latentmoe_workspace_layout(const lmoe_handle* h, int T, lmoe_ws_layout* out) {
    if (!h || !out || T < 1 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
    Plan p;
    plan_of(h->cfg, T, p);
    out->logits_f32 = p.logits;
    out->z_f32 = p.o;
    out->z = p.z;
    out->flag_list = p.flaglist;
    out->perm = p.perm;
    out->slot = p.slot;
    out->total = p.total;
    out->offsets = p.offsets;
    out->act_e = p.aperm;
    out->act_s = p.as;
    return LMOE_OK;
}

lmoe_status latentmoe_read_stats(const lmoe_handle* h, const void* ws, lmoe_stats* out) {
    if (!h || !ws || !out) return LMOE_ERR_INVALID_ARG;
    WsStats st;
    if (cudaMemcpy(&st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return LMOE_ERR_CUDA;
    out->flagged_tokens = st.flagged;
    out->distinct_experts = st.distinct;
    out->max_expert_tokens = st.max_count;
    out->device_error = st.device_error;
    out->kernel_launches = h->launches;
    out->cuda_error = h->last_cuda_error;
    out->z_rechecked = st.zflagged;
    out->ae_rechecked = st.aeflagged;
    out->as_rechecked = st.asflagged;
    return LMOE_OK;
}

lmoe_status latentmoe_update_bias(lmoe_handle* h, const int32_t* expert_counts, const float* bias_in, float eta,
                                  float* bias_out, double* maxvio_out, void* stream) {
    if (!h || !expert_counts || !bias_in || !bias_out || !aligned(expert_counts, 4) || !aligned(bias_in, 4) ||
        !aligned(bias_out, 4) || (maxvio_out && !aligned(maxvio_out, 8)) || !(eta == eta) || isinf(eta))
        return LMOE_ERR_INVALID_ARG;
    return cuda_status(launch_update_bias(expert_counts, bias_in, h->cfg.num_experts, (double)eta, bias_out, maxvio_out,
                                          static_cast<cudaStream_t>(stream)));
}

lmoe_status latentmoe_ep_front(lmoe_handle* h, const void* x, int T, void* send_rows, float* send_w,
                               int32_t* expert_counts, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    lmoe_status s = validate_call(h, x, T, ws, ws_bytes, p);
    if (s != LMOE_OK || T == 0) return s;
    if (!send_rows || !aligned(send_rows, 16) || !send_w || !aligned(send_w, 4) || !expert_counts ||
        !aligned(expert_counts, 4))
        return LMOE_ERR_INVALID_ARG;
    s = take_device_error(h);
    if (s != LMOE_OK) return s;
    Ctx c = make_ctx(h, p, ws, stream);
    h->launches = 0;
    mark(c, 0);
    const bool merged = router_in_input_gemm(c);
    s = route_head(c, x, !merged);
    if (s != LMOE_OK) return s;
    mark(c, 1);
    s = stage_front(c, x, send_rows, RouteOut{nullptr, nullptr, expert_counts}, merged);
    if (s != LMOE_OK) return s;
    LMOE_TRY(cudaMemcpyAsync(send_w, c.ws + p.wperm, (size_t)p.A * 4, cudaMemcpyDeviceToDevice, c.s));
    k_publish_error<<<1, 1, 0, c.s>>>(c.err, h->derr);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

lmoe_status latentmoe_ep_workspace_size(const lmoe_handle* h, int n_rows, int n_src, size_t* bytes) {
    if (!h || !bytes || n_rows < 0 || n_src < 1) return LMOE_ERR_INVALID_ARG;
    const int nb = n_src * experts_held(h->cfg);
    if (nb > kMaxE) return LMOE_ERR_UNSUPPORTED;
    EpPlan p;
    ep_plan_of(h->cfg, n_rows, nb, p);
    *bytes = p.total;
    return LMOE_OK;
}

lmoe_status latentmoe_ep_experts(lmoe_handle* h, const void* recv_rows, const float* recv_w,
                                 const int32_t* recv_counts, int n_src, int n_rows, float* recv_o, void* ws,
                                 size_t ws_bytes, void* stream) {
    if (!h || n_src < 1 || n_rows < 0 || !recv_counts || !aligned(recv_counts, 4)) return LMOE_ERR_INVALID_ARG;
    const lmoe_config& cf = h->cfg;
    const int El = experts_held(cf), nb = n_src * El;
    if (nb > kMaxE || (long long)n_rows > (long long)cf.max_tokens * cf.top_k * n_src) return LMOE_ERR_UNSUPPORTED;
    if (n_rows == 0) return LMOE_OK;
    if (!recv_rows || !aligned(recv_rows, 16) || !recv_w || !aligned(recv_w, 4) || !recv_o || !aligned(recv_o, 16))
        return LMOE_ERR_INVALID_ARG;
    EpPlan q;
    ep_plan_of(cf, n_rows, nb, q);
    if (!ws || !aligned(ws, 256) || ws_bytes < q.total) return LMOE_ERR_WORKSPACE;
    lmoe_status s = take_device_error(h);
    if (s != LMOE_OK) return s;
    // a plan carrying only what the GEMM launchers read (row count of the grouped problems)
    Plan p;
    memset(&p, 0, sizeof(p));
    p.T = n_rows;
    p.A = n_rows;
    Ctx c;
    c.h = h;
    c.p = &p;
    c.ws = static_cast<char*>(ws);
    c.s = static_cast<cudaStream_t>(stream);
    c.r.offsets = reinterpret_cast<const int*>(c.ws + q.offsets);
    c.r.pfx128 = reinterpret_cast<const int*>(c.ws + q.pfx128);
    c.r.pfx64 = reinterpret_cast<const int*>(c.ws + q.pfx64);
    c.r.pfxdec = reinterpret_cast<const int*>(c.ws + q.pfxdec);
    c.r.pfx256 = reinterpret_cast<const int*>(c.ws + q.pfx256);
    c.r.rec32 = reinterpret_cast<const int4*>(c.ws + q.rec32);
    c.r.rec64 = reinterpret_cast<const int4*>(c.ws + q.rec64);
    c.r.rec128 = reinterpret_cast<const int4*>(c.ws + q.rec128);
    c.r.rec256 = reinterpret_cast<const int4*>(c.ws + q.rec256);
    c.r.E = nb;
    c.err = &reinterpret_cast<WsStats*>(c.ws + q.stats)->device_error;
    c.st = reinterpret_cast<WsStats*>(c.ws + q.stats);
    c.alist = reinterpret_cast<int2*>(c.ws + q.alist);
    c.alist_cap = q.alist_cap;
    c.simt = h->gemm_path == 3 || cf.mode == LMOE_MODE_FP32;
    if (h->gemm_path == 1 || h->gemm_path == 4) c.decode = false;
    else if (h->gemm_path == 2) c.decode = true;
    else c.decode = (long long)n_rows <= 64LL * El * n_src;  // <= 64 rows per block on average, as the forward
    h->launches = 0;
    LMOE_TRY(cudaMemsetAsync(c.ws + q.stats, 0, sizeof(WsStats), c.s));
    LMOE_TRY(cudaMemcpyAsync(c.ws + q.bcounts, recv_counts, (size_t)nb * 4, cudaMemcpyDeviceToDevice, c.s));
    LMOE_LAUNCH(2, launch_group_scan(reinterpret_cast<int*>(c.ws + q.bcounts), nb, n_rows,
                                     reinterpret_cast<int*>(c.ws + q.counts), reinterpret_cast<int*>(c.ws + q.offsets),
                                     reinterpret_cast<int*>(c.ws + q.pfx128), reinterpret_cast<int*>(c.ws + q.pfx64),
                                     reinterpret_cast<int*>(c.ws + q.pfxdec), reinterpret_cast<int*>(c.ws + q.pfx256),
                                     reinterpret_cast<int4*>(c.ws + q.rec32), reinterpret_cast<int4*>(c.ws + q.rec64),
                                     reinterpret_cast<int4*>(c.ws + q.rec128), reinterpret_cast<int4*>(c.ws + q.rec256),
                                     reinterpret_cast<WsStats*>(c.ws + q.stats), c.s));
    s = stage_experts(c, recv_rows, n_rows, recv_w, c.ws + q.a, recv_o, El);
    if (s != LMOE_OK) return s;
    k_publish_error<<<1, 1, 0, c.s>>>(c.err, h->derr);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

lmoe_status latentmoe_ep_back(lmoe_handle* h, const float* send_o, int T, float* y, void* ws, size_t ws_bytes,
                              void* stream) {
    if (!h || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
    if (T == 0) return LMOE_OK;
    Plan p;
    plan_of(h->cfg, T, p);
    if (!ws || !aligned(ws, 256) || ws_bytes < p.total) return LMOE_ERR_WORKSPACE;
    if (!send_o || !aligned(send_o, 16) || !y || !aligned(y, 16)) return LMOE_ERR_INVALID_ARG;
    lmoe_status s = take_device_error(h);
    if (s != LMOE_OK) return s;
    Ctx c = make_ctx(h, p, ws, stream);
    h->launches = 0;
    s = stage_back(c, send_o, y, nullptr);
    if (s != LMOE_OK) return s;
    k_publish_error<<<1, 1, 0, c.s>>>(c.err, h->derr);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

lmoe_status latentmoe_quantize_nvfp4(const void* w, long long n_mat, int R, int K, void* codes, void* sf, float* gs,
                                     void* stream) {
    if (n_mat < 0 || R <= 0 || K <= 0) return LMOE_ERR_INVALID_ARG;
    if (n_mat == 0) return LMOE_OK;
    if (!w || !codes || !sf || !gs || !aligned(w, 16) || !aligned(codes, 16) || !aligned(sf, 16) || !aligned(gs, 4))
        return LMOE_ERR_INVALID_ARG;
    if (R % 128 || K % 64 || n_mat > 65535 || (long long)R * K > (1LL << 40) / n_mat) return LMOE_ERR_UNSUPPORTED;
    return cuda_status(launch_quantize_nvfp4(static_cast<const uint16_t*>(w), n_mat, R, K, static_cast<uint8_t*>(codes),
                                             static_cast<uint8_t*>(sf), gs, static_cast<cudaStream_t>(stream)));
}

lmoe_status latentmoe_set_profile_events(lmoe_handle* h, void* const* events, int n) {
    if (!h || (events && n < 8)) return LMOE_ERR_INVALID_ARG;
    for (int i = 0; events && i < 8; ++i)
        if (!events[i]) return LMOE_ERR_INVALID_ARG;  // e.g. a framework event not created yet
    h->prof_events = events;
    h->prof_n = events ? n : 0;
    return LMOE_OK;
}

lmoe_status latentmoe_selftest_bounded_wait(lmoe_handle* h) {
    if (!h) return LMOE_ERR_INVALID_ARG;
    int* d = nullptr;
    if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) return LMOE_ERR_CUDA;
    int v = 0;
    cudaError_t e = cudaMemset(d, 0, sizeof(int));
    if (e == cudaSuccess) e = launch_selftest_wait(d, h->spin_limit, 0);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(&v, d, sizeof(int), cudaMemcpyDeviceToHost);
    cudaFree(d);
    if (e != cudaSuccess) return LMOE_ERR_CUDA;
    return (lmoe_status)v;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Routing without any allocation.
//
// Some callers cannot allocate device memory at the moment they route: code
// running inside a real-time or latency-critical section where cudaMalloc's
// implicit synchronisation is not allowed, inference runtimes whose memory is
// owned by a fixed arena, plugin hosts that forbid allocation from extension
// code. latentmoe_route_noalloc gives them routing with no workspace argument:
// its scratch is the file-scope array below, which every GPU that loads this
// library holds until the process exits.
static constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is asked from the
// runtime once per device (with that device current) and cached.
lmoe_status noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LMOE_ERR_CUDA;
    if (dev >= kMaxDevices) return LMOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LMOE_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LMOE_OK;
}
}  // namespace

extern "C" lmoe_status latentmoe_route_noalloc(lmoe_handle* h, const void* x, int T, int32_t* topk_idx,
                                               float* topk_w, int32_t* expert_counts, void* stream) {
    if (!h || T < 0 || T > h->cfg.max_tokens) return LMOE_ERR_INVALID_ARG;
    if (T == 0) return LMOE_OK;
    if (!x || !aligned(x, 16)) return LMOE_ERR_INVALID_ARG;
    if ((topk_idx && !aligned(topk_idx, 4)) || (topk_w && !aligned(topk_w, 4)) ||
        (expert_counts && !aligned(expert_counts, 4)))
        return LMOE_ERR_INVALID_ARG;
    Plan p;
    plan_of(h->cfg, T, p);
    // routing touches only the buffers up to the row weights (they come first in the plan)
    const size_t need = p.wperm + al256((size_t)p.A * 4);
    if (need > kNoAllocScratchBytes) return LMOE_ERR_WORKSPACE;
    void* scratch = nullptr;
    lmoe_status s = noalloc_scratch(&scratch);
    if (s != LMOE_OK) return s;
    s = take_device_error(h);
    if (s != LMOE_OK) return s;
    Ctx c = make_ctx(h, p, scratch, stream);
    h->launches = 0;
    s = do_route(c, x, topk_idx, topk_w, expert_counts);  // clears the stats block first
    if (s != LMOE_OK) return s;
    k_publish_error<<<1, 1, 0, c.s>>>(c.err, h->derr);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}
