// lmoe_internal.h -- structures shared by the host entry points and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/latentmoe.h"

#ifndef LMOE_CHECKS
#define LMOE_CHECKS 0  // 1: the checking build (device-side bounds checks, see lmoe_check)
#endif

namespace lmoe {

// Device-side bounds check of the checking build (LMOE_CHECKS=1): a false
// condition records LMOE_ERR_INVALID_ARG in the call's error word and the
// caller skips the access it guards. In the default build it is always true
// and compiles away.
__device__ __forceinline__ bool lmoe_check(bool ok, int* err) {
#if LMOE_CHECKS
    if (!ok) atomicCAS(err, 0, 1);
    return ok;
#else
    (void)err;
    return true;
#endif
}

constexpr int kBM = 128;          // tensor-core tile rows (MMA M)
constexpr int kBK = 64;           // K elements per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kSimtBM = 64;       // SIMT validation kernels tile rows
constexpr int kDecodeTN = 32;     // token tile of the swap-AB decode variant (MMA N)
constexpr int kMaxProblems = 3;   // dense problems in one GEMM launch (router, fc1, shared up)
constexpr int kMaxTensorMaps = 8; // tensor maps in one GEMM launch
constexpr float kBandEps = 1e-6f; // tie band of the routing rule
constexpr int kMaxK = 64;
constexpr int kMaxE = 1024;
constexpr int kMaxG = 32;

// Small block at the head of the workspace.
struct WsStats {
    int flagged;        // tokens appended to the fp64 re-check list
    int distinct;       // experts with at least one token
    int max_count;      // largest per-expert count
    int device_error;   // lmoe_status from a device check
    int zflagged;       // z elements listed for the exact re-rounding
    int aeflagged;      // expert activations listed for the exact re-rounding
    int asflagged;      // shared-expert activations listed for the exact re-rounding
    int zrows;          // row segments of z with listed elements (entries of the row table)
    int pad[56];
};

// Epilogue kinds of the GEMM kernels.
enum Epi : int {
    EPI_F32 = 0,        // out fp32 = acc
    EPI_BF16 = 1,       // out bf16 = acc
    EPI_RELU2_BF16 = 2, // out bf16 = relu(acc)^2
    EPI_SCALE_F32 = 3,  // out fp32 = row_scale[row] * acc
    EPI_RELU2_F32 = 4,  // out fp32 = relu(acc)^2 (validation mode)
};

// One GEMM problem: out[m, n] = epi(sum_k A[m, k] B[n, k]) over up to two
// K segments (segment 1 continues the same accumulator: K concatenation).
// Dense problems have m_rows rows; grouped problems take their row ranges
// from offsets[E+1] and B rows from expert e's block (b_rows_per_expert).
struct GemmProblem {
    int grouped;            // 0 dense, 1 grouped by expert
    int m_rows;             // dense only
    int n;                  // N (columns of out)
    int nseg;               // 1 or 2
    int kdim[2];            // K of each segment
    int a_map[2], b_map[2]; // tensor-map indices (tensor-core path)
    const void* a_ptr[2];   // operand pointers (SIMT path); A row stride = kdim[s]
    const void* b_ptr[2];   // B row stride = kdim[s]
    int b_rows_per_expert;  // grouped: rows of B per expert
    int epi;
    void* out;
    long long ldo;          // elements
    const float* row_scale; // EPI_SCALE_F32
    int out_map;            // tensor map of `out` for bulk tensor stores (-1: plain stores)
    const uint16_t* resid;  // EPI_F32 only: bf16 [rows, ldo] added to the result (block residual)
    // NVFP4 weights (grouped swap-AB problems only): B is given as E2M1 codes and
    // E4M3 block scales in 128-row x 64-K tiles, and each expert's accumulator is
    // multiplied by wscale[e] before the epilogue operation.
    const uint8_t* wq_codes;  // tile t at wq_codes + 4096 t
    const uint8_t* wq_sf;     // tile t at wq_sf + 512 t
    const float* wscale;      // [E] matrix scale per expert
    // Grouped problems: when non-zero, group g uses the weights of expert
    // g % expert_mod (expert parallelism: groups are (source rank, local expert)
    // blocks of received rows in arrival order).
    int expert_mod;
    // K accumulated per TMEM chunk, in k-blocks (0: the engine's default).
    int chunk_kb;
    // Exact re-rounding list of a relu2 bf16 output (rr_list non-null): every
    // activation a = max(h, 0)^2 above rr_tau2_bits (the fp32 pattern of tau^2)
    // whose fp32 value lies within rr_ulps fp32 ulps of a bf16 rounding midpoint
    // is appended as (row, weight row) for an exact recomputation (rr_flag).
    int2* rr_list;
    int* rr_count;
    int rr_cap;
    uint32_t rr_tau2_bits, rr_ulps;
};

// Accumulation-error margin c0 + c1 h of a relu2 pre-activation h, and the
// smallest threshold the exact re-rounding of the activations accepts (below it
// the margin, over a's fp32 ulp, grows as 1/tau^2 and the list would have to
// be much larger).
constexpr double kActC0 = 1.6e-6, kActC1 = 0.9e-6, kActTauMin = 0.5;
// rr_flag's margin in fp32 ulps of a = h^2 at its largest relative size (a = tau^2).
inline uint32_t act_margin_ulps(double tau, double c0, double c1) {
    const double u = 16777216.0 * (c0 / (tau * tau) + c0 + 2.0 * c1);
    return u >= 16384.0 ? 0x4000u : (uint32_t)u + 1u;
}
// List room that holds every activation rr_flag can list out of n, for any
// tau >= kActTauMin: a listed value has its low 16 bits in a window of
// 2 * ulps of the 65536 patterns around 0x8000, and the window's share is
// largest at the smallest tau.
inline size_t act_list_room(size_t n) {
    const size_t w = 2u * act_margin_ulps(kActTauMin, kActC0, kActC1);
    return n / 65536 * w + ((n % 65536) * w + 65535) / 65536 + 64;
}

// Whether a = max(h, 0)^2, computed in fp32, is above tau^2 and within `ulps`
// fp32 ulps of a bf16 rounding midpoint. For a positive fp32 value the bf16
// values are the patterns with zero low 16 bits and the only midpoint between
// two of them has low bits 0x8000, so the distance in ulps is |low16 - 0x8000|.
// The host derives `ulps` from the accumulation-error margin of h (c0 + c1 h,
// carried through the square: about 2h (c0 + c1 h) <= c0 + (c0 + 2 c1) a, with
// h <= (a + 1) / 2) and from ulp(a) >= a 2^-24, so the test lists every
// element the margin asks for and at most a few times more.
__device__ __forceinline__ bool rr_flag(float a, uint32_t tau2_bits, uint32_t ulps) {
    const uint32_t u = __float_as_uint(a);
    return u > tau2_bits && (u & 0xFFFFu) - (0x8000u - ulps) < 2u * ulps;
}

// Lists one element for re-rounding (rare: a handful per tile). Entries past the
// list's room are counted, not written.
static __device__ __noinline__ void rr_append(const GemmProblem& pr, int row, int wrow) {
    const int pos = atomicAdd(pr.rr_count, 1);
    if (pos < pr.rr_cap) pr.rr_list[pos] = make_int2(row, wrow);
}

struct DeviceRouting {
    const int* offsets;     // [E+1] permuted row offset of each expert
    const int* pfx128;      // [E+1] prefix of ceil(count/128)
    const int* pfx64;       // [E+1] prefix of ceil(count/64)
    const int* pfxdec;      // [E+1] prefix of ceil(count/kDecodeTN)
    const int* pfx256;      // [E+1] prefix of ceil(count/256) (2-SM pair tiles)
    // Tile records per activation-tile height R = 32, 64, 128, 256: entry j of
    // recR is {expert, first permuted row, rows, 0} of the j-th R-row tile in
    // expert order (pfxR[E] entries), so a GEMM finds its tile with one load.
    const int4* rec32;
    const int4* rec64;
    const int4* rec128;
    const int4* rec256;
    int E;
};

// Workspace carving for one call.
struct Plan {
    size_t total;
    size_t stats, logits, logits64, flaglist, idx, wgt, counts, offsets, pfx128, pfx64, pfxdec, pfx256, rec32, rec64,
        rec128, rec256, blockcounts, perm, slot, wperm, xbf, xnorm, z, zperm, aperm, o, comb, as, zlist, alist, zrowtab;
    int alist_cap;  // entries of the activation re-rounding list
    int T, A, nblk;
};

}  // namespace lmoe

// ---- launchers (all asynchronous on `stream`; return cudaError_t) ----------
struct lmoe_handle;
namespace lmoe {
cudaError_t launch_convert_x(const float* x, uint16_t* xb, long long n, int sms, cudaStream_t s);
cudaError_t launch_router_select(const lmoe_handle* h, const Plan& p, char* ws, bool fp64_all, cudaStream_t s);
cudaError_t launch_router_logits64(const lmoe_handle* h, const void* x, const Plan& p, char* ws, bool all,
                                   cudaStream_t s);
cudaError_t launch_router_select64(const lmoe_handle* h, const Plan& p, char* ws, bool all, cudaStream_t s);
cudaError_t launch_permute(const lmoe_handle* h, const Plan& p, char* ws, int32_t* counts_out, cudaStream_t s);
cudaError_t launch_group_scan(int* blockcounts, int nb, int n_rows, int* counts, int* offsets, int* pfx128, int* pfx64,
                              int* pfxdec, int* pfx256, int4* rec32, int4* rec64, int4* rec128, int4* rec256,
                              WsStats* st, cudaStream_t s);
cudaError_t launch_z_round_flag(const float* z32, uint16_t* z, int rows, int L, float m0, float m1, int2* list, int cap,
                                int* count, int4* rowtab, int* nrowtab, int sms, cudaStream_t s);
cudaError_t launch_recheck_rows(const uint16_t* A, int a_rows, const uint16_t* W, int w_rows, int K, int* err,
                                const int2* list, int cap, const int4* rowtab, const int* nrowtab, uint16_t* out,
                                int ldo, int sms, cudaStream_t s);
cudaError_t launch_recheck(bool relu2, const uint16_t* A, int a_rows, const uint16_t* W, int w_rows, int K, int* err,
                           const int2* list, const int* count, int cap, uint16_t* out, int ldo, int sms, cudaStream_t s);
cudaError_t launch_gather_rows(const void* src, int src_rows, int* err, void* dst, const int* perm, int rows_total_max,
                               const int* offsets_E,
                               int row_bytes, int sms, cudaStream_t s);
cudaError_t launch_combine(const float* o, int o_rows, int* err, const int* slot, void* comb, int T, int k, int L,
                           bool out_bf16, int sms, cudaStream_t s);
cudaError_t launch_rmsnorm(const uint16_t* x, const uint16_t* gamma, double eps, int T, int H, uint16_t* out, int sms, cudaStream_t s);
cudaError_t launch_update_bias(const int32_t* counts, const float* bias_in, int E, double eta, float* bias_out,
                               double* maxvio, cudaStream_t s);
cudaError_t launch_copy_routing(const int* idx, const float* w, int32_t* idx_out, float* w_out, long long n, int sms, cudaStream_t s);
cudaError_t launch_gemm_simt(const GemmProblem* probs, int nprob, bool a_f32, const DeviceRouting& r, int max_rows,
                             cudaStream_t s);
cudaError_t launch_gemm_tc(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                           const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s);
cudaError_t launch_gemm_tc_pair(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob,
                                const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s);
// bn: tokens per tile, kDecodeTN or (dense problems of at most 64 rows) 64.
cudaError_t launch_gemm_tc_decode(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                                  const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s);
cudaError_t launch_gemm_tc_nvfp4(const CUtensorMap* maps, int nmaps, const GemmProblem* probs, int nprob, int bn,
                                 const DeviceRouting& r, int* err, unsigned spin_limit, cudaStream_t s);
cudaError_t launch_quantize_nvfp4(const uint16_t* w, long long n_mat, int R, int K, uint8_t* codes, uint8_t* sf,
                                  float* gs, cudaStream_t s);
cudaError_t launch_selftest_wait(int* err, unsigned spin_limit, cudaStream_t s);
int tc_num_sms();
}  // namespace lmoe
