/*
 * latentmoe.h -- C ABI of the B200 (sm_100a) LatentMoE layer forward.
 *
 * What the layer computes (page "Nemotron 3 Ultra 架构 QA", Q5.1, Q5.2, Q5.7,
 * Q5.8, Q2.6; article "Nemotron-3-Labs-Ultra-Math-SFT", section
 * "LatentMoE 层 / 路由与共享专家"):
 *
 *   logits = x W_r^T (fp32)          sigma = sigmoid(logits)
 *   choice = sigma + e_score_correction_bias        (selection only)
 *   S      = grouped top-k of choice                (n_group, topk_group, top_k)
 *   w_e    = routed_scaling_factor * sigma_e / sum_{j in S} sigma_j
 *   z      = x W_fc1^T                              fc1_latent_proj, H -> L
 *   o_e    = relu(z W_up[e]^T)^2 W_down[e]^T        non-gated relu2 expert, L -> I -> L
 *   y      = (sum_{e in S} w_e o_e) W_fc2^T + relu(x W_su^T)^2 W_sd^T
 *
 * Ties: tau = k-th largest eligible choice score; every expert above
 * tau + 1e-6 is taken and the remaining slots go to |choice - tau| <= 1e-6 in
 * ascending expert id (same rule for groups, group score = sum of the two
 * largest choice scores of the group's E/G contiguous experts).
 *
 * Layouts: row-major, nn.Linear [out, in]. Expert weights are one tensor each,
 * up [E, I, L] and down [E, L, I] (page "Nemotron 3 Ultra 架构 QA", Q5.6).
 * All weights are bf16; e_bias is fp32. x is bf16 or fp32 ([T, H]); y is
 * fp32 [T, H]. Every pointer is device memory owned by the caller and must be
 * 16-byte aligned. H, L, I and Is must be multiples of 64.
 *
 * Modes: LMOE_MODE_BF16 feeds bf16 operands to tensor-core GEMMs with fp32
 * accumulation (z, the expert activations, the weighted sum and the shared
 * activations are rounded to bf16 as GEMM operands; z, which every routed
 * expert of a token reads, is re-rounded so that it equals the exact rounding
 * of x W_fc1^T whenever the fp32 error of an element is below the margin of
 * LMOE_OPT_Z_RECHECK_DELTA, and the expert and shared-expert activations with
 * h above LMOE_OPT_ACT_RECHECK_TAU likewise);
 * LMOE_MODE_FP32 is a validation mode with fp32 operands and no intermediate
 * rounding.
 *
 * Errors: every argument is validated before anything is launched; on
 * LMOE_ERR_INVALID_ARG / _WORKSPACE / _UNSUPPORTED no output is touched. The
 * library never synchronises the caller's stream and never aborts. A device
 * wait that exceeds its bound makes the kernel record LMOE_ERR_TIMEOUT in
 * host-visible memory and return; the call that launched it, or the next call
 * on the handle, returns LMOE_ERR_TIMEOUT. Launch failures return
 * LMOE_ERR_CUDA. T = 0 returns LMOE_OK and launches nothing.
 *
 * Streams: calls are asynchronous on the caller's stream. latentmoe_forward,
 * latentmoe_forward_block and latentmoe_ep_front also use a second stream the
 * handle owns (created by latentmoe_create on the device current then): within
 * the call the routing kernels are forked onto it after the input GEMM and
 * joined back into the caller's stream before the first kernel that reads
 * their outputs, so work enqueued afterwards on the caller's stream sees the
 * call complete. These calls can be captured into a CUDA graph. A handle's
 * calls must not be issued from several host threads at once; calls from one
 * thread on different streams are correct, and their routing kernels run in
 * turn on the handle's stream.
 *
 * Determinism: the same inputs give bitwise-identical outputs (no floating-
 * point atomics; sums run in a fixed order).
 */
#ifndef LATENTMOE_H
#define LATENTMOE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LMOE_OK = 0,
    LMOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or shape      */
    LMOE_ERR_UNSUPPORTED = 2,  /* shape outside what the kernels implement        */
    LMOE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required       */
    LMOE_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed      */
    LMOE_ERR_TIMEOUT = 5,      /* a bounded device wait ran out                    */
    LMOE_ERR_INTERNAL = 6
} lmoe_status;

typedef enum { LMOE_BF16 = 0, LMOE_FP32 = 1 } lmoe_dtype;
typedef enum { LMOE_MODE_BF16 = 0, LMOE_MODE_FP32 = 1 } lmoe_mode;
/* Storage of the routed experts' up/down weights. NVFP4 ("Nemotron 3 Ultra 架构
 * QA", Q1.3 and Q8.1: the experts' up and down projections are the NVFP4
 * layers, the latent projections, router and shared expert stay BF16): see
 * latentmoe_quantize_nvfp4 for the format and the tiled layout. */
typedef enum { LMOE_EXPERTS_BF16 = 0, LMOE_EXPERTS_NVFP4 = 1 } lmoe_expert_format;

typedef struct {
    int hidden;              /* H (multiple of 64)                               */
    int latent;              /* L = moe_latent_size (multiple of 64)             */
    int num_experts;         /* E = n_routed_experts                             */
    int top_k;               /* k = num_experts_per_tok                          */
    int n_group;             /* G; E % G == 0; G <= 32                           */
    int topk_group;          /* Gk <= G                                          */
    int expert_inter;        /* I = moe_intermediate_size (multiple of 64)       */
    int shared_inter;        /* Is = moe_shared_expert_intermediate_size (x64)   */
    int max_tokens;          /* largest T a call may pass                        */
    float routed_scaling_factor;
    lmoe_dtype x_dtype;      /* dtype of x                                       */
    lmoe_mode mode;          /* BF16 (tensor cores) or FP32 (validation)         */
    lmoe_expert_format expert_format;  /* BF16 (default) or NVFP4               */
    int local_experts;       /* expert parallelism: experts whose up/down weights
                                this handle holds (0 = all E)                     */
    int expert_base;         /* first of them (global expert id)                  */
} lmoe_config;
/* Supported: E <= 1024, k <= min(64, Gk * E / G), E / G >= 2 when G > 1.
 * NVFP4 experts: mode LMOE_MODE_BF16, I and L multiples of 128. */

typedef struct {
    const void* router_w;       /* [E, H]  bf16                                   */
    const float* e_bias;        /* [E]     fp32 e_score_correction_bias           */
    const void* fc1_w;          /* [L, H]  bf16 fc1_latent_proj                   */
    const void* fc2_w;          /* [H, L]  bf16 fc2_latent_proj                   */
    const void* up_w;           /* [E, I, L] bf16 expert up_proj                  */
    const void* down_w;         /* [E, L, I] bf16 expert down_proj                */
    const void* shared_up_w;    /* [Is, H] bf16 shared expert up_proj             */
    const void* shared_down_w;  /* [H, Is] bf16 shared expert down_proj           */
    /* NVFP4 experts only (expert_format = LMOE_EXPERTS_NVFP4; ignored otherwise):
     * up_w and down_w then hold E2M1 codes, E*I*L/2 bytes each, in the tiled
     * layout of latentmoe_quantize_nvfp4 (up: E matrices of [I, L]; down: E
     * matrices of [L, I]), and these hold their scales.                        */
    const void* up_sf;          /* E4M3 block scales of up_w, E*I*L/16 bytes      */
    const void* down_sf;        /* E4M3 block scales of down_w, E*L*I/16 bytes    */
    const float* up_gs;         /* [E] fp32 matrix scale of each expert's up_w    */
    const float* down_gs;       /* [E] fp32 matrix scale of each expert's down_w  */
} lmoe_weights;

typedef struct lmoe_handle lmoe_handle;

/* Validates the configuration, records the (borrowed) weight pointers and
 * pre-encodes the weight TMA descriptors. Allocates no device memory; the
 * weights must outlive the handle. *out is set only on LMOE_OK. */
lmoe_status latentmoe_create(const lmoe_config* cfg, const lmoe_weights* w, lmoe_handle** out);

/* Bytes of device workspace a call with T tokens needs (T <= max_tokens). */
lmoe_status latentmoe_workspace_size(const lmoe_handle* h, int T, size_t* bytes);

/* Routing only: topk_idx [T, k] int32 (ascending expert id per token),
 * topk_w [T, k] fp32 (normalised and scaled), expert_counts [E] int32
 * (tokens routed to each expert). Any output may be NULL. */
lmoe_status latentmoe_route(lmoe_handle* h, const void* x, int T, int32_t* topk_idx, float* topk_w,
                            int32_t* expert_counts, void* ws, size_t ws_bytes, void* stream);

/* Full layer: y [T, H] fp32. The routing outputs are optional (NULL = not
 * returned). ws must be at least latentmoe_workspace_size(T) bytes, 256-byte
 * aligned, and not in use by another call in flight. */
lmoe_status latentmoe_forward(lmoe_handle* h, const void* x, int T, float* y, void* ws, size_t ws_bytes,
                              void* stream, int32_t* topk_idx, float* topk_w, int32_t* expert_counts);

/* The layer inside its pre-norm residual block ("Nemotron 3 Ultra 架构 QA",
 * Q2.1: each mixer sits behind a pre-norm and a residual; Q2.8: the RMSNorm
 * upcasts, multiplies by rsqrt(mean(x^2) + eps), rounds back, scales by gamma):
 *   xn = bf16(gamma * bf16(x / sqrt(mean_h x^2 + eps)))      (fp64 inside)
 *   y  = x + layer(xn)                                         (fp32)
 * x [T, H] bf16 (the handle must have x_dtype LMOE_BF16, else
 * LMOE_ERR_UNSUPPORTED), norm_w = gamma [H] bf16, norm_eps >= 0 (1e-5 on the
 * pages). Same workspace and optional routing outputs as latentmoe_forward;
 * the routing is that of xn. */
lmoe_status latentmoe_forward_block(lmoe_handle* h, const void* x, int T, const void* norm_w, float norm_eps,
                                    float* y, void* ws, size_t ws_bytes, void* stream, int32_t* topk_idx,
                                    float* topk_w, int32_t* expert_counts);

/* NVFP4 quantisation of n_mat bf16 matrices [R, K] (w, row-major, contiguous;
 * e.g. all E expert up_proj weights with R = I, K = L). Format: E2M1 elements
 * (bit 3 sign, 2 exponent bits with bias 1, 1 mantissa bit: 0, 0.5, 1, 1.5, 2,
 * 3, 4, 6), one E4M3 scale S per 16 consecutive elements along K (bias 7,
 * 3 mantissa bits, subnormals, max 448), one fp32 scale g per matrix; the
 * element's value is code * S * g. Recipe, every step an fp32 operation
 * rounded to nearest even:
 *   g = amax(matrix) / 2688 (1 if the matrix is zero)
 *   S = nearest E4M3 to (amax(block) / g) / 6, saturating at 448
 *   code = nearest E2M1 to w / (S * g), ties to the even mantissa, saturating
 *          at 6, sign bit = (w / (S * g) < 0); a block with S = 0 gets code 0.
 * Layout, in tiles of 128 rows x 64 K (gr = m * R + r is the global row):
 *   tile = (gr / 128) * (K / 64) + k / 64
 *   codes[tile * 4096 + (gr % 128) * 32 + (k % 64) / 2], element k even in
 *   the low nibble;  sf[tile * 512 + (gr % 128) * 4 + (k % 64) / 16].
 * codes (n_mat*R*K/2 bytes), sf (n_mat*R*K/16 bytes) and gs ([n_mat] fp32)
 * are device memory written by the call; w, codes and sf 16-byte aligned.
 * R % 128 == 0 and K % 64 == 0, else LMOE_ERR_UNSUPPORTED. Asynchronous on
 * `stream`; deterministic. Needs no handle: a weight-conversion step run once
 * before latentmoe_create. */
lmoe_status latentmoe_quantize_nvfp4(const void* w, long long n_mat, int R, int K, void* codes, void* sf, float* gs,
                                     void* stream);

/* ---- Expert parallelism --------------------------------------------------
 * The layer split into the three stages around the exchange of expert
 * parallelism ("Nemotron-3-Labs-Ultra-Math-SFT" article: section 什么是 Latent
 * 瓶颈, the experts exchange 2048-wide latent rows, a quarter of the hidden
 * width, to cut the traffic of multi-GPU expert parallelism; deployment notes:
 * the 512 experts sharded over the GPUs). The experts are partitioned
 * over P ranks in contiguous blocks of E/P ids; each rank's handle holds the
 * router, fc1/fc2 and the shared expert in full and the up/down weights of its
 * own block only (local_experts = E/P, expert_base = rank * E/P). Per forward:
 *   1 latentmoe_ep_front   routing, z = fc1(x), a_s, and the rows of z in
 *                          expert order (send_rows [T*k, L] bf16) with their
 *                          routing weights (send_w [T*k] fp32) and the
 *                          per-expert counts [E]; rows for rank r are the
 *                          rows of experts r*E/P .. (r+1)*E/P-1, contiguous.
 *   (caller) exchange counts and rows all-to-all (rows of source s arrive in
 *            expert order; recv_counts [n_src, local_experts] int32)
 *   2 latentmoe_ep_experts the local experts on the received rows in their
 *                          arrival order: recv_o = w * down(relu2(up(row)))
 *                          [n_rows, L] fp32, same order (the weights are
 *                          applied here, as in the single-GPU path)
 *   (caller) return recv_o to the sources all-to-all (in the order they sent)
 *   3 latentmoe_ep_back    combine the k returned rows of each token in
 *                          ascending expert id, y = comb W_fc2^T + a_s W_sd^T
 * Steps 1 and 3 use the same workspace (sized by latentmoe_workspace_size(T)),
 * which carries the permutation and a_s between them; step 2 its own
 * (latentmoe_ep_workspace_size). With P = 1 the three steps give the same y
 * bit for bit as latentmoe_forward. All pointers are device memory. */
lmoe_status latentmoe_ep_front(lmoe_handle* h, const void* x, int T, void* send_rows, float* send_w,
                               int32_t* expert_counts, void* ws, size_t ws_bytes, void* stream);
/* recv_counts: device int32 [n_src * local_experts] (source-major); n_rows =
 * their sum; n_src * local_experts <= 1024. */
lmoe_status latentmoe_ep_workspace_size(const lmoe_handle* h, int n_rows, int n_src, size_t* bytes);
lmoe_status latentmoe_ep_experts(lmoe_handle* h, const void* recv_rows, const float* recv_w,
                                 const int32_t* recv_counts, int n_src, int n_rows, float* recv_o, void* ws,
                                 size_t ws_bytes, void* stream);
/* send_o: [T*k, L] fp32, row i = the result for send_rows row i. */
lmoe_status latentmoe_ep_back(lmoe_handle* h, const float* send_o, int T, float* y, void* ws, size_t ws_bytes,
                              void* stream);

/* Releases the handle (host memory only). */
void latentmoe_destroy(lmoe_handle* h);

const char* latentmoe_status_string(lmoe_status s);

/* Load-balancing step for the bias the router adds to its choice scores
 * ("Nemotron 3 Ultra 架构 QA", Q5.3: the training framework counts the tokens
 * each expert received and lowers the bias of overloaded experts; Q5.4 reports
 * MaxVio). With mean = sum(expert_counts) / E, in fp64:
 *   bias_out[e] = fp32(bias_in[e] - eta * (expert_counts[e] - mean))
 *   *maxvio_out = (max_e expert_counts[e] - mean) / mean   (0 if no token)
 * expert_counts [E] int32 (e.g. the counts latentmoe_route/forward return),
 * bias_in/bias_out [E] fp32, maxvio_out one double (may be NULL); all device
 * memory. bias_out may alias bias_in, including the handle's own e_bias: the
 * handle reads the bias through its pointer, so the next call uses it.
 * Asynchronous on `stream`. */
lmoe_status latentmoe_update_bias(lmoe_handle* h, const int32_t* expert_counts, const float* bias_in, float eta,
                                  float* bias_out, double* maxvio_out, void* stream);

/* ---- diagnostics --------------------------------------------------------- */
typedef enum {
    LMOE_OPT_GEMM_PATH = 0,      /* 0 auto, 1 tcgen05 prefill tiles (128 x BN per SM), 2 tcgen05
                                    decode (swap-AB) tiles, 3 SIMT fp32 kernels (validation),
                                    4 prefill tiles of 256 x 256 on 2-SM pairs (cta_group::2).
                                    NVFP4 expert GEMMs always run weight-stationary tiles (32
                                    tokens at decode sizes, else 128); the option then applies to
                                    the dense GEMMs, and 3 is unsupported (LMOE_ERR_UNSUPPORTED). */
    LMOE_OPT_ROUTER_FP64_ALL = 1,/* 1: every token's logits recomputed in fp64 (validation)      */
    LMOE_OPT_FLAG_DELTA = 2,     /* near-edge margin delta of the fp64 re-check, in 1e-9 units
                                    (default 20000 = 2e-5): a token is re-decided from exact
                                    fp64 logits when its k-th / (k+1)-th fp32 choice-score gap
                                    is within 1e-6 + delta (group scores: 1e-6 + 2 delta); the
                                    routing is exact whenever every fp32 choice score is within
                                    delta / 2 of its exact value                               */
    LMOE_OPT_SPIN_LIMIT = 3,     /* bound on device mbarrier polls before LMOE_ERR_TIMEOUT        */
    LMOE_OPT_Z_RECHECK_DELTA = 4,/* margin scale d of the exact re-rounding of z, in 1e-9 units
                                    (default 6000 = 6e-6; 0 disables). bf16 mode: the fc1
                                    product is kept in fp32, rounded to bf16 nearest-even, and
                                    every element whose fp32 value lies within d (1 + 0.4 |z|) of
                                    a bf16 rounding midpoint is recomputed as an error-free sum
                                    of the exact bf16 products and rounded again, so z is the
                                    exactly rounded x W_fc1^T whenever the fp32 error of each
                                    element is below its margin (z is the rounding point that
                                    every routed expert of a token reads). Valid 0 .. 1e8. */
    LMOE_OPT_ACT_RECHECK_TAU = 5 /* threshold tau of the exact re-rounding of the relu2
                                    activations (expert and shared-expert up projections), in
                                    1e-3 units (default 2000 = 2.0; 0 disables; values from 1
                                    to 499 are refused: below tau = 0.5 the list, sized at
                                    create, could not hold every activation the test can list,
                                    whatever the inputs). bf16 mode,
                                    bf16 experts: an activation a = max(h, 0)^2 with h > tau whose
                                    fp32 value lies within the fp32 accumulation error of h
                                    (1.6e-6 + 0.9e-6 h, carried through the square) of a bf16
                                    rounding midpoint is recomputed exactly. A flipped rounding
                                    moves the output by about one bf16 step of a, which grows as
                                    h^2, so the large activations carry most of that error. */
} lmoe_option;
lmoe_status latentmoe_set_option(lmoe_handle* h, lmoe_option opt, long long value);

typedef struct {
    int flagged_tokens;     /* tokens whose routing was re-decided in fp64      */
    int distinct_experts;   /* experts with at least one token                  */
    int max_expert_tokens;  /* largest per-expert token count                   */
    int device_error;       /* lmoe_status recorded by a device-side check      */
    int kernel_launches;    /* kernels the last route/forward call on the handle launched */
    int cuda_error;         /* cudaError_t of the last CUDA runtime call on the handle that
                               failed (a call that returned LMOE_ERR_CUDA), 0 if none     */
    int z_rechecked;        /* z elements listed and re-rounded exactly (LMOE_OPT_Z_RECHECK_DELTA);
                               the list has room for all T*L elements                    */
    int ae_rechecked;       /* expert activations listed for exact re-rounding
                               (LMOE_OPT_ACT_RECHECK_TAU); the list has room for every
                               activation the test can list at any accepted tau (about
                               0.5% of max(T*Is, T*top_k*expert_inter))                 */
    int as_rechecked;       /* shared-expert activations listed, same list room          */
} lmoe_stats;
/* Reads the statistics of the last call that used ws (synchronises the device;
 * for tests and benchmarks, not for the hot path). */
lmoe_status latentmoe_read_stats(const lmoe_handle* h, const void* ws, lmoe_stats* out);

/* Byte offsets, from the start of a call's workspace, of intermediate buffers
 * that tests and tools read back after a call on T tokens (a diagnostic: the
 * layout may change between versions). logits_f32 [T, E] fp32 router logits
 * (latentmoe_route/forward); z_f32 [T, L] fp32 fc1 product before rounding
 * (bf16 mode with z re-rounding on, valid after latentmoe_ep_front: a forward
 * overwrites it with the expert outputs); z [T, L] bf16 latent after
 * re-rounding; flag_list: int32 ids of the tokens re-decided in fp64
 * (lmoe_stats.flagged_tokens of them); perm [T*k] int32: token of each row in
 * expert order; slot [T, k] int32: row in expert order of each (token, j);
 * total = latentmoe_workspace_size(T); offsets [E + 1] int32: first row of
 * each expert in expert order; act_e [T*k, I] bf16 expert activations
 * relu2(z W_up^T) in expert order and act_s [T, Is] bf16 shared-expert
 * activations (bf16 mode, after latentmoe_forward). */
typedef struct {
    size_t logits_f32, z_f32, z, flag_list, perm, slot, total, offsets, act_e, act_s;
} lmoe_ws_layout;
lmoe_status latentmoe_workspace_layout(const lmoe_handle* h, int T, lmoe_ws_layout* out);

/* Routing for callers that cannot allocate device memory (a real-time or
 * latency-critical section where cudaMalloc's implicit synchronisation is not
 * allowed, a runtime whose device memory belongs to a fixed arena, a plugin
 * host that forbids allocation from extension code). Same outputs as
 * latentmoe_route, but there is no workspace argument and the call allocates
 * nothing: its scratch is an 8 MiB array in this library's static device
 * memory, held by every GPU that loads the library until the process exits.
 * The pages have no counterpart of this entry point.
 *  - Capacity: routing needs about 6.5 KiB per token at E = 512, k = 22, so
 *    T up to roughly 1200 tokens fits at the Ultra shape; a T whose scratch
 *    need exceeds 8 MiB returns LMOE_ERR_WORKSPACE and launches nothing.
 *  - The first call on each device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; each call clears what must start at zero. Calls whose GPU work
 *    overlaps (other streams, other threads, other handles) race on it:
 *    order them on one stream or synchronise between them.
 * The handle comes from latentmoe_create as usual. */
lmoe_status latentmoe_route_noalloc(lmoe_handle* h, const void* x, int T, int32_t* topk_idx, float* topk_w,
                                    int32_t* expert_counts, void* stream);

/* Stage markers for timing inside a real call: when set (n >= 8), the next
 * latentmoe_forward calls record events[i] (cudaEvent_t) on their stream at
 * stage boundary i: 0 start, 1 routing head done (the statistics reset, and
 * the router GEMM when it cannot be the first problem of the input GEMM
 * launch), 2 input stage done (the input GEMM; selection, fp64 re-check and
 * permutation on the second stream; the exact re-roundings of z and a_s),
 * 3 gather done, 4 expert up GEMM done, 5 expert down GEMM done, 6 combine
 * done, 7 output GEMM done. NULL turns it off. The events are borrowed and must exist (a
 * NULL event among the first 8 returns LMOE_ERR_INVALID_ARG); a record that
 * fails is skipped and does not fail the call it times. */
lmoe_status latentmoe_set_profile_events(lmoe_handle* h, void* const* events, int n);

/* Runs one kernel that waits, with the handle's spin limit, on an mbarrier
 * that nothing ever completes, and returns the status it reports
 * (LMOE_ERR_TIMEOUT when the bounded wait works). Synchronises the device. */
lmoe_status latentmoe_selftest_bounded_wait(lmoe_handle* h);

#ifdef __cplusplus
}
#endif
#endif
