/*
 * oracle.h -- plain, slow fp64 CPU reference of the LatentMoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library. It shares no code with
 * the CUDA library and must never be used as a fallback for it.
 *
 * Sources (page title, section):
 *   - "Nemotron 3 Ultra 架构 QA", Q5.1: order of the layer (fc1_latent_proj ->
 *     experts -> fc2_latent_proj -> + shared expert on the raw input).
 *   - same page, Q5.2: router logits = fp32 linear of the un-projected hidden
 *     state; scores = sigmoid(logits); choice scores = scores + bias.
 *   - same page, Q5.3: the bias is used for selection only.
 *   - same page, Q5.7: y = fc2(sum_e w_e Expert_e(fc1(x))) + Shared(x).
 *   - same page, Q5.8: top-k weights multiplied by routed_scaling_factor.
 *   - same page, Q2.6: experts are non-gated, act = relu2 = max(0, x)^2.
 *   - same page, Q5.5/Q5.6: expert weights up [E, I, L], down [E, L, I].
 *   - "Nemotron-3-Labs-Ultra-Math-SFT" article, section "路由与共享专家":
 *     sigmoid scoring, top-k within groups, weights normalised then x 5.0,
 *     shared expert applied in parallel to the pre-projection input.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - group score = sum of the two largest choice scores in each contiguous
 *     block of E/G experts; experts outside the kept groups are excluded;
 *   - ties: tau = k-th largest eligible choice score; every expert above
 *     tau + 1e-6 is taken, the rest come from |c - tau| <= 1e-6 in ascending
 *     expert id (same rule for groups, with the Gk-th group score);
 *   - normalisation divides by the plain sum of the selected sigmoid scores;
 *   - rounding points (bf16 mode): x, z, a_e, comb and a_s are rounded to
 *     bf16 (nearest-even) because they are GEMM operands; everything else is
 *     fp64 here; in fp32 validation mode no rounding is applied;
 *   - selected experts are reported in ascending expert id.
 */
#ifndef LMOE_ORACLE_H
#define LMOE_ORACLE_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int H, L, E, k, G, Gk, I, Is;
    double s;       /* routed_scaling_factor */
    int x_f32;      /* 1: x is fp32; 0: x is bf16 (uint16 bits) */
    int fp32_mode;  /* 1: fp32 validation mode, no bf16 rounding of intermediates */
} lmo_cfg;

typedef struct {
    const uint16_t* router_w;      /* [E, H] bf16 */
    const float* e_bias;           /* [E] fp32 */
    const uint16_t* fc1_w;         /* [L, H] */
    const uint16_t* fc2_w;         /* [H, L] */
    const uint16_t* const* up_w;   /* E pointers, each [I, L]; NULL where unused */
    const uint16_t* const* down_w; /* E pointers, each [L, I]; NULL where unused */
    const uint16_t* shared_up_w;   /* [Is, H] */
    const uint16_t* shared_down_w; /* [H, Is] */
    /* Per-expert matrix scales of block-scaled (NVFP4) experts, or NULL (1.0):
     * h = up_gs[e] * (z . W_up[e] row), o = w * down_gs[e] * (a . W_down[e] row),
     * the scale applied to the accumulated product before the activation. */
    const float* up_gs;            /* [E] or NULL */
    const float* down_gs;          /* [E] or NULL */
} lmo_weights;

#define LMO_EPS 1e-6

/* Round to the nearest bf16 value, ties to even (exact result as a double). */
double lmo_round_bf16(double v);

/* Choice of k experts from choice scores c[E] (grouped top-k with the band
 * rule). sel[k] receives expert ids in ascending order. Returns 0 or -1. */
int lmo_select(const lmo_cfg* cfg, const double* c, int32_t* sel);

/* Logits (fp64) for n tokens: out[t, e] = sum_h x[t, h] * W_r[e, h]. */
int lmo_logits(const lmo_cfg* cfg, const void* x, const uint16_t* router_w, int64_t n, double* out);

/* Routing for n tokens: idx[n, k] ascending ids, w[n, k] weights. */
int lmo_route(const lmo_cfg* cfg, const void* x, const uint16_t* router_w, const float* e_bias, int64_t n,
              int32_t* idx, double* w);

/* fc1_latent_proj before its rounding ("Nemotron 3 Ultra 架构 QA", Q5.1; the
 * step z = rho(x^ W_fc1^T) of lmo_forward without rho): out[t, l] =
 * sum_h rho(x[t, h]) W_fc1[l, h] in fp64, for n tokens. */
int lmo_latent(const lmo_cfg* cfg, const void* x, const uint16_t* fc1_w, int64_t n, double* out);

/* Full layer for n tokens. x holds those n rows; y[n, H] fp64. idx/w may be NULL. */
int lmo_forward(const lmo_cfg* cfg, const void* x, const lmo_weights* wts, int64_t n, int32_t* idx, double* w,
                double* y);

/* Pre-norm RMSNorm of the block around the layer ("Nemotron 3 Ultra 架构 QA",
 * Q2.8, the quoted forward; Q2.1: pre-norm + residual around each mixer):
 *   r = 1 / sqrt(mean_h x[h]^2 + eps),  xt = bf16(x * r),  out = bf16(gamma * xt)
 * x and gamma bf16, out bf16 bits; the mean and r in fp64 (the page upcasts). */
int lmo_rmsnorm(int H, const uint16_t* x, const uint16_t* gamma, double eps, int64_t n, uint16_t* out);

/* Block: y = x + layer(rmsnorm(x)) for n tokens (x bf16; y fp64 [n, H]). */
int lmo_forward_block(const lmo_cfg* cfg, const uint16_t* x, const uint16_t* gamma, double eps,
                      const lmo_weights* wts, int64_t n, int32_t* idx, double* w, double* y);

/* Load-balancing bias update ("Nemotron 3 Ultra 架构 QA", Q5.3: the training
 * framework counts the tokens each expert received and moves the bias against
 * the overload): mean = sum(counts) / E,
 *   bias_out[e] = fp32(bias[e] - eta * (counts[e] - mean))      (fp64 inside)
 * and MaxVio (Q5.4, load violation relative to the ideal load)
 *   = (max_e counts[e] - mean) / mean   (0 when no token was routed).
 * bias_out may alias bias. Returns 0. */
int lmo_update_bias(int E, const int32_t* counts, const float* bias, double eta, float* bias_out, double* maxvio);

/* ---- NVFP4 block-scaled expert weights ("Nemotron 3 Ultra 架构 QA", Q1.3 and
 * Q8.1: the 512 experts' up and down weights are the layers kept in NVFP4, the
 * latent projections fc1/fc2 stay BF16; overview page: NVFP4 quantisation for
 * inference). The pages name the format but do not spell it out; this is its
 * public definition:
 *   element  E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa;
 *            magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6
 *   block    16 consecutive elements along K share one E4M3 scale S (finite
 *            variant: bias 7, 3 mantissa bits, subnormals, max 448, no inf)
 *   matrix   one fp32 scale g per matrix (per expert and projection)
 *   value    w = code_value * S * g
 * Quantisation (reading of the usual recipe, all decisions in fp32 with
 * round-to-nearest-even operations):
 *   amax = max |w| of the matrix;  g = amax / 2688 (6 * 448), or 1 if amax = 0
 *   per block: S = E4M3 nearest to (bmax / g) / 6, saturating at 448
 *   per element: q = w / (S * g) (product rounded to fp32 first);
 *                code = E2M1 nearest to q, ties to the even mantissa,
 *                saturating at 6; sign bit = (q < 0); S = 0 gives code 0.
 * Storage (tiles of 128 rows x 64 K; R multiple of 128, K multiple of 64):
 *   global row gr = m * R + r, tile id = (gr / 128) * (K / 64) + k / 64
 *   codes: byte tile*4096 + (gr % 128)*32 + (k % 64)/2, even k in the low nibble
 *   scales: byte tile*512 + (gr % 128)*4 + (k % 64)/16                      */
double lmo_e2m1_value(int code);
double lmo_e4m3_value(int byte);            /* NaN for 0x7F / 0xFF */
int lmo_e2m1_encode(float q);               /* nearest code, ties to even, saturating */
int lmo_e4m3_encode(float u);               /* u >= 0: nearest, ties to even, saturating */
/* n_mat matrices of [R, K] bf16 -> codes, scales (tiled layout) and g[n_mat].
 * Returns 0, or -1 when R % 128 or K % 64 is non-zero. */
int lmo_nvfp4_quantize(const uint16_t* w, int64_t n_mat, int R, int K, uint8_t* codes, uint8_t* sf, float* g);
/* bf16 bits of code_value * S (exact) for the n_mat x R x K elements (g not applied). */
int lmo_nvfp4_dequant(const uint8_t* codes, const uint8_t* sf, int64_t n_mat, int R, int K, uint16_t* out);

#ifdef __cplusplus
}
#endif
#endif
