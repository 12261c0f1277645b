/*
 * oracle.c -- plain fp64 CPU reference of the LatentMoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h): loops written straight from the
 * layer's definition, OpenMP over tokens, no blocking or fusion. Every
 * function names the passage it follows.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

static inline double bf(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static inline double x_at(const lmo_cfg* c, const void* x, int64_t t, int64_t h) {
    if (c->x_f32) return (double)((const float*)x)[t * c->H + h];
    return bf(((const uint16_t*)x)[t * c->H + h]);
}

/* Nearest bf16 (8 significant bits), ties to even: v = m * 2^e with
 * |m| in [0.5, 1); keep 8 bits of m with rint (round-half-even). Values below
 * the normal range are quantised on the bf16 subnormal grid 2^-133. */
double lmo_round_bf16(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    frexp(v, &e);
    int q = e - 8;
    if (q < -133) q = -133;
    return ldexp(rint(ldexp(v, -q)), q);
}

static inline double rho(const lmo_cfg* c, double v) { return c->fp32_mode ? v : lmo_round_bf16(v); }

static int cmp_desc(const void* a, const void* b) {
    double x = *(const double*)a, y = *(const double*)b;
    return (x < y) - (x > y);
}

/* Band top-k: choose k of the n candidates cand[] (ascending ids) by value v[].
 * tau is the k-th largest value; everything above tau + eps is taken, the rest
 * is filled from |v - tau| <= eps in ascending id. chosen[i] marks cand[i]. */
static void band_topk(const double* v, const int* cand, int n, int k, char* chosen) {
    double* tmp = (double*)malloc(sizeof(double) * (size_t)n);
    for (int i = 0; i < n; ++i) tmp[i] = v[cand[i]];
    qsort(tmp, (size_t)n, sizeof(double), cmp_desc);
    double tau = tmp[k - 1];
    free(tmp);
    int m = 0;
    for (int i = 0; i < n; ++i) {
        chosen[i] = v[cand[i]] > tau + LMO_EPS;
        m += chosen[i];
    }
    for (int i = 0; i < n && m < k; ++i)
        if (!chosen[i] && fabs(v[cand[i]] - tau) <= LMO_EPS) {
            chosen[i] = 1;
            ++m;
        }
}

/* Grouped top-k ("Nemotron-3-Labs-Ultra-Math-SFT" article, section
 * "路由与共享专家": top-k within groups on the bias-corrected sigmoid score).
 * Group score = sum of the two largest c in the group; keep Gk groups; then
 * k experts among the kept groups. */
int lmo_select(const lmo_cfg* cfg, const double* c, int32_t* sel) {
    const int E = cfg->E, G = cfg->G, Gk = cfg->Gk, k = cfg->k;
    if (G < 1 || G > 1024 || E % G || Gk < 1 || Gk > G || k < 1 || k > 512 || k > Gk * (E / G)) return -1;
    const int per = E / G;
    int* cand = (int*)malloc(sizeof(int) * (size_t)E);
    char* chosen = (char*)malloc((size_t)E);
    int n = 0;
    if (G == 1) {
        for (int e = 0; e < E; ++e) cand[n++] = e;
    } else {
        if (per < 2) {
            free(cand);
            free(chosen);
            return -1;
        }
        double gs[1024];
        int gid[1024];
        char gkeep[1024];
        for (int g = 0; g < G; ++g) {
            double a = -INFINITY, b = -INFINITY; /* largest, second largest */
            for (int e = g * per; e < (g + 1) * per; ++e) {
                if (c[e] > a) {
                    b = a;
                    a = c[e];
                } else if (c[e] > b) {
                    b = c[e];
                }
            }
            gs[g] = a + b;
            gid[g] = g;
        }
        band_topk(gs, gid, G, Gk, gkeep);
        for (int g = 0; g < G; ++g)
            if (gkeep[g])
                for (int e = g * per; e < (g + 1) * per; ++e) cand[n++] = e;
    }
    band_topk(c, cand, n, k, chosen);
    int m = 0;
    for (int i = 0; i < n; ++i)
        if (chosen[i]) sel[m++] = cand[i];
    free(cand);
    free(chosen);
    return m == k ? 0 : -1;
}

/* Router logits ("Nemotron 3 Ultra 架构 QA", Q5.2): an fp32 linear of the
 * un-projected hidden state with no bias; here the exact dot product in fp64. */
int lmo_logits(const lmo_cfg* cfg, const void* x, const uint16_t* router_w, int64_t n, double* out) {
    const int H = cfg->H, E = cfg->E;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h) acc += x_at(cfg, x, t, h) * bf(router_w[(int64_t)e * H + h]);
            out[t * E + e] = acc;
        }
    return 0;
}

/* One token's routing from its logits (Q5.2 sigmoid and bias; Q5.3 bias for
 * choice only; Q5.8 normalise then x routed_scaling_factor). */
static int route_one(const lmo_cfg* cfg, const double* logit, const float* e_bias, int32_t* idx, double* w) {
    const int E = cfg->E, k = cfg->k;
    double* sig = (double*)malloc(sizeof(double) * (size_t)E * 2);
    double* ch = sig + E;
    for (int e = 0; e < E; ++e) {
        sig[e] = 1.0 / (1.0 + exp(-logit[e]));
        ch[e] = sig[e] + (double)e_bias[e];
    }
    int rc = lmo_select(cfg, ch, idx);
    if (rc == 0) {
        double sum = 0.0;
        for (int j = 0; j < k; ++j) sum += sig[idx[j]];
        for (int j = 0; j < k; ++j) w[j] = cfg->s * sig[idx[j]] / sum;
    }
    free(sig);
    return rc;
}

int lmo_route(const lmo_cfg* cfg, const void* x, const uint16_t* router_w, const float* e_bias, int64_t n,
              int32_t* idx, double* w) {
    const int E = cfg->E, k = cfg->k;
    double* lg = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * E);
    lmo_logits(cfg, x, router_w, n, lg);
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t t = 0; t < n; ++t) bad |= route_one(cfg, lg + t * E, e_bias, idx + t * k, w + t * k) != 0;
    free(lg);
    return bad ? -1 : 0;
}

/* fc1_latent_proj of n tokens, unrounded ("Nemotron 3 Ultra 架构 QA", Q5.1). */
int lmo_latent(const lmo_cfg* cfg, const void* x, const uint16_t* fc1_w, int64_t n, double* out) {
    const int H = cfg->H, L = cfg->L;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t) {
        double* xh = (double*)malloc(sizeof(double) * (size_t)H);
        for (int h = 0; h < H; ++h) xh[h] = rho(cfg, x_at(cfg, x, t, h));
        for (int l = 0; l < L; ++l) {
            double s = 0.0;
            for (int h = 0; h < H; ++h) s += xh[h] * bf(fc1_w[(int64_t)l * H + h]);
            out[t * L + l] = s;
        }
        free(xh);
    }
    return 0;
}

/* Full layer for each token ("Nemotron 3 Ultra 架构 QA", Q5.1 and Q5.7):
 *   z    = rho(x^ W_fc1^T)                       fc1_latent_proj, H -> L
 *   a_e  = rho(relu(z W_up[e]^T)^2)              expert up + relu2 (Q2.6)
 *   o_e  = a_e W_down[e]^T                       expert down, I -> L
 *   comb = rho(sum_{e in S, ascending} w_e o_e)  weighted sum (index_add_)
 *   a_s  = rho(relu(x^ W_su^T)^2)                shared expert on raw x (Q5.7)
 *   y    = comb W_fc2^T + a_s W_sd^T             fc2_latent_proj + shared down
 * with x^ = rho(x). */
int lmo_forward(const lmo_cfg* cfg, const void* x, const lmo_weights* wts, int64_t n, int32_t* idx_out,
                double* w_out, double* y) {
    const int H = cfg->H, L = cfg->L, E = cfg->E, k = cfg->k, I = cfg->I, Is = cfg->Is;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t t = 0; t < n; ++t) {
        double* buf = (double*)malloc(sizeof(double) * ((size_t)E + H + L + I + L + L + Is + k));
        double* lg = buf;
        double* xh = lg + E;
        double* z = xh + H;
        double* a = z + L;
        double* acc = a + I;
        double* comb = acc + L;
        double* as = comb + L;
        double* w = as + Is;
        int32_t idx[512];
        /* routing on the un-projected, un-rounded input */
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h) s += x_at(cfg, x, t, h) * bf(wts->router_w[(int64_t)e * H + h]);
            lg[e] = s;
        }
        if (route_one(cfg, lg, wts->e_bias, idx, w) != 0) {
            bad = 1;
            free(buf);
            continue;
        }
        for (int h = 0; h < H; ++h) xh[h] = rho(cfg, x_at(cfg, x, t, h));
        for (int l = 0; l < L; ++l) {
            double s = 0.0;
            for (int h = 0; h < H; ++h) s += xh[h] * bf(wts->fc1_w[(int64_t)l * H + h]);
            z[l] = rho(cfg, s);
        }
        for (int l = 0; l < L; ++l) acc[l] = 0.0;
        for (int j = 0; j < k; ++j) {
            const uint16_t* up = wts->up_w[idx[j]];
            const uint16_t* dn = wts->down_w[idx[j]];
            if (!up || !dn) {
                bad = 1;
                break;
            }
            const double gu = wts->up_gs ? (double)wts->up_gs[idx[j]] : 1.0;
            const double gd = wts->down_gs ? (double)wts->down_gs[idx[j]] : 1.0;
            for (int i = 0; i < I; ++i) {
                double s = 0.0;
                for (int l = 0; l < L; ++l) s += z[l] * bf(up[(int64_t)i * L + l]);
                s *= gu;
                double r = s > 0.0 ? s : 0.0;
                a[i] = rho(cfg, r * r);
            }
            for (int l = 0; l < L; ++l) {
                double s = 0.0;
                for (int i = 0; i < I; ++i) s += a[i] * bf(dn[(int64_t)l * I + i]);
                acc[l] += w[j] * (gd * s);
            }
        }
        for (int l = 0; l < L; ++l) comb[l] = rho(cfg, acc[l]);
        for (int i = 0; i < Is; ++i) {
            double s = 0.0;
            for (int h = 0; h < H; ++h) s += xh[h] * bf(wts->shared_up_w[(int64_t)i * H + h]);
            double r = s > 0.0 ? s : 0.0;
            as[i] = rho(cfg, r * r);
        }
        for (int h = 0; h < H; ++h) {
            double yr = 0.0, ys = 0.0;
            for (int l = 0; l < L; ++l) yr += comb[l] * bf(wts->fc2_w[(int64_t)h * L + l]);
            for (int i = 0; i < Is; ++i) ys += as[i] * bf(wts->shared_down_w[(int64_t)h * Is + i]);
            y[t * H + h] = yr + ys;
        }
        if (idx_out)
            for (int j = 0; j < k; ++j) idx_out[t * k + j] = idx[j];
        if (w_out)
            for (int j = 0; j < k; ++j) w_out[t * k + j] = w[j];
        free(buf);
    }
    return bad ? -1 : 0;
}

/* Bias update and MaxVio ("Nemotron 3 Ultra 架构 QA", Q5.3 and Q5.4). */
int lmo_update_bias(int E, const int32_t* counts, const float* bias, double eta, float* bias_out, double* maxvio) {
    long long total = 0, mx = 0;
    for (int e = 0; e < E; ++e) {
        total += counts[e];
        if (counts[e] > mx) mx = counts[e];
    }
    const double mean = (double)total / (double)E;
    for (int e = 0; e < E; ++e) bias_out[e] = (float)((double)bias[e] - eta * ((double)counts[e] - mean));
    if (maxvio) *maxvio = mean > 0.0 ? ((double)mx - mean) / mean : 0.0;
    return 0;
}

static uint16_t bf16_bits_of(double v) { /* v already a bf16 value */
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* RMSNorm ("Nemotron 3 Ultra 架构 QA", Q2.8): fp64 mean of squares, r =
 * 1/sqrt(mean + eps), bf16 rounding of x*r, then of gamma times that. */
int lmo_rmsnorm(int H, const uint16_t* x, const uint16_t* gamma, double eps, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        double ss = 0.0;
        for (int h = 0; h < H; ++h) {
            double v = bf(x[t * H + h]);
            ss += v * v;
        }
        const double r = 1.0 / sqrt(ss / (double)H + eps);
        for (int h = 0; h < H; ++h) {
            const double xt = lmo_round_bf16(bf(x[t * H + h]) * r);
            out[t * H + h] = bf16_bits_of(lmo_round_bf16(bf(gamma[h]) * xt));
        }
    }
    return 0;
}

/* Pre-norm residual block around the layer (Q2.1): y = x + layer(rmsnorm(x)). */
int lmo_forward_block(const lmo_cfg* cfg, const uint16_t* x, const uint16_t* gamma, double eps,
                      const lmo_weights* wts, int64_t n, int32_t* idx, double* w, double* y) {
    if (cfg->x_f32) return -1;
    const int H = cfg->H;
    uint16_t* xn = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n > 0 ? n : 1) * H);
    lmo_rmsnorm(H, x, gamma, eps, n, xn);
    int rc = lmo_forward(cfg, xn, wts, n, idx, w, y);
    for (int64_t i = 0; rc == 0 && i < n * H; ++i) y[i] += bf(x[i]);
    free(xn);
    return rc;
}

/* ---------------------------------------------------------------- NVFP4
 * Format and recipe as stated in oracle.h. Decoding follows the bit fields;
 * encoding is a brute-force search over every representable value, so no
 * bit trick of the encoder needs checking. */
double lmo_e2m1_value(int code) {
    const int e = (code >> 1) & 3, m = code & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (code & 8) ? -mag : mag;
}

double lmo_e4m3_value(int byte) {
    const int e = (byte >> 3) & 15, m = byte & 7;
    if ((byte & 0x7F) == 0x7F) return NAN;
    const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (byte & 0x80) ? -mag : mag;
}

/* nearest of the candidate codes lo..hi (non-negative values, ascending), ties to the even code */
static int nearest_code(double a, int hi, double (*val)(int)) {
    int best = 0;
    double bd = fabs(val(0) - a);
    for (int c = 1; c <= hi; ++c) {
        const double d = fabs(val(c) - a);
        if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bd = d;
        }
    }
    return best;
}

int lmo_e2m1_encode(float q) {
    const int s = q < 0.0f;
    const double a = fabs((double)q);
    const int m = a >= 6.0 ? 7 : nearest_code(a, 7, lmo_e2m1_value);
    return (s << 3) | m;
}

int lmo_e4m3_encode(float u) {
    if (!(u > 0.0f)) return 0;
    if ((double)u >= 448.0) return 0x7E;
    return nearest_code((double)u, 0x7E, lmo_e4m3_value);
}

static inline int64_t tile_of(int64_t gr, int K, int k) { return (gr / 128) * (K / 64) + k / 64; }

int lmo_nvfp4_quantize(const uint16_t* w, int64_t n_mat, int R, int K, uint8_t* codes, uint8_t* sf, float* g) {
    if (R <= 0 || K <= 0 || R % 128 || K % 64) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < n_mat; ++m) {
        const uint16_t* wm = w + m * (int64_t)R * K;
        float amax = 0.0f;
        for (int64_t i = 0; i < (int64_t)R * K; ++i) {
            const float a = fabsf((float)bf(wm[i]));
            if (a > amax) amax = a;
        }
        const float gm = amax > 0.0f ? amax / 2688.0f : 1.0f;
        g[m] = gm;
        for (int r = 0; r < R; ++r) {
            const int64_t gr = m * R + r;
            for (int b = 0; b < K / 16; ++b) {
                const int k0 = b * 16;
                float bmax = 0.0f;
                for (int i = 0; i < 16; ++i) {
                    const float a = fabsf((float)bf(wm[(int64_t)r * K + k0 + i]));
                    if (a > bmax) bmax = a;
                }
                const float t = bmax / gm;
                const float u = t / 6.0f;
                const int sb = lmo_e4m3_encode(u);
                const float S = (float)lmo_e4m3_value(sb);
                sf[tile_of(gr, K, k0) * 512 + (gr % 128) * 4 + (k0 % 64) / 16] = (uint8_t)sb;
                const float d = S * gm;
                for (int i = 0; i < 16; i += 2) {
                    int c[2];
                    for (int h = 0; h < 2; ++h) {
                        const float wv = (float)bf(wm[(int64_t)r * K + k0 + i + h]);
                        c[h] = S == 0.0f ? 0 : lmo_e2m1_encode(wv / d);
                    }
                    const int k = k0 + i;
                    codes[tile_of(gr, K, k) * 4096 + (gr % 128) * 32 + (k % 64) / 2] = (uint8_t)(c[0] | (c[1] << 4));
                }
            }
        }
    }
    return 0;
}

int lmo_nvfp4_dequant(const uint8_t* codes, const uint8_t* sf, int64_t n_mat, int R, int K, uint16_t* out) {
    if (R <= 0 || K <= 0 || R % 128 || K % 64) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t gr = 0; gr < n_mat * R; ++gr) {
        for (int k = 0; k < K; ++k) {
            const int64_t t = tile_of(gr, K, k);
            const uint8_t byte = codes[t * 4096 + (gr % 128) * 32 + (k % 64) / 2];
            const int code = (k & 1) ? byte >> 4 : byte & 15;
            const double S = lmo_e4m3_value(sf[t * 512 + (gr % 128) * 4 + (k % 64) / 16]);
            const double v = lmo_e2m1_value(code) * S;
            if (lmo_round_bf16(v) != v) bad = 1; /* code * S always has <= 6 significant bits */
            out[gr * K + k] = bf16_bits_of(v);
        }
    }
    return bad ? -1 : 0;
}
