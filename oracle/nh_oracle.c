/*
 * nh_oracle.c -- plain fp64 CPU oracle of the Nemotron-H non-gated MoE block.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file's library.  It shares no code, header
 * or constant with the CUDA library; the two meet only in the seeded inputs.
 *
 * What it computes, one token at a time, with no intermediate rounding
 * (every stored input is widened exactly to double):
 *
 *   1. router logits  l_e = sum_h x[h] * Wr[e][h]
 *      (the router "gate" of the MoE layer: ModelOpt descriptor
 *      "NemotronHMoELayerDescriptor", gate_name='gate'; the router stays fp32,
 *      auto-round PR #1712, the gate is in the ignored layers of the log)
 *   2. scores  s_e = 1 / (1 + exp(-l_e))
 *   3. group score = max of the selection scores s_e (+ correction bias, when
 *      given) over the g = E/G experts of each group;
 *   4. keep the topk_group groups with the largest group score, ties to the
 *      lower group id;
 *   5. among the experts of the kept groups take the num_experts_per_tok
 *      largest selection scores, ties to the lower expert id, output order
 *      (score desc, id asc);
 *   6. weight w_j = alpha * s_j / sum_i s_i when norm_topk_prob, else
 *      alpha * s_j (the unbiased scores s);
 *      (steps 3-6: baseRT issue #46, "MoE: 128 routed experts, 6 per token,
 *      grouped top-k (n_groups=8, topk_group=1), routed_scaling_factor=2.5,
 *      norm_topk_prob"; the config fields n_group .. routed_scaling_factor of
 *      ModelArgs in the exo commit "Add support for Nemotron sharding")
 *   7. y = sum_j w_j * Wd[e_j] relu(Wu[e_j] x)^2  +  Wsd relu(Wsu x)^2
 *      (routed experts up_proj -> relu^2 -> down_proj with no gate_proj:
 *      vllm.cpp PR #518 "Non-gated MoE"; expert shapes from the auto-round
 *      PR #1712 log; the always-on shared expert NemotronHMLP with up_proj
 *      and down_proj, exo commit, nemotron_h.pyi; "1 shared expert (3712
 *      wide)", baseRT issue #46).  The shared expert is unscaled.
 *
 * Layouts are row-major, PyTorch Linear [out, in]: Wr [E][H] float32,
 * Wu [E][I][H], Wd [E][H][I], Wsu [S][H], Wsd [H][S]; x [T][H].  Activations
 * and expert weights are float32 (dtype 0) or bf16 bit patterns (dtype 1).
 *
 * Expert and shared weights may instead be NVFP4 (vllm.cpp PR #518: the
 * checkpoint keeps routed and shared expert weights in 4-bit NVFP4 with one
 * scale per 16 inputs, activations in 16 bits).  Reading of that format (the
 * PR names it and no more): every element is
 * an E2M1 code (sign, 2 exponent bits with bias 1, 1 mantissa bit; values
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per byte with the even column in the low
 * nibble; every 16 consecutive columns of a row share one E4M3 scale byte
 * (sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
 * S.1111.111 is NaN), rows of scale bytes padded to a multiple of 16 bytes;
 * and each matrix has one float32 global scale.  The weight is
 *   w = e2m1(code) * e4m3(scale) * global.
 *
 * nho_forward_latent adds latent projections around the routed experts
 * (ModelOpt descriptor NemotronHMoELayerDescriptor names fc1_latent_proj and
 * fc2_latent_proj and gives no formula): PARITY UNPINNED as a reading of the
 * sources; its tests pin it to the plain block at identity and permutation
 * projections.
 *
 * Single-threaded, plain loops, built -O2 without fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t H, E, G, tg, k, I, S;
    int64_t n_shared;     /* 0 or 1 */
    int64_t norm;         /* norm_topk_prob */
    double alpha;         /* routed_scaling_factor */
    int64_t dtype;        /* 0 = float32, 1 = bf16 */
    int64_t group_score;  /* 0 = max of the group (the reading used); 1 = sum of the top two */
} nho_cfg;

enum { NHO_OK = 0, NHO_BAD_CONFIG = -1, NHO_BAD_ARG = -2, NHO_NOMEM = -3 };

#define NHO_MAX_E 4096

/* exact widening of one stored element to double */
static double load(const void *p, int64_t i, int64_t dtype) {
    if (dtype == 1) {
        uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)p)[i];
}

/* One stacked weight tensor [n_mat][rows][cols] in one of three formats. */
typedef struct {
    int64_t format;          /* 0 float32, 1 bf16, 2 NVFP4 */
    const void *data;        /* elements; NVFP4: codes [n_mat][rows][cols / 2] */
    const uint8_t *scales;   /* NVFP4: E4M3 [n_mat][rows][scale_pitch] */
    const float *global;     /* NVFP4: [n_mat] */
    int64_t rows, cols, scale_pitch;
} nho_wt;

/* E2M1 value of a 4-bit code, from its bit fields */
static double e2m1_value(unsigned code) {
    const unsigned sign = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    const double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, (int)e - 1);
    return sign ? -mag : mag;
}

/* E4M3 value of a byte, from its bit fields (S.1111.111 is NaN) */
static double e4m3_value(unsigned byte) {
    const unsigned sign = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
    if (e == 15u && m == 7u) return NAN;
    const double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, (int)e - 7);
    return sign ? -mag : mag;
}

/* element idx = row * cols + col of matrix `mat`, exactly as a double */
static double wt_get(const nho_wt *w, int64_t mat, int64_t idx) {
    const int64_t per = w->rows * w->cols;
    if (w->format != 2) return load(w->data, mat * per + idx, w->format);
    const int64_t r = idx / w->cols, col = idx - r * w->cols;
    const uint8_t byte = ((const uint8_t *)w->data)[mat * per / 2 + r * (w->cols / 2) + col / 2];
    const unsigned code = (col & 1) ? (byte >> 4) : (byte & 15u);
    const uint8_t sb = w->scales[(mat * w->rows + r) * w->scale_pitch + col / 16];
    return e2m1_value(code) * e4m3_value(sb) * (double)w->global[mat];
}

/* dense float64 copy of matrix `mat` of a weight tensor (for the tests' pins) */
int nho_dequant(const nho_wt *w, int64_t mat, double *out) {
    if (!w || !out || w->rows < 1 || w->cols < 1) return -2;
    if (w->format == 2 && (w->cols % 2 || !w->scales || !w->global ||
                           w->scale_pitch * 16 < w->cols)) return -2;
    for (int64_t i = 0; i < w->rows * w->cols; ++i) out[i] = wt_get(w, mat, i);
    return 0;
}

int nho_check_config(const nho_cfg *c) {
    if (!c) return NHO_BAD_ARG;
    if (c->H < 1 || c->E < 1 || c->G < 1 || c->E > NHO_MAX_E) return NHO_BAD_CONFIG;
    if (c->E % c->G != 0) return NHO_BAD_CONFIG;
    if (c->tg < 1 || c->tg > c->G) return NHO_BAD_CONFIG;
    if (c->k < 1 || c->k > c->tg * (c->E / c->G)) return NHO_BAD_CONFIG;
    if (c->I < 1) return NHO_BAD_CONFIG;
    if (c->n_shared != 0 && c->n_shared != 1) return NHO_BAD_CONFIG;
    if (c->n_shared == 1 && c->S < 1) return NHO_BAD_CONFIG;
    if (!isfinite(c->alpha)) return NHO_BAD_CONFIG;
    if (c->dtype != 0 && c->dtype != 1) return NHO_BAD_CONFIG;
    if (c->group_score != 0 && c->group_score != 1) return NHO_BAD_CONFIG;
    if (c->group_score == 1 && c->E / c->G < 2) return NHO_BAD_CONFIG;
    return NHO_OK;
}

/* "a ranks before b": larger value first, equal values by lower id */
static int before(double va, int64_t ia, double vb, int64_t ib) {
    if (va != vb) return va > vb;
    return ia < ib;
}

/* insertion sort of ids[0..n) by (val[id] desc, id asc) */
static void sort_desc(int64_t *ids, int64_t n, const double *val) {
    for (int64_t a = 1; a < n; ++a) {
        int64_t id = ids[a];
        int64_t b = a - 1;
        while (b >= 0 && before(val[id], id, val[ids[b]], ids[b])) {
            ids[b + 1] = ids[b];
            --b;
        }
        ids[b + 1] = id;
    }
}

/*
 * Route one token.  scratch needs 4*E doubles + 2*E int64.
 * gap_group: group score of rank tg-1 minus rank tg (INFINITY when tg == G).
 * gap_expert: smallest difference between neighbouring selection scores over
 * the ranks 0..k of the candidate order (INFINITY when nothing to compare).
 */
static void route_one(const nho_cfg *c, const void *x, int64_t t, const float *wr,
                      const float *bias, int32_t *idx, double *w, double *gap_group,
                      double *gap_expert, double *scr, int64_t *iscr) {
    const int64_t H = c->H, E = c->E, G = c->G, g = c->E / c->G;
    double *s = scr;            /* sigmoid scores      [E] */
    double *sel = scr + E;      /* selection scores    [E] */
    double *gs = scr + 2 * E;   /* group scores        [G] */
    int64_t *gid = iscr;        /* group order         [G] */
    int64_t *cand = iscr + E;   /* candidate experts   [tg*g] */

    for (int64_t e = 0; e < E; ++e) {
        double l = 0.0;
        for (int64_t h = 0; h < H; ++h)
            l += load(x, t * H + h, c->dtype) * (double)wr[e * H + h];
        s[e] = 1.0 / (1.0 + exp(-l));
        sel[e] = s[e] + (bias ? (double)bias[e] : 0.0);
    }
    for (int64_t q = 0; q < G; ++q) {
        if (c->group_score == 0) {
            double m = sel[q * g];
            for (int64_t i = 1; i < g; ++i)
                if (sel[q * g + i] > m) m = sel[q * g + i];
            gs[q] = m;
        } else {
            /* sum of the two largest selection scores of the group */
            int64_t tmp[NHO_MAX_E];
            for (int64_t i = 0; i < g; ++i) tmp[i] = q * g + i;
            sort_desc(tmp, g, sel);
            gs[q] = sel[tmp[0]] + sel[tmp[1]];
        }
        gid[q] = q;
    }
    sort_desc(gid, G, gs);
    *gap_group = (c->tg < G) ? gs[gid[c->tg - 1]] - gs[gid[c->tg]] : INFINITY;

    int64_t nc = 0;
    for (int64_t r = 0; r < c->tg; ++r)
        for (int64_t i = 0; i < g; ++i) cand[nc++] = gid[r] * g + i;
    sort_desc(cand, nc, sel);

    double gap = INFINITY;
    int64_t last = (c->k < nc) ? c->k : nc - 1;
    for (int64_t r = 0; r < last; ++r) {
        double d = sel[cand[r]] - sel[cand[r + 1]];
        if (d < gap) gap = d;
    }
    *gap_expert = gap;

    double sum = 0.0;
    for (int64_t j = 0; j < c->k; ++j) sum += s[cand[j]];
    for (int64_t j = 0; j < c->k; ++j) {
        idx[j] = (int32_t)cand[j];
        w[j] = c->norm ? c->alpha * s[cand[j]] / sum : c->alpha * s[cand[j]];
    }
}

/* Routing of T tokens.  idx [T][k], w [T][k]; gaps [T] each (may be NULL). */
int nho_route(const nho_cfg *c, int64_t T, const void *x, const float *wr, const float *bias,
              int32_t *idx, double *w, double *gap_group, double *gap_expert) {
    int rc = nho_check_config(c);
    if (rc) return rc;
    if (T < 0 || (T > 0 && (!x || !wr || !idx || !w))) return NHO_BAD_ARG;
    double *scr = (double *)malloc(sizeof(double) * (size_t)(3 * c->E));
    int64_t *iscr = (int64_t *)malloc(sizeof(int64_t) * (size_t)(2 * c->E));
    if (!scr || !iscr) { free(scr); free(iscr); return NHO_NOMEM; }
    for (int64_t t = 0; t < T; ++t) {
        double gg, ge;
        route_one(c, x, t, wr, bias, idx + t * c->k, w + t * c->k, &gg, &ge, scr, iscr);
        if (gap_group) gap_group[t] = gg;
        if (gap_expert) gap_expert[t] = ge;
    }
    free(scr);
    free(iscr);
    return NHO_OK;
}

/* out[H] += scale * Wd relu(Wu xt)^2 for matrix `mat` of the up tensor (rows n,
 * cols H) and the down tensor (rows H, cols n); u is scratch of n doubles.
 * H is the width of xt and out (the hidden size, or the latent size). */
static void mlp_relu2(int64_t H, const double *xt, const nho_wt *up, const nho_wt *down,
                      int64_t mat, int64_t n, double scale, double *u, double *out) {
    for (int64_t i = 0; i < n; ++i) {
        double a = 0.0;
        for (int64_t h = 0; h < H; ++h) a += wt_get(up, mat, i * H + h) * xt[h];
        double r = a > 0.0 ? a : 0.0;
        u[i] = r * r;
    }
    for (int64_t h = 0; h < H; ++h) {
        double a = 0.0;
        for (int64_t i = 0; i < n; ++i) a += wt_get(down, mat, h * down->cols + i) * u[i];
        out[h] += scale * a;
    }
}

/*
 * Full block output for the listed tokens.
 *   tokens [n_tok]: token ids into x;   y [n_tok][H] (written)
 *   ovr_idx/ovr_w [n_tok][k]: when non-NULL, this routing replaces the
 *     oracle's own (to check expert maths under another side's routing);
 *   idx_out/w_out [n_tok][k]: the routing used (may be NULL).
 * up [E][I][H], down [E][H][I], su [1][S][H], sd [1][H][S] in any format.
 */
int nho_forward_wt(const nho_cfg *c, int64_t T, const void *x, const float *wr, const float *bias,
                   const nho_wt *up, const nho_wt *down, const nho_wt *su, const nho_wt *sd,
                   const int32_t *ovr_idx, const double *ovr_w, const int64_t *tokens,
                   int64_t n_tok, double *y, int32_t *idx_out, double *w_out) {
    int rc = nho_check_config(c);
    if (rc) return rc;
    if (n_tok < 0 || (n_tok > 0 && (!x || !tokens || !y || !up || !down))) return NHO_BAD_ARG;
    if (!ovr_idx && !wr) return NHO_BAD_ARG;
    if (c->n_shared && (!su || !sd)) return NHO_BAD_ARG;
    const int64_t H = c->H, I = c->I, S = c->S, k = c->k;
    if (up->rows != I || up->cols != H || down->rows != H || down->cols != I) return NHO_BAD_ARG;
    if (c->n_shared && (su->rows != S || su->cols != H || sd->rows != H || sd->cols != S))
        return NHO_BAD_ARG;
    int64_t nmax = I > S ? I : S;
    double *xt = (double *)malloc(sizeof(double) * (size_t)H);
    double *u = (double *)malloc(sizeof(double) * (size_t)nmax);
    double *scr = (double *)malloc(sizeof(double) * (size_t)(3 * c->E));
    int64_t *iscr = (int64_t *)malloc(sizeof(int64_t) * (size_t)(2 * c->E));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    double *w = (double *)malloc(sizeof(double) * (size_t)k);
    if (!xt || !u || !scr || !iscr || !idx || !w) {
        free(xt); free(u); free(scr); free(iscr); free(idx); free(w);
        return NHO_NOMEM;
    }
    rc = NHO_OK;
    for (int64_t n = 0; n < n_tok; ++n) {
        int64_t t = tokens[n];
        if (t < 0 || t >= T) { rc = NHO_BAD_ARG; break; }
        for (int64_t h = 0; h < H; ++h) xt[h] = load(x, t * H + h, c->dtype);
        if (ovr_idx) {
            for (int64_t j = 0; j < k; ++j) {
                idx[j] = ovr_idx[n * k + j];
                w[j] = ovr_w[n * k + j];
                if (idx[j] < 0 || idx[j] >= c->E) rc = NHO_BAD_ARG;
            }
            if (rc) break;
        } else {
            double gg, ge;
            route_one(c, x, t, wr, bias, idx, w, &gg, &ge, scr, iscr);
        }
        double *yt = y + n * H;
        for (int64_t h = 0; h < H; ++h) yt[h] = 0.0;
        for (int64_t j = 0; j < k; ++j) mlp_relu2(H, xt, up, down, idx[j], I, w[j], u, yt);
        if (c->n_shared) mlp_relu2(H, xt, su, sd, 0, S, 1.0, u, yt);
        if (idx_out)
            for (int64_t j = 0; j < k; ++j) idx_out[n * k + j] = idx[j];
        if (w_out)
            for (int64_t j = 0; j < k; ++j) w_out[n * k + j] = w[j];
    }
    free(xt); free(u); free(scr); free(iscr); free(idx); free(w);
    return rc;
}

/* nho_forward_wt with float32 / bf16 weights given as plain arrays in c->dtype */
int nho_forward(const nho_cfg *c, int64_t T, const void *x, const float *wr, const float *bias,
                const void *w_up, const void *w_down, const void *w_su, const void *w_sd,
                const int32_t *ovr_idx, const double *ovr_w, const int64_t *tokens,
                int64_t n_tok, double *y, int32_t *idx_out, double *w_out) {
    int rc = nho_check_config(c);
    if (rc) return rc;
    const nho_wt up = {c->dtype, w_up, NULL, NULL, c->I, c->H, 0};
    const nho_wt down = {c->dtype, w_down, NULL, NULL, c->H, c->I, 0};
    const nho_wt su = {c->dtype, w_su, NULL, NULL, c->S, c->H, 0};
    const nho_wt sd = {c->dtype, w_sd, NULL, NULL, c->H, c->S, 0};
    if (n_tok > 0 && (!w_up || !w_down)) return NHO_BAD_ARG;
    if (c->n_shared && (!w_su || !w_sd)) return NHO_BAD_ARG;
    return nho_forward_wt(c, T, x, wr, bias, &up, &down, c->n_shared ? &su : NULL,
                          c->n_shared ? &sd : NULL, ovr_idx, ovr_w, tokens, n_tok, y, idx_out,
                          w_out);
}

/*
 * Latent MoE: the routed experts work in a latent width L between two
 * projections (ModelOpt descriptor "NemotronHMoELayerDescriptor", parameters
 * latent_fc1_name='fc1_latent_proj' and latent_fc2_name='fc2_latent_proj';
 * the descriptor names the two modules and no more).  Reading used:
 *   xl = Wl1 x                           (fc1_latent_proj, [L][H])
 *   yl = sum_j w_j * Wd[e_j] relu(Wu[e_j] xl)^2   (experts in width L:
 *                                         Wu [E][I][L], Wd [E][L][I])
 *   y  = Wl2 yl + Wsd relu(Wsu x)^2      (fc2_latent_proj, [H][L]; the
 *                                         router and the shared expert see
 *                                         the full-width x)
 * with the routing of steps 1-6 on x.  No intermediate rounding.
 * PARITY UNPINNED as a reading of the pages (they give no formula); the
 * tests pin this function to the plain block at identity projections.
 * wl1, wl2 are in c->dtype.  Other arguments as nho_forward_wt.
 */
int nho_forward_latent(const nho_cfg *c, int64_t L, int64_t T, const void *x, const float *wr,
                       const float *bias, const nho_wt *up, const nho_wt *down,
                       const nho_wt *su, const nho_wt *sd, const void *wl1, const void *wl2,
                       const int32_t *ovr_idx, const double *ovr_w, const int64_t *tokens,
                       int64_t n_tok, double *y, int32_t *idx_out, double *w_out) {
    int rc = nho_check_config(c);
    if (rc) return rc;
    if (L < 1 || n_tok < 0 || (n_tok > 0 && (!x || !tokens || !y || !up || !down || !wl1 || !wl2)))
        return NHO_BAD_ARG;
    if (!ovr_idx && !wr) return NHO_BAD_ARG;
    if (c->n_shared && (!su || !sd)) return NHO_BAD_ARG;
    const int64_t H = c->H, I = c->I, S = c->S, k = c->k;
    if (up->rows != I || up->cols != L || down->rows != L || down->cols != I) return NHO_BAD_ARG;
    if (c->n_shared && (su->rows != S || su->cols != H || sd->rows != H || sd->cols != S))
        return NHO_BAD_ARG;
    int64_t nmax = I > S ? I : S;
    double *xt = (double *)malloc(sizeof(double) * (size_t)H);
    double *xl = (double *)malloc(sizeof(double) * (size_t)L);
    double *yl = (double *)malloc(sizeof(double) * (size_t)L);
    double *u = (double *)malloc(sizeof(double) * (size_t)nmax);
    double *scr = (double *)malloc(sizeof(double) * (size_t)(3 * c->E));
    int64_t *iscr = (int64_t *)malloc(sizeof(int64_t) * (size_t)(2 * c->E));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    double *w = (double *)malloc(sizeof(double) * (size_t)k);
    if (!xt || !xl || !yl || !u || !scr || !iscr || !idx || !w) {
        free(xt); free(xl); free(yl); free(u); free(scr); free(iscr); free(idx); free(w);
        return NHO_NOMEM;
    }
    rc = NHO_OK;
    for (int64_t n = 0; n < n_tok; ++n) {
        int64_t t = tokens[n];
        if (t < 0 || t >= T) { rc = NHO_BAD_ARG; break; }
        for (int64_t h = 0; h < H; ++h) xt[h] = load(x, t * H + h, c->dtype);
        if (ovr_idx) {
            for (int64_t j = 0; j < k; ++j) {
                idx[j] = ovr_idx[n * k + j];
                w[j] = ovr_w[n * k + j];
                if (idx[j] < 0 || idx[j] >= c->E) rc = NHO_BAD_ARG;
            }
            if (rc) break;
        } else {
            double gg, ge;
            route_one(c, x, t, wr, bias, idx, w, &gg, &ge, scr, iscr);
        }
        for (int64_t l = 0; l < L; ++l) {
            double a = 0.0;
            for (int64_t h = 0; h < H; ++h) a += load(wl1, l * H + h, c->dtype) * xt[h];
            xl[l] = a;
            yl[l] = 0.0;
        }
        for (int64_t j = 0; j < k; ++j) mlp_relu2(L, xl, up, down, idx[j], I, w[j], u, yl);
        double *yt = y + n * H;
        for (int64_t h = 0; h < H; ++h) {
            double a = 0.0;
            for (int64_t l = 0; l < L; ++l) a += load(wl2, h * L + l, c->dtype) * yl[l];
            yt[h] = a;
        }
        if (c->n_shared) mlp_relu2(H, xt, su, sd, 0, S, 1.0, u, yt);
        if (idx_out)
            for (int64_t j = 0; j < k; ++j) idx_out[n * k + j] = idx[j];
        if (w_out)
            for (int64_t j = 0; j < k; ++j) w_out[n * k + j] = w[j];
    }
    free(xt); free(xl); free(yl); free(u); free(scr); free(iscr); free(idx); free(w);
    return rc;
}
