/*
 * Plain CPU oracle for one sparse MoE block of the Beam model (forward pass).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  The CUDA library
 * shares no code, header, table or helper with it.
 *
 * What it computes follows the Beam launch blog ("Introducing Beam",
 * section "Mixture of Experts": sigmoid scores over all 256 experts, 8 groups
 * of 32, a group's score is the sum of its two best scores, keep the best 4
 * groups, top-8 experts inside them, normalised router weights, output scaled
 * by 2.5; section "Residual Stream": depth-scaled residual update and the
 * FP32 sites) and the Beam transformers documentation page ("Overview",
 * "Sparse MoE" bullet: per-expert learned bias, n_group / topk_group,
 * normalised routing weights, routed_scaling_factor; "sandwich norm" bullet:
 * RMSNorm after each sub-layer; closing paragraph: router weights and expert
 * bias kept in FP32).  The DeepSeek-V3 conventions the pages leave open are
 * read as: the bias steers selection only, the group score uses the biased
 * scores, the combine weights are the unbiased sigmoid scores normalised to
 * sum 1, and ties go to the lower index.
 *
 * Precision.  Every quantity is evaluated in double, sequentially in index
 * order, with no blocking or reordering.  Where the pages fix FP32 for a step
 * whose result is an integer decision or a narrowing cast, the double value is
 * rounded once to FP32 and the decision is taken on that FP32 value:
 *   - routing decisions (group ranking, expert ranking) compare FP32 biased
 *     scores, and a group's score is the FP32 sum of its two best FP32 scores;
 *   - the SwiGLU product silu(g)*u is rounded to FP32 and then to bf16, the
 *     type the down projection consumes.
 * Combine weights, the down projection and the combine stay in double; the
 * block output is rounded once, double -> bf16, round-to-nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* bf16 <-> float / double, written from the IEEE-754 formats.          */
/* ------------------------------------------------------------------ */

/* A bf16 value is the upper 16 bits of an IEEE binary32 value. */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (8-bit significand, binary32 exponent
 * range), ties to even.  Written directly from the definition: scale the
 * value so that the bf16 spacing at its binade becomes 1, round to the
 * nearest integer with ties to even, scale back. */
uint16_t oracle_double_to_bf16(double d)
{
    if (isnan(d)) return 0x7fc0;
    const double max_bf16 = ldexp(255.0 / 128.0, 127); /* 0x7f7f */
    int e;
    double m;
    float f;
    uint32_t u;
    if (d == 0.0) {
        f = (float)d; /* keeps the sign of zero */
    } else {
        m = frexp(fabs(d), &e); /* |d| = m * 2^e, m in [0.5, 1) */
        /* bf16 significand: 8 bits, so spacing in binade [2^(e-1), 2^e) is
         * 2^(e-8); below the normal range (e-1 < -126) the spacing is 2^-133. */
        int q = e - 8;
        if (e - 1 < -126) q = -133;
        double scaled = ldexp(fabs(d), -q);
        double r = floor(scaled);
        double frac = scaled - r;
        if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
        double v = ldexp(r, q);
        if (v > max_bf16) v = INFINITY;
        f = (float)(d < 0 ? -v : v); /* exact: v has <= 8 significant bits */
    }
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* Logistic sigmoid, written from its definition. */
static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* SiLU (swish-1): z * sigmoid(z). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------ */
/* Router                                                               */
/* ------------------------------------------------------------------ */

/*
 * Selection for one token from its E logits (double): sigmoid scores, FP32
 * biased scores, group scores, kept groups, top_k experts and their
 * normalised unbiased weights, plus the near-tie gaps; the outputs are the
 * token's rows of oracle_route's outputs.
 */
static void route_one(int E, int n_group, int topk_group, int top_k, const double *logit,
                      const float *bias, int32_t *idx, double *w, double *scores,
                      double *biased, double *gap_expert, double *gap_group,
                      int32_t *kept_mask, double *gap_order)
{
    const int gsize = E / n_group;
    double *s = (double *)malloc(sizeof(double) * (size_t)E);
    double *bd = (double *)malloc(sizeof(double) * (size_t)E);
    float *b32 = (float *)malloc(sizeof(float) * (size_t)E);
    float *gs = (float *)malloc(sizeof(float) * (size_t)n_group);
    double *gsd = (double *)malloc(sizeof(double) * (size_t)n_group);
    char *kept = (char *)calloc((size_t)n_group, 1);
    char *chosen = (char *)calloc((size_t)E, 1);

    /* sigmoid scores, biased scores */
    for (int e = 0; e < E; ++e) {
        s[e] = sigmoid(logit[e]);
        bd[e] = s[e] + (double)bias[e];
        b32[e] = (float)bd[e];
    }

    /* group score: sum of the two largest biased scores of the group */
    for (int j = 0; j < n_group; ++j) {
        float t1 = -INFINITY, t2 = -INFINITY;
        double d1 = -INFINITY, d2 = -INFINITY;
        for (int e = j * gsize; e < (j + 1) * gsize; ++e) {
            if (b32[e] > t1) { t2 = t1; t1 = b32[e]; }
            else if (b32[e] > t2) { t2 = b32[e]; }
            if (bd[e] > d1) { d2 = d1; d1 = bd[e]; }
            else if (bd[e] > d2) { d2 = bd[e]; }
        }
        gs[j] = t1 + t2; /* FP32 addition */
        gsd[j] = d1 + d2;
    }

    /* keep topk_group groups: greater score first, ties to lower index */
    int32_t mask = 0;
    for (int r = 0; r < topk_group; ++r) {
        int best = -1;
        for (int j = 0; j < n_group; ++j) {
            if (kept[j]) continue;
            if (best < 0 || gs[j] > gs[best]) best = j;
        }
        kept[best] = 1;
        mask |= (int32_t)1 << best;
    }

    /* top_k experts among the kept groups' experts */
    double ssum = 0.0;
    for (int r = 0; r < top_k; ++r) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (!kept[e / gsize] || chosen[e]) continue;
            if (best < 0 || b32[e] > b32[best]) best = e;
        }
        chosen[best] = 1;
        idx[r] = best;
        ssum += s[best];
    }
    for (int r = 0; r < top_k; ++r) w[r] = s[idx[r]] / ssum;

    if (gap_expert) {
        double min_sel = INFINITY, max_uns = -INFINITY;
        for (int e = 0; e < E; ++e) {
            if (!kept[e / gsize]) continue;
            if (chosen[e]) { if (bd[e] < min_sel) min_sel = bd[e]; }
            else if (bd[e] > max_uns) max_uns = bd[e];
        }
        *gap_expert = (max_uns == -INFINITY) ? INFINITY : min_sel - max_uns;
    }
    if (gap_group) {
        double min_k = INFINITY, max_d = -INFINITY;
        for (int j = 0; j < n_group; ++j) {
            if (kept[j]) { if (gsd[j] < min_k) min_k = gsd[j]; }
            else if (gsd[j] > max_d) max_d = gsd[j];
        }
        *gap_group = (max_d == -INFINITY) ? INFINITY : min_k - max_d;
    }
    if (gap_order) {
        double g = INFINITY;
        for (int r = 0; r + 1 < top_k; ++r) {
            const double d = bd[idx[r]] - bd[idx[r + 1]];
            if (d < g) g = d;
        }
        *gap_order = g;
    }
    if (kept_mask) *kept_mask = mask;
    if (scores) memcpy(scores, s, sizeof(double) * (size_t)E);
    if (biased) memcpy(biased, bd, sizeof(double) * (size_t)E);
    free(s); free(bd); free(b32); free(gs); free(gsd); free(kept); free(chosen);
}

/* The routing configurations the method defines. */
static int route_args_ok(int E, int n_group, int topk_group, int top_k)
{
    if (E <= 0 || n_group <= 0 || E % n_group != 0) return 0;
    const int gsize = E / n_group;
    if (gsize < 2 || topk_group < 1 || topk_group > n_group || n_group > 31) return 0;
    if (top_k < 1 || top_k > topk_group * gsize) return 0;
    return 1;
}

#define ROW(p, t, n) ((p) ? (p) + (size_t)(t) * (n) : NULL)

/*
 * Group-limited sigmoid routing for T tokens.
 *
 * x        bf16 [T, H] row-major
 * router_w fp32 [E, H] row-major (logit_e = x . router_w[e])
 * bias     fp32 [E]
 * Outputs (row-major, caller-allocated):
 *   idx       int32 [T, top_k]  selected experts, descending FP32 biased score,
 *                               ties to the lower expert index
 *   w         double [T, top_k] unbiased sigmoid scores of the selected
 *                               experts divided by their sum
 *   scores    double [T, E]     sigmoid(logit)            (may be NULL)
 *   biased    double [T, E]     sigmoid(logit) + bias     (may be NULL)
 *   gap_expert double [T]       min double biased score over the selected
 *                               experts minus max over the unselected
 *                               candidates of kept groups (+inf if none)
 *                               (may be NULL)
 *   gap_group double [T]        min double group score over kept groups minus
 *                               max over dropped groups (+inf if none)
 *                               (may be NULL)
 *   gap_order double [T]        smallest difference of double biased scores
 *                               between neighbours of the chosen sequence
 *                               (the order the method returns them in; +inf
 *                               for top_k == 1) (may be NULL)
 *   kept_mask int32 [T]         bit j set iff group j was kept (may be NULL)
 * Returns 0, or -1 on an argument the method does not define.
 */
int oracle_route(int T, int H, int E, int n_group, int topk_group, int top_k,
                 const uint16_t *x, const float *router_w, const float *bias,
                 int32_t *idx, double *w, double *scores, double *biased,
                 double *gap_expert, double *gap_group, int32_t *kept_mask,
                 double *gap_order)
{
    if (T < 0 || H <= 0 || !route_args_ok(E, n_group, topk_group, top_k)) return -1;

#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        double *logit = (double *)malloc(sizeof(double) * (size_t)E);
        const uint16_t *xt = x + (size_t)t * H;
        /* logits: x . router_w[e], exact products summed in double */
        for (int e = 0; e < E; ++e) {
            const float *wr = router_w + (size_t)e * H;
            double acc = 0.0;
            for (int h = 0; h < H; ++h) acc += oracle_bf16_to_double(xt[h]) * (double)wr[h];
            logit[e] = acc;
        }
        route_one(E, n_group, topk_group, top_k, logit, bias, idx + (size_t)t * top_k,
                  w + (size_t)t * top_k, ROW(scores, t, E), ROW(biased, t, E), ROW(gap_expert, t, 1),
                  ROW(gap_group, t, 1), ROW(kept_mask, t, 1), ROW(gap_order, t, 1));
        free(logit);
    }
    return 0;
}

/*
 * The same routing from given FP32 logits [T, E] (row-major) instead of x and
 * the router matrix: selection under another expert bias reuses the logits
 * (the bias steers selection only).  Outputs as oracle_route.
 */
int oracle_route_logits(int T, int E, int n_group, int topk_group, int top_k,
                        const float *logits, const float *bias, int32_t *idx, double *w,
                        double *gap_expert, double *gap_group, int32_t *kept_mask,
                        double *gap_order)
{
    if (T < 0 || !route_args_ok(E, n_group, topk_group, top_k)) return -1;

#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) {
        double *logit = (double *)malloc(sizeof(double) * (size_t)E);
        for (int e = 0; e < E; ++e) logit[e] = (double)logits[(size_t)t * E + e];
        route_one(E, n_group, topk_group, top_k, logit, bias, idx + (size_t)t * top_k,
                  w + (size_t)t * top_k, NULL, NULL, ROW(gap_expert, t, 1), ROW(gap_group, t, 1),
                  ROW(kept_mask, t, 1), ROW(gap_order, t, 1));
        free(logit);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* One SwiGLU expert                                                    */
/* ------------------------------------------------------------------ */

/*
 * y[r] = W_down . bf16(fp32(silu(W_gate . x[r]) * (W_up . x[r])))
 * for n rows through one expert (Beam blog, "Mixture of Experts": each
 * expert is a SwiGLU MLP with intermediate size 2,560; "Residual Stream":
 * the SwiGLU product is computed in FP32).
 *
 * x      bf16 [n, H]      w_gate bf16 [I, H]   w_up bf16 [I, H]
 * w_down bf16 [H, I]      y      double [n, H] (out)
 * h_out  bf16 [n, I] (out, may be NULL): the rounded SwiGLU activations.
 */
void oracle_expert_swiglu(int n, int H, int I, const uint16_t *x,
                          const uint16_t *w_gate, const uint16_t *w_up,
                          const uint16_t *w_down, double *y, uint16_t *h_out)
{
    double *hv = (double *)malloc(sizeof(double) * (size_t)I);
    for (int r = 0; r < n; ++r) {
        const uint16_t *xr = x + (size_t)r * H;
        /* every output element is one sequential sum; the threads split the
         * independent outputs, never a sum */
#pragma omp parallel for schedule(static)
        for (int i = 0; i < I; ++i) {
            const uint16_t *wg = w_gate + (size_t)i * H;
            const uint16_t *wu = w_up + (size_t)i * H;
            double g = 0.0, u = 0.0;
            for (int h = 0; h < H; ++h) {
                double xv = oracle_bf16_to_double(xr[h]);
                g += xv * oracle_bf16_to_double(wg[h]);
                u += xv * oracle_bf16_to_double(wu[h]);
            }
            float p32 = (float)(silu(g) * u);            /* FP32 SwiGLU product */
            uint16_t hb = oracle_double_to_bf16((double)p32); /* down GEMM input */
            hv[i] = oracle_bf16_to_double(hb);
            if (h_out) h_out[(size_t)r * I + i] = hb;
        }
#pragma omp parallel for schedule(static)
        for (int h = 0; h < H; ++h) {
            const uint16_t *wd = w_down + (size_t)h * I;
            double acc = 0.0;
            for (int i = 0; i < I; ++i) acc += hv[i] * oracle_bf16_to_double(wd[i]);
            y[(size_t)r * H + h] = acc;
        }
    }
    free(hv);
}

/* ------------------------------------------------------------------ */
/* One SwiGLU expert with NVFP4 weights                                 */
/* ------------------------------------------------------------------ */

/*
 * NVFP4 weights (the 4-bit checkpoint format the Beam pages name for
 * Blackwell GPUs): 4-bit E2M1 elements, one FP8 E4M3 scale per 16
 * consecutive elements of a row, one FP32 scale per tensor:
 *   w[r][k] = e2m1(code[r][k]) * e4m3(scale[r][k / 16]) * global.
 * Codes: two per byte, element 2j in the low nibble of byte j of the row.
 * Both small formats are decoded from their definitions: E2M1 is sign,
 * 2 exponent bits (bias 1), 1 mantissa bit, exponent 0 subnormal (m * 0.5);
 * E4M3 is sign, 4 exponent bits (bias 7), 3 mantissa bits, exponent 0
 * subnormal (m / 8 * 2^-6), all-ones exponent and mantissa NaN, no infinity.
 */
double oracle_e2m1_value(unsigned code)
{
    const int sgn = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sgn ? -v : v;
}

double oracle_e4m3_value(unsigned byte)
{
    const int sgn = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    double v;
    if (e == 15 && m == 7) v = NAN;
    else if (e == 0) v = ldexp(m / 8.0, -6);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* Row r of an NVFP4 matrix with K columns, decoded into w[0..K-1]. */
static void nvfp4_row(const uint8_t *codes, const uint8_t *scales, double global, int K, size_t r,
                      double *w)
{
    const uint8_t *c = codes + r * (size_t)(K / 2);
    const uint8_t *sc = scales + r * (size_t)(K / 16);
    for (int k = 0; k < K; ++k) {
        const unsigned code = (k & 1) ? (c[k / 2] >> 4) & 15u : c[k / 2] & 15u;
        w[k] = oracle_e2m1_value(code) * oracle_e4m3_value(sc[k / 16]) * global;
    }
}

/*
 * oracle_expert_swiglu with the expert's three matrices in NVFP4:
 * gate, up [I, H] and down [H, I] as codes (uint8, K/2 per row), scales
 * (uint8, K/16 per row) and a per-tensor scale.  Same arithmetic otherwise:
 * double sums in index order, the SwiGLU product rounded to FP32 then bf16.
 */
void oracle_expert_swiglu_nvfp4(int n, int H, int I, const uint16_t *x,
                                const uint8_t *gate_codes, const uint8_t *gate_scales,
                                const uint8_t *up_codes, const uint8_t *up_scales,
                                const uint8_t *down_codes, const uint8_t *down_scales,
                                double gate_global, double up_global, double down_global,
                                double *y, uint16_t *h_out)
{
    double *hv = (double *)malloc(sizeof(double) * (size_t)I);
    for (int r = 0; r < n; ++r) {
        const uint16_t *xr = x + (size_t)r * H;
#pragma omp parallel for schedule(static)
        for (int i = 0; i < I; ++i) {
            double *wg = (double *)malloc(sizeof(double) * (size_t)H);
            double *wu = (double *)malloc(sizeof(double) * (size_t)H);
            nvfp4_row(gate_codes, gate_scales, gate_global, H, (size_t)i, wg);
            nvfp4_row(up_codes, up_scales, up_global, H, (size_t)i, wu);
            double g = 0.0, u = 0.0;
            for (int h = 0; h < H; ++h) {
                double xv = oracle_bf16_to_double(xr[h]);
                g += xv * wg[h];
                u += xv * wu[h];
            }
            float p32 = (float)(silu(g) * u);
            uint16_t hb = oracle_double_to_bf16((double)p32);
            hv[i] = oracle_bf16_to_double(hb);
            if (h_out) h_out[(size_t)r * I + i] = hb;
            free(wg);
            free(wu);
        }
#pragma omp parallel for schedule(static)
        for (int h = 0; h < H; ++h) {
            double *wd = (double *)malloc(sizeof(double) * (size_t)I);
            nvfp4_row(down_codes, down_scales, down_global, I, (size_t)h, wd);
            double acc = 0.0;
            for (int i = 0; i < I; ++i) acc += hv[i] * wd[i];
            y[(size_t)r * H + h] = acc;
            free(wd);
        }
    }
    free(hv);
}

/* ------------------------------------------------------------------ */
/* Combine                                                              */
/* ------------------------------------------------------------------ */

/*
 * o[t] = scale * sum_{j=0..k-1} w[t,j] * y[t,j]   (slot order, double)
 * out[t] = bf16(o[t])
 * (Beam blog, "Mixture of Experts": expert outputs combined with the
 * normalised router weights and scaled by 2.5.)
 * y double [T, k, H]; w double [T, k]; o double [T, H] (out, may be NULL);
 * out bf16 [T, H] (out, may be NULL).
 */
void oracle_combine(int T, int H, int k, const double *y, const double *w,
                    double scale, double *o, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[(size_t)t * k + j] * y[((size_t)t * k + j) * H + h];
            double v = scale * acc;
            if (o) o[(size_t)t * H + h] = v;
            if (out) out[(size_t)t * H + h] = oracle_double_to_bf16(v);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Post-norm and depth-scaled residual update                           */
/* ------------------------------------------------------------------ */

/*
 * Sandwich post-norm (RMSNorm, weight multiplied) followed by the
 * depth-scaled residual update at step kstep (Beam blog, "Residual Stream":
 * at step k the sub-layer output enters with weight 1/sqrt(k) and the old
 * stream keeps weight sqrt((k-1)/k); every sub-layer is normalised before
 * and after).
 *   n[t]       = o[t] / sqrt(mean_h(o[t]^2) + eps) * gamma     (if gamma)
 *              = o[t]                                          (if !gamma)
 *   contrib[t] = n[t] / sqrt(kstep)
 *   stream'[t] = sqrt((kstep-1)/kstep) * stream[t] + contrib[t]
 * o double [T, H]; gamma fp32 [H] or NULL; stream fp32 [T, H];
 * contrib double [T, H] (out, may be NULL); stream_out double [T, H] (out,
 * may be NULL).
 */
void oracle_post_norm_residual(int T, int H, const double *o, const float *gamma,
                               double eps, int kstep, const float *stream,
                               double *contrib, double *stream_out)
{
    const double keep = sqrt((double)(kstep - 1) / (double)kstep);
    const double add = 1.0 / sqrt((double)kstep);
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const double *ot = o + (size_t)t * H;
        double inv_rms = 1.0;
        if (gamma) {
            double ss = 0.0;
            for (int h = 0; h < H; ++h) ss += ot[h] * ot[h];
            inv_rms = 1.0 / sqrt(ss / (double)H + eps);
        }
        for (int h = 0; h < H; ++h) {
            double n = gamma ? ot[h] * inv_rms * (double)gamma[h] : ot[h];
            double c = n * add;
            if (contrib) contrib[(size_t)t * H + h] = c;
            if (stream_out)
                stream_out[(size_t)t * H + h] = keep * (double)stream[(size_t)t * H + h] + c;
        }
    }
}
