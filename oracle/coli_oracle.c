/*
 * coli_oracle.c -- the CPU oracle (test infrastructure; see coli_oracle.h).
 *
 * Plain C99, IEEE double throughout, no blocking, no fusion, no reordering beyond what the
 * definitions state.  Each function names the passage of the pages it follows.
 */
#include "coli_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- containers (a8) -------- */

static int row_bytes(int n, int fmt, size_t *out)
{
    if (n < 0) return -1;
    if (fmt == 8) { *out = (size_t)n; return 0; }
    if (fmt == 4) { if (n % 2) return -1; *out = (size_t)n / 2; return 0; }
    if (fmt == 2) { if (n % 4) return -1; *out = (size_t)n / 4; return 0; }
    return -1;
}

/* Scales per row of a matrix with `cols` columns: one (per-row container) or cols / group
 * (group-scaled container, JustVugg/colibri README, "Get started -> 2. Get the model": the
 * recommended GLM-5.2 build is group-scaled, gs64).  -1 when group does not divide cols. */
static long scales_per_row(int cols, int group)
{
    if (group == 0) return 1;
    if (group < 0 || cols % group) return -1;
    return cols / group;
}

/* Record = three code matrices stored adjacent, then their scales (JustVugg/colibri README,
 * "Never wait for the disk twice": an expert's three matrices sit next to each other). */
int oracle_record_bytes(int hidden, int inter, int fmt, int group, size_t *bytes)
{
    size_t rh, ri;
    if (row_bytes(hidden, fmt, &rh) || row_bytes(inter, fmt, &ri)) return -1;
    const long nh = scales_per_row(hidden, group), ni = scales_per_row(inter, group);
    if (nh < 0 || ni < 0) return -1;
    *bytes = 2 * (size_t)inter * rh + (size_t)hidden * ri
           + (2 * (size_t)inter * (size_t)nh + (size_t)hidden * (size_t)ni) * sizeof(float);
    return 0;
}

/* Decode a packed row (colibri-strix README, "What's implemented": packed int4 and int2 rows
 * decode to exactly the codes of the int8 container).  Two's complement in 4 or 2 bits. */
int oracle_unpack_row(const uint8_t *row, int n, int fmt, int8_t *q)
{
    size_t nb;
    if (row_bytes(n, fmt, &nb)) return -1;
    for (int j = 0; j < n; j++) {
        int v;
        if (fmt == 8) {
            v = (int)(int8_t)row[j];
        } else if (fmt == 4) {
            int byte = row[j / 2];
            int nib = (j % 2 == 0) ? (byte & 0x0F) : ((byte >> 4) & 0x0F);
            v = (nib >= 8) ? nib - 16 : nib;
        } else {
            int byte = row[j / 4];
            int code = (byte >> (2 * (j % 4))) & 0x03;
            v = (code >= 2) ? code - 4 : code;
        }
        q[j] = (int8_t)v;
    }
    return 0;
}

int oracle_pack_row(const int8_t *q, int n, int fmt, uint8_t *row)
{
    size_t nb;
    if (row_bytes(n, fmt, &nb)) return -1;
    memset(row, 0, nb);
    for (int j = 0; j < n; j++) {
        int v = q[j];
        if (fmt == 8) {
            row[j] = (uint8_t)(int8_t)v;
        } else if (fmt == 4) {
            if (v < -8 || v > 7) return -1;
            int nib = v & 0x0F;
            row[j / 2] |= (uint8_t)((j % 2 == 0) ? nib : (nib << 4));
        } else {
            if (v < -2 || v > 1) return -1;
            int code = v & 0x03;
            row[j / 4] |= (uint8_t)(code << (2 * (j % 4)));
        }
    }
    return 0;
}

/* Dequantise one element: weight = code * its scale, exact in double (dequant-on-use,
 * colibri-strix README, "What's implemented").  The scale is the row's (group == 0) or that of
 * the element's group of `group` consecutive columns of the row. */
static double dequant(const uint8_t *mat, size_t rb, int fmt, const float *scales, int r, int c,
                      int cols, int group)
{
    const uint8_t *row = mat + (size_t)r * rb;
    int v;
    if (fmt == 8) {
        v = (int)(int8_t)row[c];
    } else if (fmt == 4) {
        int byte = row[c / 2];
        int nib = (c % 2 == 0) ? (byte & 0x0F) : ((byte >> 4) & 0x0F);
        v = (nib >= 8) ? nib - 16 : nib;
    } else {
        int byte = row[c / 4];
        int code = (byte >> (2 * (c % 4))) & 0x03;
        v = (code >= 2) ? code - 4 : code;
    }
    const size_t si = group == 0 ? (size_t)r : (size_t)r * (size_t)(cols / group) + (size_t)(c / group);
    return (double)v * (double)scales[si];
}

/* ---------------------------------------------------------------- activations ------------- */

static double act_value(const oracle_cfg *cfg, const void *x, size_t idx)
{
    if (cfg->act == 0) return (double)((const float *)x)[idx];
    uint16_t b = ((const uint16_t *)x)[idx];
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------- a1 gate ----------------- */

/* Router gate projection: one dot product per (token, expert), summed in h order in double
 * and rounded once to float32 (colibri-strix README, "What's implemented": sigmoid router). */
void oracle_gate(const oracle_cfg *cfg, const float *Wr, const void *x, int T, float *logits)
{
    const int H = cfg->hidden, E = cfg->n_experts;
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            double acc = 0.0;
            for (int h = 0; h < H; h++)
                acc += act_value(cfg, x, (size_t)t * H + h) * (double)Wr[(size_t)e * H + h];
            logits[(size_t)t * E + e] = (float)acc;
        }
}

/* ---------------------------------------------------------------- a2 route ---------------- */

/* "a beats b": larger value first, equal values resolved toward the lower index. */
static int beats(double va, int ia, double vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

/* The sigmoid router of DeepSeek-V3 with its noaux_tc selection bias and routed_scaling_factor
 * (colibri-strix README, "What's implemented").  Readings where the pages are silent: the
 * bias steers selection only; a group scores the sum of its two largest biased scores; only
 * experts of the kept groups can be chosen; ties go to the lower index; slots are ordered by
 * descending biased score; weights are the unbiased scores renormalised to sum to one, then
 * multiplied by routed_scaling. */
int oracle_route(const oracle_cfg *cfg, const float *logits, const float *bias, int T,
                 int32_t *ids, float *w, double *margin_expert, double *margin_group)
{
    const int E = cfg->n_experts, K = cfg->top_k, G = cfg->n_group, TG = cfg->topk_group;
    if (E <= 0 || K <= 0 || G <= 0 || E % G != 0 || TG <= 0 || TG > G) return -1;
    const int gs = E / G;
    if (G > 1 && gs < 2) return -1;
    if (K > TG * gs) return -1;

    double *s = (double *)malloc(sizeof(double) * E);
    double *c = (double *)malloc(sizeof(double) * E);
    double *gscore = (double *)malloc(sizeof(double) * G);
    int *kept = (int *)malloc(sizeof(int) * G);
    int *taken = (int *)malloc(sizeof(int) * E);
    double *sel_s = (double *)malloc(sizeof(double) * K);

    for (int t = 0; t < T; t++) {
        for (int e = 0; e < E; e++) {
            double l = (double)logits[(size_t)t * E + e];
            s[e] = 1.0 / (1.0 + exp(-l));
            c[e] = s[e] + (double)bias[e];
        }
        /* group stage */
        double mg = INFINITY;
        if (G == 1 || TG == G) {
            for (int g = 0; g < G; g++) kept[g] = 1;
        } else {
            for (int g = 0; g < G; g++) {
                int b1 = -1, b2 = -1;
                for (int e = g * gs; e < (g + 1) * gs; e++) {
                    if (b1 < 0 || beats(c[e], e, c[b1], b1)) { b2 = b1; b1 = e; }
                    else if (b2 < 0 || beats(c[e], e, c[b2], b2)) { b2 = e; }
                }
                gscore[g] = c[b1] + c[b2];
                kept[g] = 0;
            }
            double last = 0.0;
            for (int r = 0; r < TG; r++) {
                int best = -1;
                for (int g = 0; g < G; g++)
                    if (!kept[g] && (best < 0 || beats(gscore[g], g, gscore[best], best))) best = g;
                kept[best] = 1;
                last = gscore[best];
            }
            double next = -INFINITY;
            for (int g = 0; g < G; g++)
                if (!kept[g] && gscore[g] > next) next = gscore[g];
            mg = last - next;
        }
        /* expert stage: K repeated arg-max picks among kept experts */
        for (int e = 0; e < E; e++) taken[e] = 0;
        double lastc = 0.0;
        for (int k = 0; k < K; k++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (!kept[e / gs] || taken[e]) continue;
                if (best < 0 || beats(c[e], e, c[best], best)) best = e;
            }
            taken[best] = 1;
            ids[(size_t)t * K + k] = best;
            sel_s[k] = s[best];
            lastc = c[best];
        }
        double nextc = -INFINITY;
        for (int e = 0; e < E; e++)
            if (kept[e / gs] && !taken[e] && c[e] > nextc) nextc = c[e];
        /* renormalise (sum in slot order) and scale */
        double denom = 0.0;
        for (int k = 0; k < K; k++) denom += sel_s[k];
        for (int k = 0; k < K; k++)
            w[(size_t)t * K + k] = (float)((sel_s[k] / denom) * cfg->routed_scaling);
        if (margin_expert) margin_expert[t] = lastc - nextc;
        if (margin_group) margin_group[t] = mg;
    }
    free(s); free(c); free(gscore); free(kept); free(taken); free(sel_s);
    return 0;
}

/* ---------------------------------------------------------------- a3 group ---------------- */

/* Batch-union grouping (colibri-strix README, "What's implemented": an expert chosen anywhere
 * in the batch is fetched once and used for all the positions that chose it): a stable
 * counting sort of the slots by expert id. */
int oracle_group(int T, int K, int E, const int32_t *ids, int32_t *counts, int32_t *offsets,
                 int32_t *perm, int32_t *unique, int32_t *n_unique)
{
    const int n = T * K;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int s = 0; s < n; s++) {
        if (ids[s] < 0 || ids[s] >= E) return -1;
        counts[ids[s]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (E > 0 ? E : 1));
    for (int e = 0; e < E; e++) cursor[e] = offsets[e];
    for (int s = 0; s < n; s++) perm[cursor[ids[s]]++] = s;
    free(cursor);
    int u = 0;
    for (int e = 0; e < E; e++)
        if (counts[e] > 0) unique[u++] = e;
    for (int e = u; e < E; e++) unique[e] = -1;
    *n_unique = u;
    return 0;
}

/* ---------------------------------------------------------------- a4/a5 expert FFN -------- */

/* SwiGLU expert over the dequantised record: a = SiLU(Wg x) .* (Wu x), y = Wd a, with
 * SiLU(g) = g / (1 + exp(-g)).  Weights are dequantised element by element (dequant-on-use). */
void oracle_expert(const oracle_cfg *cfg, const uint8_t *record, int inter, const double *x,
                   double *y)
{
    const int H = cfg->hidden, I = inter, fmt = cfg->fmt;
    size_t rh = 0, ri = 0;
    if (H <= 0 || I <= 0 || row_bytes(H, fmt, &rh) || row_bytes(I, fmt, &ri)) {
        for (int j = 0; j < H; j++) y[j] = NAN;
        return;
    }
    const int grp = cfg->group;
    const long nh = scales_per_row(H, grp), ni = scales_per_row(I, grp);
    if (nh < 0 || ni < 0) {
        for (int j = 0; j < H; j++) y[j] = NAN;
        return;
    }
    const uint8_t *Wg = record;
    const uint8_t *Wu = Wg + (size_t)I * rh;
    const uint8_t *Wd = Wu + (size_t)I * rh;
    const float *sg = (const float *)(Wd + (size_t)H * ri);
    const float *su = sg + (size_t)I * nh;
    const float *sd = su + (size_t)I * nh;

    double *a = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; i++) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; h++) {
            g += dequant(Wg, rh, fmt, sg, i, h, H, grp) * x[h];
            u += dequant(Wu, rh, fmt, su, i, h, H, grp) * x[h];
        }
        a[i] = (g / (1.0 + exp(-g))) * u;
    }
    for (int j = 0; j < H; j++) {
        double acc = 0.0;
        for (int i = 0; i < I; i++) acc += dequant(Wd, ri, fmt, sd, j, i, I, grp) * a[i];
        y[j] = acc;
    }
    free(a);
}

/* ---------------------------------------------------------------- a6/a7 combine ----------- */

static int ffn_token(const oracle_cfg *cfg, const uint8_t *const *experts, const uint8_t *shared,
                     const double *xt, const int32_t *ids_t, const float *w_t, double *out_t,
                     double *ybuf)
{
    const int H = cfg->hidden, K = cfg->top_k;
    for (int j = 0; j < H; j++) out_t[j] = 0.0;
    for (int k = 0; k < K; k++) {
        int e = ids_t[k];
        if (e < 0 || e >= cfg->n_experts || experts[e] == NULL) return -1;
        oracle_expert(cfg, experts[e], cfg->inter, xt, ybuf);
        for (int j = 0; j < H; j++) out_t[j] += (double)w_t[k] * ybuf[j];
    }
    if (cfg->n_shared > 0) {
        if (shared == NULL) return -1;
        oracle_expert(cfg, shared, cfg->shared_inter, xt, ybuf);
        for (int j = 0; j < H; j++) out_t[j] += ybuf[j];
    }
    return 0;
}

/* Weighted combine of the routed experts plus the always-on shared expert (colibri-strix
 * README, "What's implemented": shared expert).  The shared expert is added with weight one. */
int oracle_ffn(const oracle_cfg *cfg, const uint8_t *const *experts, const uint8_t *shared,
               const void *x, int T, const int32_t *ids, const float *w, double *out)
{
    const int H = cfg->hidden, K = cfg->top_k;
    double *xt = (double *)malloc(sizeof(double) * H);
    double *yb = (double *)malloc(sizeof(double) * H);
    int rc = 0;
    for (int t = 0; t < T && rc == 0; t++) {
        for (int h = 0; h < H; h++) xt[h] = act_value(cfg, x, (size_t)t * H + h);
        rc = ffn_token(cfg, experts, shared, xt, ids + (size_t)t * K, w + (size_t)t * K,
                       out + (size_t)t * H, yb);
    }
    free(xt); free(yb);
    return rc;
}

int oracle_ffn_union(const oracle_cfg *cfg, const uint8_t *const *experts,
                     const uint8_t *shared, const void *x, int T, const int32_t *ids,
                     const float *w, double *out)
{
    const int H = cfg->hidden, K = cfg->top_k, E = cfg->n_experts;
    const int n = T * K;
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (E + 1));
    int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (n > 0 ? n : 1));
    int32_t *uniq = (int32_t *)malloc(sizeof(int32_t) * E);
    int32_t nu = 0;
    double *yslot = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * H);
    double *xt = (double *)malloc(sizeof(double) * H);
    int rc = oracle_group(T, K, E, ids, counts, offsets, perm, uniq, &nu);
    /* each unique expert once, applied to every slot routed to it */
    for (int u = 0; u < nu && rc == 0; u++) {
        int e = uniq[u];
        if (experts[e] == NULL) { rc = -1; break; }
        for (int p = offsets[e]; p < offsets[e + 1]; p++) {
            int s = perm[p], t = s / K;
            for (int h = 0; h < H; h++) xt[h] = act_value(cfg, x, (size_t)t * H + h);
            oracle_expert(cfg, experts[e], cfg->inter, xt, yslot + (size_t)s * H);
        }
    }
    /* combine per token, k ascending, shared last */
    for (int t = 0; t < T && rc == 0; t++) {
        double *o = out + (size_t)t * H;
        for (int j = 0; j < H; j++) o[j] = 0.0;
        for (int k = 0; k < K; k++) {
            const double *ys = yslot + ((size_t)t * K + k) * H;
            for (int j = 0; j < H; j++) o[j] += (double)w[(size_t)t * K + k] * ys[j];
        }
        if (cfg->n_shared > 0) {
            if (shared == NULL) { rc = -1; break; }
            for (int h = 0; h < H; h++) xt[h] = act_value(cfg, x, (size_t)t * H + h);
            double *yb = (double *)malloc(sizeof(double) * H);
            oracle_expert(cfg, shared, cfg->shared_inter, xt, yb);
            for (int j = 0; j < H; j++) o[j] += yb[j];
            free(yb);
        }
    }
    free(counts); free(offsets); free(perm); free(uniq); free(yslot); free(xt);
    return rc;
}

/* ---------------------------------------------------------------- residual ---------------- */

/* float -> bf16 bits, round to nearest even on the dropped low half. */
static uint16_t bf16_round_even(float v) {
    uint32_t u;
    memcpy(&u, &v, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* NaN */
    uint32_t keep = u >> 16, dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

void oracle_residual(const oracle_cfg *cfg, const void *x, const float *out, size_t n, void *x_next) {
    if (cfg->act == 1) {
        const uint16_t *xb = (const uint16_t *)x;
        uint16_t *nb = (uint16_t *)x_next;
        for (size_t i = 0; i < n; i++) {
            uint32_t u = (uint32_t)xb[i] << 16;
            float xv;
            memcpy(&xv, &u, sizeof xv);
            float s = xv + out[i];
            nb[i] = bf16_round_even(s);
        }
    } else {
        const float *xf = (const float *)x;
        float *nf = (float *)x_next;
        for (size_t i = 0; i < n; i++) nf[i] = xf[i] + out[i];
    }
}

/* ---------------------------------------------------------------- whole layer ------------- */

int oracle_layer(const oracle_cfg *cfg, const float *Wr, const float *bias,
                 const uint8_t *const *experts, const uint8_t *shared, const void *x, int T,
                 double *out, int32_t *ids, float *w, float *logits, int n_threads)
{
    const int H = cfg->hidden, E = cfg->n_experts, K = cfg->top_k;
    int rc = 0;
    if (n_threads < 1) n_threads = 1;
#ifdef _OPENMP
#pragma omp parallel for num_threads(n_threads) schedule(dynamic, 1) reduction(| : rc)
#endif
    for (int t = 0; t < T; t++) {
        float *lg = (float *)malloc(sizeof(float) * E);
        int32_t *it = (int32_t *)malloc(sizeof(int32_t) * K);
        float *wt = (float *)malloc(sizeof(float) * K);
        double *xt = (double *)malloc(sizeof(double) * H);
        double *yb = (double *)malloc(sizeof(double) * H);
        const void *xrow = (cfg->act == 0) ? (const void *)((const float *)x + (size_t)t * H)
                                           : (const void *)((const uint16_t *)x + (size_t)t * H);
        oracle_gate(cfg, Wr, xrow, 1, lg);
        int r = oracle_route(cfg, lg, bias, 1, it, wt, NULL, NULL);
        if (r == 0) {
            for (int h = 0; h < H; h++) xt[h] = act_value(cfg, xrow, (size_t)h);
            r = ffn_token(cfg, experts, shared, xt, it, wt, out + (size_t)t * H, yb);
        }
        if (ids) memcpy(ids + (size_t)t * K, it, sizeof(int32_t) * K);
        if (w) memcpy(w + (size_t)t * K, wt, sizeof(float) * K);
        if (logits) memcpy(logits + (size_t)t * E, lg, sizeof(float) * E);
        free(lg); free(it); free(wt); free(xt); free(yb);
        rc |= (r != 0);
    }
    return rc ? -1 : 0;
}
