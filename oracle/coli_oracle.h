/*
 * coli_oracle.h -- plain, slow, obviously-correct CPU oracle for the routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is the yardstick the CUDA path is checked against.
 * Nothing in the product path may link, load or call it: only the tests, the package's smoke
 * check and the benchmark's CPU-baseline leg do.  It shares no code, header, table or helper
 * with the CUDA library; the only thing the two have in common is the record *format* (an
 * interface) and the seeded inputs they are both fed.
 *
 * Everything is computed in IEEE double from the dequantised weights, following the fixture
 * rule of the JustVugg/colibri README, section "File: c/tools/README.md" (the reference output
 * is computed from the dequantised weights so that an engine reproduces it exactly).
 *
 * What the layer computes (colibri-strix README, "What's implemented": a DeepSeek-V3 sigmoid
 * router (noaux_tc bias, routed_scaling_factor), a shared expert, batch-union MoE,
 * int8 / packed int4 / packed int2 containers with per-row scales and dequant-on-use):
 *
 *   a1 gate     logits[t,e] = (float) sum_h x[t,h] * Wr[e,h]            (double sum, h order)
 *   a2 route    s = sigmoid(logit); c = s + bias; group score = top-2 sum of c in the group;
 *               keep topk_group groups; top_k of c among kept experts; w_k = s_k/sum(s)*rsf
 *   a3 group    counting sort of the T*K slots by expert id (stable), unique ids ascending
 *   a4/a5 FFN   y = Wd * (SiLU(Wg x) .* (Wu x)), weights = code * row scale (exact in double)
 *   a6/a7       out[t] = sum_k w[t,k] * y_{e_k}(x_t)  (k ascending)  +  y_shared(x_t)
 *
 * Parity status: every function here is pinned by tests that do not call it back (brute-force
 * top-k enumeration, exhaustive container round trips, closed-form FFN cases, invariants).
 * The absolute values of a full-size layer output are pinned only through those pieces; the
 * pages print no worked numeric example of the layer.
 */
#ifndef COLI_ORACLE_H
#define COLI_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Layer configuration (host).  fmt: bits per weight code (4 = packed int4, 8 = int8, 2 = packed
 * int2).  act: 0 = float32 activations, 1 = bfloat16 activations (raw 16-bit patterns). */
typedef struct {
    int hidden;        /* H */
    int inter;         /* I, routed expert intermediate size */
    int n_experts;     /* E */
    int top_k;         /* K */
    int n_group;       /* G */
    int topk_group;    /* TG */
    int n_shared;      /* 0 or 1 */
    int shared_inter;  /* I_s */
    double routed_scaling;
    int fmt;           /* 4, 8 or 2 */
    int act;           /* 0 f32, 1 bf16 */
    int group;         /* 0: one scale per row; g > 0: one scale per g consecutive columns */
} oracle_cfg;

/* Bytes of one expert record with intermediate size `inter` (unpadded; callers pad to 256).
 * Record layout: Wg codes [I][H], Wu codes [I][H], Wd codes [H][I] (row-major, each row packed
 * to whole bytes), then float32 scales sg, su, sd: per row (sg[I], su[I], sd[H]) when group is
 * 0, else per group of `group` consecutive columns (sg[I][H/group], su[I][H/group],
 * sd[H][I/group]).  Returns 0 on success, -1 when a size does not fit the format. */
int oracle_record_bytes(int hidden, int inter, int fmt, int group, size_t *bytes);

/* Container decode: n codes of one packed row -> two's-complement integers.
 * int4: element 2j in the low nibble of byte j, 2j+1 in the high nibble, range [-8, 7].
 * int2: element 4j+k in bits [2k, 2k+1] of byte j, range [-2, 1].
 * int8: one signed byte per element.  Returns 0, or -1 on a bad fmt / length. */
int oracle_unpack_row(const uint8_t *row, int n, int fmt, int8_t *q);

/* Container encode (used only by the bit-identity pins).  Codes outside the format's range are
 * rejected with -1. */
int oracle_pack_row(const int8_t *q, int n, int fmt, uint8_t *row);

/* a1: logits[T,E] (float32). x is [T,H] float32 or bf16 bits per cfg->act; Wr is [E,H] f32. */
void oracle_gate(const oracle_cfg *cfg, const float *Wr, const void *x, int T, float *logits);

/* a2: ids[T,K], w[T,K].  Optional diagnostics (may be NULL): margin_expert[t] = c of the K-th
 * pick minus the best c left out among kept experts (+inf if none is left), margin_group[t] =
 * TG-th minus (TG+1)-th group score (+inf when G == 1 or TG == G).  Returns 0, -1 on bad cfg. */
int oracle_route(const oracle_cfg *cfg, const float *logits, const float *bias, int T,
                 int32_t *ids, float *w, double *margin_expert, double *margin_group);

/* a3: counting sort of slots s = t*K + k by ids[s].  counts[E], offsets[E+1], perm[T*K],
 * unique[E] (first n_unique entries valid, ascending), n_unique[1].  Returns 0, -1 on an id out
 * of range. */
int oracle_group(int T, int K, int E, const int32_t *ids, int32_t *counts, int32_t *offsets,
                 int32_t *perm, int32_t *unique, int32_t *n_unique);

/* One expert on one token: y[H] = Wd (SiLU(Wg x) .* (Wu x)) over the dequantised record. */
void oracle_expert(const oracle_cfg *cfg, const uint8_t *record, int inter, const double *x,
                   double *y);

/* a4..a7 for given routing, per token (token by token, slot k ascending, shared last).
 * experts[e] points at expert e's record (may be NULL for experts no slot selects).
 * shared may be NULL when cfg->n_shared == 0.  out is [T,H] double. */
int oracle_ffn(const oracle_cfg *cfg, const uint8_t *const *experts, const uint8_t *shared,
               const void *x, int T, const int32_t *ids, const float *w, double *out);

/* Same result computed the batch-union way: each unique expert is visited once and applied to
 * every slot routed to it, then slots are combined per token in k order.  Must equal
 * oracle_ffn bit for bit (same double operations in the same order per (token, expert)). */
int oracle_ffn_union(const oracle_cfg *cfg, const uint8_t *const *experts,
                     const uint8_t *shared, const void *x, int T, const int32_t *ids,
                     const float *w, double *out);

/* The whole layer: gate, route, FFN.  ids/w/logits outputs may be NULL.  n_threads > 1 runs
 * independent tokens on that many OpenMP threads (same arithmetic per token). */
int oracle_layer(const oracle_cfg *cfg, const float *Wr, const float *bias,
                 const uint8_t *const *experts, const uint8_t *shared, const void *x, int T,
                 double *out, int32_t *ids, float *w, float *logits, int n_threads);

/* Residual update between chained layers (JustVugg/colibri README, "Never wait for the disk
 * twice": the residual stream stays on the device from layer to layer).  For n elements,
 * x_next = x + out as one IEEE single addition; with bf16 activations (cfg->act = 1) x and
 * x_next are bf16 bit patterns and the sum is rounded to bf16, round to nearest even (a NaN
 * stays a quiet NaN); with float32 activations both are float32. */
void oracle_residual(const oracle_cfg *cfg, const void *x, const float *out, size_t n, void *x_next);

#ifdef __cplusplus
}
#endif
#endif /* COLI_ORACLE_H */
