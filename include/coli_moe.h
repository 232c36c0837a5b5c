/*
 * coli_moe.h -- C ABI of the routed-expert MoE layer on NVIDIA B200 (sm_100a).
 *
 * The layer (colibri-strix README, "What's implemented"): a sigmoid router in the DeepSeek-V3
 * manner, whose noaux_tc bias steers the selection and whose weights are renormalised and scaled
 * by routed_scaling_factor; batch-union grouping, in which every expert that some token of the
 * batch selects is fetched one time and serves all of those tokens; SwiGLU experts stored as
 * packed int4 (also int8 / packed int2) with per-row scales, dequantised on use; a shared
 * expert; and the weighted combine.  The JustVugg/colibri README ("Never wait for the disk
 * twice") keeps an expert's gate, up and down matrices together in one record.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library allocates no
 *     device memory; scratch comes from a caller-provided workspace (coli_moe_workspace_size).
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).  Host-side validation happens before any launch; a non-OK
 *     status means nothing was launched.
 *   - Device-side anomalies (an expert id out of range, inconsistent grouping arrays) never
 *     trap: the kernel skips the bad item and records a code in the workspace's error word,
 *     which coli_moe_error_word() reads back.
 *   - There is no CPU fallback: every step runs in this library's CUDA kernels.
 *
 * Record format (one per expert; the same for the shared expert with its own inter size)
 *   Wg codes [I][H] | Wu codes [I][H] | Wd codes [H][I] | sg | su | sd (float32 scales),
 *   rows packed to whole bytes: int4 element 2j in the low nibble of byte j and 2j+1 in the
 *   high nibble (two's complement, [-8,7]); int2 element 4j+k in bits [2k,2k+1] of byte j
 *   ([-2,1]); int8 one signed byte.  Per-row container (group_size 0): sg[I], su[I], sd[H], the
 *   weight is code * scale of its output row.  Group-scaled container (group_size 64, int4 only;
 *   the JustVugg/colibri README, "Get started -> 2. Get the model", recommends this GLM-5.2
 *   build): sg[I][H/64], su[I][H/64], sd[H][I/64], the weight is code * scale of its group of 64
 *   consecutive columns of the row.  Records sit `expert_stride` bytes apart (a multiple of
 *   256) and the record base must be 256-byte aligned.
 *
 * Tensor layouts (row-major):
 *   x        [T][H]   float32 (act = COLI_ACT_F32) or bfloat16 bits (COLI_ACT_BF16), 16-B aligned
 *   logits   [T][E]   float32
 *   topk_ids [T][K]   int32, slot order = descending biased score (ties: lower expert id)
 *   topk_w   [T][K]   float32
 *   out      [T][H]   float32, 16-B aligned
 */
#ifndef COLI_MOE_H
#define COLI_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    COLI_OK = 0,
    COLI_ERR_INVALID_ARG = 1,  /* NULL pointer, negative size, bad enum value */
    COLI_ERR_SHAPE = 2,        /* sizes inconsistent with each other or with the formats */
    COLI_ERR_ALIGN = 3,        /* a pointer or stride misses its required alignment */
    COLI_ERR_UNSUPPORTED = 4,  /* a valid configuration that this library does not implement */
    COLI_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch, attribute, copy) */
    COLI_ERR_DEVICE = 6,       /* the device error word was set by a kernel */
    COLI_ERR_WORKSPACE = 7     /* workspace NULL, misaligned or smaller than required */
} coli_status;

typedef enum { COLI_W_INT2 = 2, COLI_W_INT4 = 4, COLI_W_INT8 = 8 } coli_wfmt;
typedef enum { COLI_ACT_F32 = 0, COLI_ACT_BF16 = 1 } coli_act;

/* Device error word codes (bit flags, OR-ed together by the kernels). */
#define COLI_DEVERR_EXPERT_ID 0x1   /* an expert id or unique-list entry outside [0, E) */
#define COLI_DEVERR_GROUPING 0x2    /* offsets/perm inconsistent (slot outside [0, T*K)) */
#define COLI_DEVERR_TIMEOUT 0x4     /* a bounded device-side wait ran out (the call's output is invalid) */

typedef struct {
    int hidden;             /* H */
    int inter;              /* I, routed expert intermediate size */
    int n_experts;          /* E (<= 1024) */
    int top_k;              /* K (<= 32) */
    int n_group;            /* G; E % G == 0 */
    int topk_group;         /* TG, 1 <= TG <= G */
    int n_shared;           /* 0 or 1 */
    int shared_inter;       /* I_s; must equal inter when n_shared == 1 */
    double routed_scaling;  /* rsf */
    int wfmt;               /* coli_wfmt */
    int act;                /* coli_act */
    int group_size;         /* 0: one scale per weight row; 64: one per 64 columns (int4 only) */
} coli_moe_config;

typedef struct {
    const float *router_w;     /* [E][H] float32 */
    const float *router_bias;  /* [E] float32, the noaux_tc selection bias */
    const uint8_t *experts;    /* E records, expert_stride bytes apart, 256-B aligned */
    size_t expert_stride;      /* bytes; multiple of 256 and >= the record size */
    const uint8_t *shared;     /* the shared expert's record (NULL when n_shared == 0) */
} coli_moe_weights;

/* Text for a status code (static storage). */
const char *coli_moe_status_str(coli_status s);

/* Name and text of the CUDA error behind the calling thread's last COLI_ERR_CUDA ("" if none). */
const char *coli_moe_last_cuda_error(void);

/* Bytes of one record for (hidden, inter, wfmt, group_size), before padding to 256.  Host only. */
coli_status coli_moe_record_bytes(int hidden, int inter, int wfmt, int group_size, size_t *bytes);

/* Validates a configuration (the same checks every call makes).  Host only. */
coli_status coli_moe_check_config(const coli_moe_config *cfg);

/* Workspace bytes that coli_moe_layer / coli_moe_ffn / coli_moe_group need for up to
 * max_tokens tokens.  The workspace must be 256-byte aligned and is owned by the caller; calls
 * that share one workspace must be ordered on the GPU (same stream or events).  Its first 512
 * bytes (error word and the counters of the fused decode path) must be zero before its first
 * use: call coli_moe_clear_error once after allocating it (and after a call that reported
 * COLI_DEVERR_TIMEOUT).  Complete calls leave the header ready for the next call.  Host only. */
coli_status coli_moe_workspace_size(const coli_moe_config *cfg, int max_tokens, size_t *bytes);

/* Number of kernels coli_moe_layer launches for T tokens with this configuration (1 on the fused
 * decode path: one persistent kernel for the whole layer; 7 on the tensor-core path; 5
 * otherwise).  Host only. */
coli_status coli_moe_layer_kernels(const coli_moe_config *cfg, int T, int *n_kernels);

/* Zeroes the workspace header: the device error word and the counters (asynchronous). */
coli_status coli_moe_clear_error(void *ws, void *stream);

/* Synchronises `stream` and returns the workspace's device error word in *code (0 = clean). */
coli_status coli_moe_error_word(void *ws, void *stream, int *code);

/* a1, router gate projection (colibri-strix README, "What's implemented": sigmoid router).
 * logits[t][e] = float32( sum_h x[t][h] * router_w[e][h] ), the products and the sum taken in
 * double precision, rounded once to float32.  T = 0 is a no-op. */
coli_status coli_moe_gate(const coli_moe_config *cfg, const float *router_w, const void *x,
                          int T, float *logits, void *stream);

/* a2, noaux_tc routing (colibri-strix README, "What's implemented": the DeepSeek-V3 sigmoid
 * router, its noaux_tc bias and routed_scaling_factor).  Per token, in double: s = 1/(1+exp(-logit)),
 * c = s + bias; if G > 1 each group scores the sum of its two largest c and the TG best groups
 * are kept (ties: lower group); the K largest c among kept experts are selected (ties: lower
 * id), written in descending c order; topk_w[k] = float32(s_k / sum_k s_k * routed_scaling).
 * The bias steers selection only.  T = 0 is a no-op. */
coli_status coli_moe_route(const coli_moe_config *cfg, const float *logits, const float *bias,
                           int T, int32_t *topk_ids, float *topk_w, void *stream);

/* a3, batch-union grouping (colibri-strix README, "What's implemented": batch-union MoE).
 * A stable counting sort of the T*K slots s = t*K + k by expert id: counts[E], offsets[E+1]
 * (exclusive scan, offsets[E] = T*K), perm[T*K] (slot indices grouped by expert, ascending
 * slot index inside each expert), unique_ids[E] (ids with counts > 0, ascending, the rest -1),
 * n_unique[1].  Ids outside [0,E) are skipped and flagged in the error word of `ws`. */
coli_status coli_moe_group(const coli_moe_config *cfg, const int32_t *topk_ids, int T,
                           int32_t *counts, int32_t *offsets, int32_t *perm,
                           int32_t *unique_ids, int32_t *n_unique, void *ws, size_t ws_bytes,
                           void *stream);

/* a4..a7 for a given routing (JustVugg/colibri README, "Never wait for the disk twice":
 * the experts a batch needs are fetched once for all of its positions; colibri-strix README,
 * "What's implemented":
 * dequant-on-use, shared expert).  For every unique expert e and every slot routed to it:
 * y = sd .* (Qd (SiLU(sg .* (Qg x)) .* (su .* (Qu x)))) with the codes Q dequantised in
 * registers; out[t] = sum over t's experts of topk_w * y + y_shared (weight 1).  The grouping
 * arrays are those coli_moe_group writes.  `out` is fully overwritten.  Each expert's weights
 * are streamed from HBM once per call. */
coli_status coli_moe_ffn(const coli_moe_config *cfg, const coli_moe_weights *w, const void *x,
                         int T, const float *topk_w, const int32_t *offsets,
                         const int32_t *perm, const int32_t *unique_ids,
                         const int32_t *n_unique, float *out, void *ws, size_t ws_bytes,
                         void *stream);

/* The whole layer: gate, route, group, ffn (all of the above, in that order, on `stream`).
 * topk_ids_out / topk_w_out may be NULL; when given they receive the routing.
 * The call issues no host-blocking operation and reads no device data on the host, so it may be
 * captured into a CUDA graph and replayed: the fused decode kernel keeps its counters in the
 * workspace header, and consecutive calls (or replays) on one workspace must be ordered on the
 * GPU, as calls on one stream are.  Replays read the pointers captured with the call. */
coli_status coli_moe_layer(const coli_moe_config *cfg, const coli_moe_weights *w,
                           const void *x, int T, float *out, int32_t *topk_ids_out,
                           float *topk_w_out, void *ws, size_t ws_bytes, void *stream);

/* Residual update between chained layers (JustVugg/colibri README, "Never wait for the disk
 * twice": the GPU-resident pipeline keeps the residual stream on the device across layers).
 * x_next[t][h] = x[t][h] + out[t][h] for t < T, h < hidden: one float32 addition (round to
 * nearest even); with bf16 activations (cfg->act) x and x_next are bf16 and the sum is rounded
 * to bf16 (round to nearest even, NaN kept), with float32 activations they are float32.
 *   x, x_next  [T][hidden] device, row-major, the activation type of cfg; x_next may be x (in
 *              place) but must not overlap out.
 *   out        [T][hidden] float32 device, a layer's output.
 * Pointers 16-byte aligned (COLI_ERR_ALIGN otherwise); T < 0 is COLI_ERR_SHAPE, T = 0 a no-op.
 * Asynchronous on `stream`; allocates nothing. */
coli_status coli_moe_residual(const coli_moe_config *cfg, const void *x, const float *out, int T,
                              void *x_next, void *stream);

/* a5' per-expert dispatch on the grouped tensor-core path (batches above 4 tokens): within a call,
 * work experts with at most max_tokens routed tokens are computed by the CUDA-core GEMV kernels
 * (streaming their codes once at HBM speed) and the others by the grouped GEMM; the GEMV kernels'
 * down projection adds into out alongside the GEMM's combine.  0 puts every expert on the tensor
 * cores.  Process-wide, read at each call; coli_moe_layer_kernels then reports 9 kernels on that
 * path instead of 7.  Host only; COLI_ERR_INVALID_ARG outside [0, 65536]. */
coli_status coli_moe_set_dispatch_threshold(int max_tokens);
int coli_moe_dispatch_threshold(void);

/* Testing aid for the bounded device-side waits of the fused decode kernel (the one-launch
 * path that coli_moe_layer_kernels reports as 1 kernel).  wait_cycles > 0 replaces the default
 * bound (about 2 s of SM clock) of every wait in that kernel's later launches made by the
 * calling thread; unreachable != 0 raises its grid-barrier targets beyond reach, so that every
 * such wait runs out: the call still completes, each wait ends within its bound, nothing traps,
 * the workspace's error word gets COLI_DEVERR_TIMEOUT and the outputs are invalid.  (0, 0)
 * restores the defaults.  Host only; COLI_ERR_INVALID_ARG for a negative bound. */
coli_status coli_moe_debug_set_wait(long long wait_cycles, int unreachable);

/* Size of the static scratch array behind coli_moe_layer_noalloc (8 MiB per GPU). */
#define COLI_MOE_STATIC_SCRATCH_BYTES (8u << 20)

/* The whole layer, like coli_moe_layer, for callers that cannot allocate device memory: a
 * plugin inside a serving engine whose GPU memory pool is fixed when the engine starts, or a
 * real-time loop that must never pay for cudaMalloc's device-wide synchronisation.  The pages
 * have no counterpart of this call; it exists for such callers only.
 *   - Allocates nothing.  The caller passes x, out and the optional routing outputs as for
 *     coli_moe_layer; every other byte the layer needs lives in one static device array of
 *     COLI_MOE_STATIC_SCRATCH_BYTES that every GPU loading this library holds until exit.
 *   - The first call on each device looks up that array's device address (cudaGetSymbolAddress
 *     with the device current) and caches it; make that first call before any stream capture.
 *   - Returns COLI_ERR_WORKSPACE when the call needs more scratch than the array holds
 *     (coli_moe_workspace_size(cfg, T) > COLI_MOE_STATIC_SCRATCH_BYTES), before any launch.
 *   - All calls on a device share the one array and it keeps the last call's contents; each call
 *     clears the part that must start at zero.  Calls that overlap on the GPU (different streams
 *     without ordering between them) race on the array and give wrong results: order them.
 *   - The device error word lives inside the array: coli_moe_noalloc_error_word reads it.
 *     Device anomalies never trap. */
coli_status coli_moe_layer_noalloc(const coli_moe_config *cfg, const coli_moe_weights *w,
                                   const void *x, int T, float *out, int32_t *topk_ids_out,
                                   float *topk_w_out, void *stream);

/* Synchronises `stream` and returns in *code the device error word of the current device's
 * static scratch array (the one coli_moe_layer_noalloc uses): 0 = clean, else COLI_DEVERR_*
 * bits of the last coli_moe_layer_noalloc call on this device (each call clears it first).
 * code NULL: COLI_ERR_INVALID_ARG; COLI_ERR_CUDA if the array cannot be reached.  Like the first
 * coli_moe_layer_noalloc call, the first call on a device looks the array up (before any
 * stream capture). */
coli_status coli_moe_noalloc_error_word(void *stream, int *code);

#ifdef __cplusplus
}
#endif
#endif /* COLI_MOE_H */
