// internal.h -- declarations shared by the translation units of libcoli_moe.so (not installed).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "coli_moe.h"

namespace coli {

// Parameters of the expert half of the layer (a4..a7), shared by the GEMV and MMA kernels.
struct FfnParams {
    int H, I, E, K, T, S;              // S = n_shared (0 or 1); shared inter == I
    int fmt;                           // 4, 8, 2
    int act;                           // coli_act of x
    int group;                         // 0: per-row scales; 64: per 64 columns of a row
    int nsh, nsi;                      // scales per gate/up row and per down row
    const uint8_t *experts;            // E records
    size_t stride;                     // record stride, bytes
    const uint8_t *shared;             // shared record or nullptr
    size_t off_wu, off_wd, off_sg, off_su, off_sd;  // byte offsets inside a record
    size_t rb_h, rb_i;                 // bytes of a row of length H / of length I
    const void *x;                     // [T][H] f32 or bf16
    const float *topk_w;               // [T*K]
    const int32_t *offsets;            // [E+1]
    const int32_t *perm;               // [T*K]
    const int32_t *unique;             // [E]
    const int32_t *n_unique;           // [1]
    float *h;                          // [(T*K + T*S)][I] f32 intermediate (GEMV path)
    float *out;                        // [T][H]
    int *err;                          // device error word
    // per-expert dispatch (a5'): the GEMV kernels take the work experts with at most gemv_nmax
    // tokens, the grouped GEMM those with more than tc_nmin; gemv_atomic: the GEMV down kernel
    // adds into out (zeroed before) instead of writing it
    int gemv_nmax, tc_nmin, gemv_atomic;
};

// Workspace header (first 512 bytes): error word; then the fused decode path's phase word and
// two sets of counters (per set: the arrival count of the logits and the grid barrier at
// WS_GBAR + 32 * set, the converted h chunks per work expert at WS_READY + 160 * set).  A call
// uses the set the phase names; once every CTA has read the phase it zeroes the other set and
// flips the phase.  All must be zero before the first call on a workspace
// (coli_moe_clear_error zeroes them).
constexpr int WS_ERR = 0, WS_PHASE = 32, WS_GBAR = 64, WS_READY = 128;
constexpr int WS_HEADER = 512;
// Fused decode path: h of every (work expert, chunk of the down rows' K) converted once, as the
// chunk's MMA B block (one column per token and slice, at most 12 columns of at most 256
// bytes) followed by the tokens' 4 scales: [33 work experts][16 chunks] of 12 * 256 + 16 bytes.
constexpr int DEC_WE = 33, DEC_CH = 16;
constexpr size_t WS_DSL_BYTES = static_cast<size_t>(DEC_WE) * DEC_CH * (12 * 256 + 16);

// Shared-memory plan of the fused decode kernel (decode.cu).
struct DecodePlan {
    int grid, S, SB, st_sd;                           // ring: S stages of SB bytes
    size_t off_route, off_rtok, off_gate, off_red1, off_x, off_frag, off_ring, smem;
    int lag;                                          // down-projection lag (experts)
    int fslot;                                        // bytes of a down stage's fragment slot
};

// Parameters of the fused decode kernel.
struct DecodeParams {
    FfnParams f;
    // gate + route + group
    const float *Wr, *bias;
    float *logits;
    int32_t *ids;
    float *wts;
    int32_t *f_counts, *f_offsets, *f_perm, *f_unique, *f_nuniq;
    double rsf;
    int G, TG;
    unsigned *phase;        // which counter set this call uses
    unsigned *gbar;         // [2 sets, 8 words apart]: logits and grid-barrier arrivals
    unsigned *ready;        // [2 sets, 40 words apart][33]: converted h chunks per work expert
    uint4 *dsl;             // h chunks converted once (WS_DSL_BYTES)
    int route_here;         // 1: the kernel routes from its own logits; 0: routing arrays are inputs
    long long wait_cycles;  // bound of every device-side wait (0: the default, ~2 s)
    unsigned gate_extra;    // added to the logits-arrival target (nonzero only to test the bound)
    // plan (copied from DecodePlan)
    int grid, S, SB, st_sd, lag, fslot;
    size_t off_route, off_rtok, off_gate, off_red1, off_x, off_frag, off_ring;
};

bool decode_plan(const coli_moe_config &c, int T, DecodePlan *plan);
// the GEMV kernels one at a time (the grouped-GEMM path runs them for its small experts)
cudaError_t launch_ffn_gemv_gateup(const FfnParams &p, cudaStream_t st);
cudaError_t launch_ffn_gemv_down(const FfnParams &p, cudaStream_t st);
cudaError_t launch_ffn_decode(DecodeParams p, const DecodePlan &pl, cudaStream_t st);

// Buffers of the tensor-core grouped-GEMM path (ffn_tc.cu), carved from the workspace.
struct TcBuffers {
    int8_t *xq;          // [2*slots][H]: x of each slot's token as 16-bit fixed point, hi/lo rows
    int8_t *hq;          // [2*slots][I]: h of each slot, same encoding
    float *sx, *sh;      // [slots]: row scales of xq, hq
    int *tok_of;         // [slots]: token of the slot
    float *w_of;         // [slots]: combine weight of the slot
    float *hbuf;         // [slots][I]: h in float32
    int4 *chunks;        // chunk table
    int *n_chunks;
    int max_chunks;
};

int tc_max_chunks(const coli_moe_config &c, int T);
bool tc_shape_ok(const coli_moe_config &c);
cudaError_t launch_ffn_tc(const FfnParams &f, const TcBuffers &b, cudaStream_t st);

// Batches above this many tokens take the tensor-core path when its shape rules hold (measured
// on B200: from 8 tokens up it beats the CUDA-core GEMV path 3-13x on GLM- and OLMoE-shaped
// layers; up to 4 tokens the fused decode kernel runs).
constexpr int TC_MIN_TOKENS = 4;
// Default of the per-expert dispatch threshold on that path (work experts with at most this many
// tokens take the GEMV kernels), chosen by measurement on B200: on the 2048-token Zipf layer
// (194 unique experts, 23 of them with one token) thresholds 0/1/2/4/8/16 took 2.06/2.51/2.80/
// 3.46/4.67/8.80 ms; on the 512-token 64-expert Zipf layer 0.58/0.66/0.69/0.78/1.06/2.01 ms.
// A one-token expert costs about as much on the tensor cores as streaming its codes through the
// GEMV kernels, which also walk the whole expert list: every expert stays on the tensor cores.
constexpr int DISPATCH_DEFAULT = 0;

// Workspace carve-up (all offsets 256-B aligned).
struct WsLayout {
    size_t err;      // int error word (+ pad)
    size_t logits;   // [T][E] f32
    size_t ids;      // [T*K] i32
    size_t w;        // [T*K] f32
    size_t counts;   // [E] i32
    size_t offsets;  // [E+1] i32
    size_t perm;     // [T*K] i32
    size_t unique;   // [E] i32
    size_t nuniq;    // [1] i32
    size_t dsl;      // fused decode path: h chunks converted once (WS_DSL_BYTES)
    size_t h;        // [(T*K+T*S)][I] f32 intermediate
    // tensor-core path only (zero size otherwise)
    size_t xq, hq, sx, sh, tok_of, w_of, chunks, n_chunks;
    size_t total;
};

WsLayout ws_layout(const coli_moe_config &c, int T);

// Launchers (return cudaGetLastError()).
cudaError_t launch_gate(const coli_moe_config &c, const float *Wr, const void *x, int T,
                        float *logits, cudaStream_t st);
cudaError_t launch_route(const coli_moe_config &c, const float *logits, const float *bias,
                         int T, int32_t *ids, float *w, cudaStream_t st);
cudaError_t launch_group(const coli_moe_config &c, const int32_t *ids, int T, int32_t *counts,
                         int32_t *offsets, int32_t *perm, int32_t *unique, int32_t *n_unique,
                         int *err, cudaStream_t st);
cudaError_t launch_ffn_gemv(const FfnParams &p, cudaStream_t st);

// Shape rules of the GEMV path (checked on the host before launch).
bool gemv_shape_ok(int row_bytes);
int gemv_max_tokens(const coli_moe_config &c);

// Host-side checks of a whole-layer call other than the workspace's (weights, pointers,
// alignment, token count); T >= 1.  No launch.
coli_status layer_args_status(const coli_moe_config *c, const coli_moe_weights *w, const void *x,
                              int T, const float *out, const int32_t *topk_ids_out,
                              const float *topk_w_out);

int device_sm_count();
size_t device_smem_optin();  // max dynamic shared memory per block (opt-in)
void record_cuda_error(cudaError_t e);

}  // namespace coli
