// coli_moe.cu -- the C ABI of libcoli_moe.so: argument validation, workspace carve-up, and the
// launch sequence of the layer.  No device memory is allocated here; no CPU fallback exists.
#include <atomic>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "coli_moe.h"
#include "internal.h"
#include "residual.h"

namespace coli {

namespace {

inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

inline bool aligned(const void *p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

thread_local char g_last_cuda_error[256] = "";
// testing aid (coli_moe_debug_set_wait): the fused decode kernel's wait bound and a flag that
// makes its grid-barrier targets unreachable
thread_local long long g_wait_cycles = 0;
thread_local int g_unreachable = 0;
// a5' per-expert dispatch on the grouped-GEMM path: work experts with at most this many tokens
// take the GEMV kernels (coli_moe_set_dispatch_threshold; 0 = every expert on the tensor cores)
std::atomic<int> g_dispatch{DISPATCH_DEFAULT};

coli_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return COLI_OK;
    record_cuda_error(e);
    return COLI_ERR_CUDA;
}

int row_bytes(int n, int fmt) { return n * fmt / 8; }

}  // namespace

// Batches beyond decode size take the tensor-core grouped GEMM when its shape rules hold.
static bool use_tc(const coli_moe_config *c, int T) { return T > TC_MIN_TOKENS && tc_shape_ok(*c); }

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

size_t device_smem_optin() {
    static size_t cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 227 * 1024;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || n <= 0)
            n = 227 * 1024;
        cached[dev] = static_cast<size_t>(n);
    }
    return cached[dev];
}

void record_cuda_error(cudaError_t e) {
    snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
}

WsLayout ws_layout(const coli_moe_config &c, int T) {
    WsLayout L;
    const size_t n = static_cast<size_t>(T) * c.top_k;
    const size_t E = static_cast<size_t>(c.n_experts);
    size_t o = 0;
    L.err = o;      o = align256(o + WS_HEADER);
    L.dsl = o;      o = align256(o + WS_DSL_BYTES);
    L.logits = o;   o = align256(o + static_cast<size_t>(T) * E * 4);
    L.ids = o;      o = align256(o + n * 4);
    L.w = o;        o = align256(o + n * 4);
    L.counts = o;   o = align256(o + E * 4);
    L.offsets = o;  o = align256(o + (E + 1) * 4);
    L.perm = o;     o = align256(o + n * 4);
    L.unique = o;   o = align256(o + E * 4);
    L.nuniq = o;    o = align256(o + 4);
    const size_t slots = n + static_cast<size_t>(T) * c.n_shared;
    L.h = o;        o = align256(o + slots * c.inter * 4);
    const bool tc = use_tc(&c, T);
    const size_t H = static_cast<size_t>(c.hidden), I = static_cast<size_t>(c.inter);
    L.xq = o;       o = align256(o + (tc ? 2 * slots * H : 0));
    L.hq = o;       o = align256(o + (tc ? 2 * slots * I : 0));
    L.sx = o;       o = align256(o + (tc ? slots * 4 : 0));
    L.sh = o;       o = align256(o + (tc ? slots * 4 : 0));
    L.tok_of = o;   o = align256(o + (tc ? slots * 4 : 0));
    L.w_of = o;     o = align256(o + (tc ? slots * 4 : 0));
    L.chunks = o;   o = align256(o + (tc ? static_cast<size_t>(tc_max_chunks(c, T)) * 16 : 0));
    L.n_chunks = o; o = align256(o + (tc ? 4 : 0));
    L.total = o;
    return L;
}

}  // namespace coli

using namespace coli;

extern "C" {

const char *coli_moe_status_str(coli_status s) {
    switch (s) {
        case COLI_OK: return "ok";
        case COLI_ERR_INVALID_ARG: return "invalid argument";
        case COLI_ERR_SHAPE: return "inconsistent shape";
        case COLI_ERR_ALIGN: return "misaligned pointer or stride";
        case COLI_ERR_UNSUPPORTED: return "unsupported configuration";
        case COLI_ERR_CUDA: return "CUDA runtime error";
        case COLI_ERR_DEVICE: return "device error word set";
        case COLI_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    }
    return "unknown status";
}

const char *coli_moe_last_cuda_error(void) { return g_last_cuda_error; }

coli_status coli_moe_set_dispatch_threshold(int max_tokens) {
    if (max_tokens < 0 || max_tokens > 65536) return COLI_ERR_INVALID_ARG;
    g_dispatch.store(max_tokens);
    return COLI_OK;
}

int coli_moe_dispatch_threshold(void) { return g_dispatch.load(); }

coli_status coli_moe_debug_set_wait(long long wait_cycles, int unreachable) {
    if (wait_cycles < 0) return COLI_ERR_INVALID_ARG;
    g_wait_cycles = wait_cycles;
    g_unreachable = unreachable != 0;
    return COLI_OK;
}

coli_status coli_moe_record_bytes(int hidden, int inter, int wfmt, int group_size, size_t *bytes) {
    if (!bytes) return COLI_ERR_INVALID_ARG;
    if (wfmt != COLI_W_INT4 && wfmt != COLI_W_INT8 && wfmt != COLI_W_INT2) return COLI_ERR_INVALID_ARG;
    if (group_size != 0 && group_size != 64) return COLI_ERR_INVALID_ARG;
    if (group_size && wfmt != COLI_W_INT4) return COLI_ERR_UNSUPPORTED;
    if (hidden <= 0 || inter <= 0) return COLI_ERR_SHAPE;
    if ((static_cast<long>(hidden) * wfmt) % 8 || (static_cast<long>(inter) * wfmt) % 8) return COLI_ERR_SHAPE;
    if (group_size && (hidden % group_size || inter % group_size)) return COLI_ERR_SHAPE;
    const size_t rh = static_cast<size_t>(hidden) * wfmt / 8, ri = static_cast<size_t>(inter) * wfmt / 8;
    const size_t nh = group_size ? hidden / group_size : 1, ni = group_size ? inter / group_size : 1;
    *bytes = 2 * static_cast<size_t>(inter) * rh + static_cast<size_t>(hidden) * ri +
             (2 * static_cast<size_t>(inter) * nh + static_cast<size_t>(hidden) * ni) * sizeof(float);
    return COLI_OK;
}

coli_status coli_moe_check_config(const coli_moe_config *c) {
    if (!c) return COLI_ERR_INVALID_ARG;
    if (c->wfmt != COLI_W_INT4 && c->wfmt != COLI_W_INT8 && c->wfmt != COLI_W_INT2) return COLI_ERR_INVALID_ARG;
    if (c->act != COLI_ACT_F32 && c->act != COLI_ACT_BF16) return COLI_ERR_INVALID_ARG;
    if (c->group_size != 0 && c->group_size != 64) return COLI_ERR_INVALID_ARG;
    if (c->group_size && c->wfmt != COLI_W_INT4) return COLI_ERR_UNSUPPORTED;
    if (c->hidden <= 0 || c->inter <= 0 || c->n_experts <= 0 || c->top_k <= 0 || c->n_group <= 0 ||
        c->topk_group <= 0 || c->n_shared < 0)
        return COLI_ERR_SHAPE;
    if (!(c->routed_scaling > 0.0)) return COLI_ERR_INVALID_ARG;
    if (c->n_experts % c->n_group) return COLI_ERR_SHAPE;
    if (c->topk_group > c->n_group) return COLI_ERR_SHAPE;
    const int gs = c->n_experts / c->n_group;
    if (c->n_group > 1 && c->topk_group < c->n_group && gs < 2) return COLI_ERR_SHAPE;
    if (c->top_k > c->topk_group * gs) return COLI_ERR_SHAPE;
    if (c->n_experts > 1024 || c->top_k > 32 || c->n_group > 32) return COLI_ERR_UNSUPPORTED;
    if (c->n_shared > 1) return COLI_ERR_UNSUPPORTED;
    if (c->n_shared == 1 && c->shared_inter != c->inter) return COLI_ERR_UNSUPPORTED;
    if (c->hidden % 64 || c->inter % 64) return COLI_ERR_SHAPE;
    if (!gemv_shape_ok(row_bytes(c->hidden, c->wfmt)) || !gemv_shape_ok(row_bytes(c->inter, c->wfmt)))
        return COLI_ERR_UNSUPPORTED;
    return COLI_OK;
}

coli_status coli_moe_workspace_size(const coli_moe_config *c, int max_tokens, size_t *bytes) {
    if (!bytes) return COLI_ERR_INVALID_ARG;
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (max_tokens < 0) return COLI_ERR_SHAPE;
    *bytes = ws_layout(*c, max_tokens > 0 ? max_tokens : 1).total;
    return COLI_OK;
}

coli_status coli_moe_clear_error(void *ws, void *stream) {
    if (!ws || !aligned(ws, 256)) return COLI_ERR_WORKSPACE;
    return from_cuda(cudaMemsetAsync(ws, 0, WS_HEADER, static_cast<cudaStream_t>(stream)));
}

coli_status coli_moe_error_word(void *ws, void *stream, int *code) {
    if (!ws || !code || !aligned(ws, 256)) return COLI_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return COLI_ERR_CUDA;
    *code = v;
    return COLI_OK;
}

coli_status coli_moe_layer_kernels(const coli_moe_config *c, int T, int *n_kernels) {
    if (!n_kernels) return COLI_ERR_INVALID_ARG;
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    DecodePlan pl;
    *n_kernels = T == 0 ? 0 : (decode_plan(*c, T, &pl) ? 1 : (use_tc(c, T) ? (g_dispatch.load() > 0 ? 9 : 7) : 5));
    return COLI_OK;
}

coli_status coli_moe_gate(const coli_moe_config *c, const float *router_w, const void *x, int T,
                          float *logits, void *stream) {
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    if (!router_w || !x || !logits) return COLI_ERR_INVALID_ARG;
    if (!aligned(router_w, 16) || !aligned(x, 16) || !aligned(logits, 4)) return COLI_ERR_ALIGN;
    return from_cuda(launch_gate(*c, router_w, x, T, logits, static_cast<cudaStream_t>(stream)));
}

coli_status coli_moe_residual(const coli_moe_config *c, const void *x, const float *out, int T,
                              void *x_next, void *stream) {
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    if (!x || !out || !x_next) return COLI_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(x_next, 16)) return COLI_ERR_ALIGN;
    return from_cuda(launch_residual(*c, x, out, T, x_next, static_cast<cudaStream_t>(stream)));
}

coli_status coli_moe_route(const coli_moe_config *c, const float *logits, const float *bias, int T,
                           int32_t *topk_ids, float *topk_w, void *stream) {
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    if (!logits || !bias || !topk_ids || !topk_w) return COLI_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(bias, 4) || !aligned(topk_ids, 4) || !aligned(topk_w, 4))
        return COLI_ERR_ALIGN;
    return from_cuda(launch_route(*c, logits, bias, T, topk_ids, topk_w, static_cast<cudaStream_t>(stream)));
}

coli_status coli_moe_group(const coli_moe_config *c, const int32_t *topk_ids, int T, int32_t *counts,
                           int32_t *offsets, int32_t *perm, int32_t *unique_ids, int32_t *n_unique,
                           void *ws, size_t ws_bytes, void *stream) {
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    if (!ws || !aligned(ws, 256) || ws_bytes < 256) return COLI_ERR_WORKSPACE;
    if (!counts || !offsets || !unique_ids || !n_unique) return COLI_ERR_INVALID_ARG;
    if (T > 0 && (!topk_ids || !perm)) return COLI_ERR_INVALID_ARG;
    if (static_cast<long>(T) * c->top_k > (1L << 30)) return COLI_ERR_SHAPE;
    return from_cuda(launch_group(*c, topk_ids, T, counts, offsets, perm, unique_ids, n_unique,
                                  static_cast<int *>(ws), static_cast<cudaStream_t>(stream)));
}

static coli_status check_weights(const coli_moe_config *c, const coli_moe_weights *w, bool need_router) {
    if (!w) return COLI_ERR_INVALID_ARG;
    if (!w->experts) return COLI_ERR_INVALID_ARG;
    if (need_router && (!w->router_w || !w->router_bias)) return COLI_ERR_INVALID_ARG;
    if (c->n_shared == 1 && !w->shared) return COLI_ERR_INVALID_ARG;
    size_t rb = 0;
    coli_status s = coli_moe_record_bytes(c->hidden, c->inter, c->wfmt, c->group_size, &rb);
    if (s != COLI_OK) return s;
    if (w->expert_stride < rb) return COLI_ERR_SHAPE;
    if (w->expert_stride % 256 || !aligned(w->experts, 256)) return COLI_ERR_ALIGN;
    if (w->shared && !aligned(w->shared, 256)) return COLI_ERR_ALIGN;
    if (need_router && (!aligned(w->router_w, 16) || !aligned(w->router_bias, 4))) return COLI_ERR_ALIGN;
    return COLI_OK;
}

static FfnParams make_params(const coli_moe_config *c, const coli_moe_weights *w, const void *x, int T,
                             const float *topk_w, const int32_t *offsets, const int32_t *perm,
                             const int32_t *unique, const int32_t *n_unique, float *out, float *h,
                             int *err) {
    FfnParams p;
    p.H = c->hidden; p.I = c->inter; p.E = c->n_experts; p.K = c->top_k; p.T = T; p.S = c->n_shared;
    p.fmt = c->wfmt; p.act = c->act;
    p.experts = w->experts; p.stride = w->expert_stride; p.shared = w->shared;
    p.rb_h = static_cast<size_t>(c->hidden) * c->wfmt / 8;
    p.rb_i = static_cast<size_t>(c->inter) * c->wfmt / 8;
    p.off_wu = static_cast<size_t>(c->inter) * p.rb_h;
    p.off_wd = 2 * p.off_wu;
    p.group = c->group_size;
    p.nsh = c->group_size ? c->hidden / c->group_size : 1;  // scales per Wg / Wu row
    p.nsi = c->group_size ? c->inter / c->group_size : 1;   // scales per Wd row
    p.off_sg = p.off_wd + static_cast<size_t>(c->hidden) * p.rb_i;
    p.off_su = p.off_sg + static_cast<size_t>(c->inter) * p.nsh * 4;
    p.off_sd = p.off_su + static_cast<size_t>(c->inter) * p.nsh * 4;
    p.x = x; p.topk_w = topk_w; p.offsets = offsets; p.perm = perm; p.unique = unique;
    p.n_unique = n_unique; p.h = h; p.out = out; p.err = err;
    p.gemv_nmax = 0x7fffffff; p.tc_nmin = 0; p.gemv_atomic = 0;  // one path takes every expert
    return p;
}

static DecodeParams make_decode(const coli_moe_config *c, const FfnParams &f, char *base) {
    DecodeParams d = {};
    d.f = f;
    d.rsf = c->routed_scaling;
    d.G = c->n_group;
    d.TG = c->topk_group;
    d.phase = reinterpret_cast<unsigned *>(base + WS_PHASE);
    d.gbar = reinterpret_cast<unsigned *>(base + WS_GBAR);
    d.ready = reinterpret_cast<unsigned *>(base + WS_READY);
    const WsLayout L = ws_layout(*c, f.T);
    d.dsl = reinterpret_cast<uint4 *>(base + L.dsl);
    d.wait_cycles = g_wait_cycles;
    d.gate_extra = g_unreachable ? 1000000u : 0u;
    return d;
}

// The expert half for a given routing: the fused decode kernel when the shape allows it, else
// the general GEMV kernels.
static coli_status run_ffn(const coli_moe_config *c, const FfnParams &p, char *base, cudaStream_t st) {
    if (use_tc(c, p.T)) {
        const WsLayout L = ws_layout(*c, p.T);
        TcBuffers b;
        b.xq = reinterpret_cast<int8_t *>(base + L.xq);
        b.hq = reinterpret_cast<int8_t *>(base + L.hq);
        b.sx = reinterpret_cast<float *>(base + L.sx);
        b.sh = reinterpret_cast<float *>(base + L.sh);
        b.tok_of = reinterpret_cast<int *>(base + L.tok_of);
        b.w_of = reinterpret_cast<float *>(base + L.w_of);
        b.hbuf = reinterpret_cast<float *>(base + L.h);
        b.chunks = reinterpret_cast<int4 *>(base + L.chunks);
        b.n_chunks = reinterpret_cast<int *>(base + L.n_chunks);
        b.max_chunks = tc_max_chunks(*c, p.T);
        FfnParams q = p;  // per-expert dispatch between the GEMV kernels and the grouped GEMM
        const int n = g_dispatch.load();
        q.gemv_nmax = n;
        q.tc_nmin = n;
        q.gemv_atomic = 1;
        return from_cuda(launch_ffn_tc(q, b, st));
    }
    DecodePlan pl;
    if (decode_plan(*c, p.T, &pl)) return from_cuda(launch_ffn_decode(make_decode(c, p, base), pl, st));
    return from_cuda(launch_ffn_gemv(p, st));
}

coli_status coli_moe_ffn(const coli_moe_config *c, const coli_moe_weights *w, const void *x, int T,
                         const float *topk_w, const int32_t *offsets, const int32_t *perm,
                         const int32_t *unique_ids, const int32_t *n_unique, float *out, void *ws,
                         size_t ws_bytes, void *stream) {
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    s = check_weights(c, w, false);
    if (s != COLI_OK) return s;
    if (!x || !topk_w || !offsets || !perm || !unique_ids || !n_unique || !out) return COLI_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16)) return COLI_ERR_ALIGN;
    if (T > gemv_max_tokens(*c) && !use_tc(c, T)) return COLI_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(*c, T);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return COLI_ERR_WORKSPACE;
    char *base = static_cast<char *>(ws);
    FfnParams p = make_params(c, w, x, T, topk_w, offsets, perm, unique_ids, n_unique, out,
                              reinterpret_cast<float *>(base + L.h), reinterpret_cast<int *>(base + L.err));
    return run_ffn(c, p, base, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// Every host-side check of coli_moe_layer except the workspace's (T >= 1).
coli_status coli::layer_args_status(const coli_moe_config *c, const coli_moe_weights *w, const void *x,
                                    int T, const float *out, const int32_t *topk_ids_out,
                                    const float *topk_w_out) {
    coli_status s = check_weights(c, w, true);
    if (s != COLI_OK) return s;
    if (!x || !out) return COLI_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16)) return COLI_ERR_ALIGN;
    if ((topk_ids_out && !aligned(topk_ids_out, 4)) || (topk_w_out && !aligned(topk_w_out, 4)))
        return COLI_ERR_ALIGN;
    if (T > gemv_max_tokens(*c) && !use_tc(c, T)) return COLI_ERR_UNSUPPORTED;
    return COLI_OK;
}

extern "C" {

coli_status coli_moe_layer(const coli_moe_config *c, const coli_moe_weights *w, const void *x, int T,
                           float *out, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                           size_t ws_bytes, void *stream) {
    coli_status s = coli_moe_check_config(c);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    s = layer_args_status(c, w, x, T, out, topk_ids_out, topk_w_out);
    if (s != COLI_OK) return s;
    const WsLayout L = ws_layout(*c, T);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return COLI_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *base = static_cast<char *>(ws);
    float *logits = reinterpret_cast<float *>(base + L.logits);
    int32_t *ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t *>(base + L.ids);
    float *wts = topk_w_out ? topk_w_out : reinterpret_cast<float *>(base + L.w);
    int32_t *counts = reinterpret_cast<int32_t *>(base + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(base + L.offsets);
    int32_t *perm = reinterpret_cast<int32_t *>(base + L.perm);
    int32_t *uniq = reinterpret_cast<int32_t *>(base + L.unique);
    int32_t *nu = reinterpret_cast<int32_t *>(base + L.nuniq);
    int *err = reinterpret_cast<int *>(base + L.err);

    FfnParams p = make_params(c, w, x, T, wts, offsets, perm, uniq, nu, out,
                              reinterpret_cast<float *>(base + L.h), err);
    DecodePlan pl;
    if (decode_plan(*c, T, &pl)) {
        // fused decode path: one persistent kernel (gate, route, group, FFN, combine)
        DecodeParams d = make_decode(c, p, base);
        d.Wr = w->router_w;
        d.bias = w->router_bias;
        d.logits = logits;
        d.ids = ids;
        d.wts = wts;
        d.f_counts = counts;
        d.f_offsets = offsets;
        d.f_perm = perm;
        d.f_unique = uniq;
        d.f_nuniq = nu;
        d.route_here = 1;
        return from_cuda(launch_ffn_decode(d, pl, st));
    }
    cudaError_t e = launch_gate(*c, w->router_w, x, T, logits, st);
    if (e == cudaSuccess) e = launch_route(*c, logits, w->router_bias, T, ids, wts, st);
    if (e == cudaSuccess) e = launch_group(*c, ids, T, counts, offsets, perm, uniq, nu, err, st);
    if (e != cudaSuccess) return from_cuda(e);
    return run_ffn(c, p, base, st);
}

}  // extern "C"
