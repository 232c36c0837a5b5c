// router.cu -- a1 gate, a2 noaux_tc routing and a3 batch-union grouping on sm_100a.
//
// The router of the colibri-strix README ("What's implemented": a DeepSeek-V3 sigmoid router,
// noaux_tc bias, routed_scaling_factor) and the batch-union step of the same section.  The
// gate sums exact double products in double and rounds once to float32; selection compares in
// double, so the float32 logits and the chosen experts do not depend on summation order beyond
// double rounding.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace coli {

namespace {

constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

template <int ACT>
__device__ __forceinline__ void load_x4(const void *x, size_t idx, float v[4]) {
    if (ACT == COLI_ACT_F32) {
        float4 f = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + idx));
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
        uint2 u = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(x) + idx));
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xffff0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xffff0000u);
    }
}

// ---------------------------------------------------------------- a1 gate, few tokens ------
// One warp per expert row; every lane walks the row with float4 loads and keeps one double
// accumulator per token of the current token block.
template <int ACT, int TT>
__global__ void __launch_bounds__(128) gate_rows_kernel(const float *__restrict__ Wr,
                                                        const void *__restrict__ x, int T,
                                                        int H, int E,
                                                        float *__restrict__ logits) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 4 + warp;
    if (e >= E) return;
    const float *wrow = Wr + static_cast<size_t>(e) * H;
    for (int t0 = 0; t0 < T; t0 += TT) {
        double acc[TT];
#pragma unroll
        for (int i = 0; i < TT; ++i) acc[i] = 0.0;
        for (int h = lane * 4; h < H; h += 128) {
            const float4 wv = __ldg(reinterpret_cast<const float4 *>(wrow + h));
#pragma unroll
            for (int i = 0; i < TT; ++i) {
                if (t0 + i < T) {
                    float xv[4];
                    load_x4<ACT>(x, static_cast<size_t>(t0 + i) * H + h, xv);
                    acc[i] = fma(static_cast<double>(wv.x), static_cast<double>(xv[0]), acc[i]);
                    acc[i] = fma(static_cast<double>(wv.y), static_cast<double>(xv[1]), acc[i]);
                    acc[i] = fma(static_cast<double>(wv.z), static_cast<double>(xv[2]), acc[i]);
                    acc[i] = fma(static_cast<double>(wv.w), static_cast<double>(xv[3]), acc[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < TT; ++i) {
            double v = acc[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
            if (lane == 0 && t0 + i < T)
                logits[static_cast<size_t>(t0 + i) * E + e] = static_cast<float>(v);
        }
    }
}

// ---------------------------------------------------------------- a1 gate, many tokens -----
// logits[T,E] = X[T,H] * Wr[E,H]^T on the fp64 tensor cores (mma.sync m8n8k4, double operands
// and accumulators): every product of a bf16 or float32 activation and a float32 weight is exact
// in double and sums are double, as in the per-row kernel above; only the summation order
// differs.  A cluster of CL CTAs (2 or 4) computes one 64-token x 64-expert tile, each CTA one
// CL-th of H (4 warps of 32 x 32, K chunks of 32 staged in shared memory as double, the next
// chunk's global loads in flight during the current chunk); partial sums travel through
// distributed shared memory and are added pairwise in a fixed order: p0 + p1 (and p2 + p3,
// then (p0 + p1) + (p2 + p3)).  Measured on B200 (2048 tokens, 256 experts, H 6144): 32 x 32
// warp tiles 260 us against 271 us for 32 x 16; the m16n8k8 double shape, 303 us.
constexpr int GM = 64, GN = 64, GK = 32;
constexpr int GKP = GK + 4;  // row pitch (doubles): the 8 x 4 fragment reads hit each bank twice

__device__ __forceinline__ void dmma(double &d0, double &d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d0), "+d"(d1) : "d"(a), "d"(b));
}

template <int ACT, int CL>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(128)
gate_dmma_kernel(const float *__restrict__ Wr, const void *__restrict__ x, int T, int H, int E,
                 float *__restrict__ logits) {
    // staging tiles of x and Wr; after the main loop, the partial-sum exchange buffer
    __shared__ double sbuf[(GM + GN) * GKP];
    double (*xs)[GKP] = reinterpret_cast<double (*)[GKP]>(sbuf);
    double (*ws)[GKP] = reinterpret_cast<double (*)[GKP]>(sbuf + GM * GKP);
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int kr = static_cast<int>(cluster.block_rank());  // part kr of H
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.y * GM, e0 = (blockIdx.x / CL) * GN;
    const int kbeg = kr * (H / CL), kend = kbeg + H / CL;
    // staging: x row tid/2, k [16*(tid%2), +16); Wr row tid/2, k [16*(tid%2), +16)
    const int xr = tid >> 1, xk = 16 * (tid & 1);
    const int wr = tid >> 1, wk = 16 * (tid & 1);
    const bool xok = t0 + xr < T, wok = e0 + wr < E;
    float xv[16], wv[16];
    auto load = [&](int k0) {
        if (xok) {
            if (ACT == COLI_ACT_F32) {
                const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) +
                                                                   static_cast<size_t>(t0 + xr) * H + k0 + xk);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 f = __ldg(p + i);
                    xv[4 * i] = f.x; xv[4 * i + 1] = f.y; xv[4 * i + 2] = f.z; xv[4 * i + 3] = f.w;
                }
            } else {
                const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) +
                                                                 static_cast<size_t>(t0 + xr) * H + k0 + xk);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint4 u = __ldg(p + i);
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        xv[8 * i + 2 * j] = __uint_as_float(w4[j] << 16);
                        xv[8 * i + 2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) xv[i] = 0.f;
        }
        if (wok) {
            const float4 *p = reinterpret_cast<const float4 *>(Wr + static_cast<size_t>(e0 + wr) * H + k0 + wk);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 f = __ldg(p + i);
                wv[4 * i] = f.x; wv[4 * i + 1] = f.y; wv[4 * i + 2] = f.z; wv[4 * i + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) wv[i] = 0.f;
        }
    };
    const int wm = warp & 1, wn = warp >> 1;  // warp tile: tokens [32*wm, +32), experts [32*wn, +32)
    const int fr = lane >> 2, fk = lane & 3;  // fragment row (token / expert) and k of this lane
    constexpr int NJ = 4;                     // 8-expert fragments per warp
    double acc[4][NJ][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

    load(kbeg);
    for (int k0 = kbeg; k0 < kend; k0 += GK) {
        __syncthreads();  // the previous chunk's fragments have been read
#pragma unroll
        for (int i = 0; i < 16; ++i) xs[xr][xk + i] = static_cast<double>(xv[i]);
#pragma unroll
        for (int i = 0; i < 16; ++i) ws[wr][wk + i] = static_cast<double>(wv[i]);
        __syncthreads();
        if (k0 + GK < kend) load(k0 + GK);
#pragma unroll
        for (int k4 = 0; k4 < GK; k4 += 4) {
            double a[4], b[NJ];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[32 * wm + 8 * i + fr][k4 + fk];
#pragma unroll
            for (int j = 0; j < NJ; ++j) b[j] = ws[32 * wn + 8 * j + fr][k4 + fk];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < NJ; ++j) dmma(acc[i][j][0], acc[i][j][1], a[i], b[j]);
        }
    }
    // partial sums through the partner's shared memory (its staging buffer, free once every CTA
    // of the cluster is past the barrier before the copy); every CTA takes every barrier
    double *xch = sbuf;  // 8 NJ doubles per thread, element i of thread tid at [i * 128 + tid]
    static_assert(8 * NJ * 128 <= (GM + GN) * GKP, "exchange buffer");
    auto send = [&](int to) {
        double *dst = cluster.map_shared_rank(xch, to);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) dst[((i * NJ + j) * 2 + h) * 128 + tid] = acc[i][j][h];
    };
    auto take = [&]() {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) acc[i][j][h] = acc[i][j][h] + xch[((i * NJ + j) * 2 + h) * 128 + tid];
    };
    cluster.sync();
    if (kr & 1) send(kr - 1);  // p1 -> rank 0, p3 -> rank 2
    cluster.sync();
    if (!(kr & 1)) take();     // rank 0: p0 + p1; rank 2: p2 + p3
    if (CL == 4) {
        cluster.sync();        // rank 0 has read its buffer
        if (kr == 2) send(0);
        cluster.sync();
        if (kr == 0) take();   // (p0 + p1) + (p2 + p3)
    }
    if (kr != 0) return;
    // accumulator (i, j): token 32*wm + 8*i + fr, experts 32*wn + 8*j + 2*fk + {0, 1}
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + 32 * wm + 8 * i + fr;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e = e0 + 32 * wn + 8 * j + 2 * fk + h;
                if (e < E) logits[static_cast<size_t>(t) * E + e] = static_cast<float>(acc[i][j][h]);
            }
    }
}

// ---------------------------------------------------------------- a2 route -----------------
__device__ __forceinline__ bool beats(double va, int ia, double vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// Warp-wide arg-max of (value desc, index asc); every lane ends with the winner.
__device__ __forceinline__ void warp_argmax(double &v, int &i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(FULL, v, o);
        const int oi = __shfl_xor_sync(FULL, i, o);
        if (beats(ov, oi, v, i)) { v = ov; i = oi; }
    }
}

// One warp per token.  Lane l holds experts e = l + 32 v, v < VPL.
template <int VPL>
__global__ void __launch_bounds__(128) route_kernel(const float *__restrict__ logits,
                                                    const float *__restrict__ bias, int T,
                                                    int E, int K, int G, int TG, double rsf,
                                                    int32_t *__restrict__ ids,
                                                    float *__restrict__ wout) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const int gs = E / G;
    double s[VPL], c[VPL];
    bool taken[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int e = lane + 32 * v;
        taken[v] = false;
        if (e < E) {
            const double l = static_cast<double>(logits[static_cast<size_t>(t) * E + e]);
            s[v] = 1.0 / (1.0 + exp(-l));
            c[v] = s[v] + static_cast<double>(bias[e]);
        } else {
            s[v] = 0.0;
            c[v] = -INFINITY;
        }
    }
    // group stage: kept-group bit mask (G <= 32)
    uint32_t kept = (G >= 32) ? FULL : ((1u << G) - 1u);
    if (G > 1 && TG < G) {
        double my_score = -INFINITY;
        for (int g = 0; g < G; ++g) {
            double a1 = -INFINITY, a2 = -INFINITY;  // two largest values of this lane
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const int e = lane + 32 * v;
                if (e < E && e / gs == g) {
                    if (c[v] > a1) { a2 = a1; a1 = c[v]; }
                    else if (c[v] > a2) { a2 = c[v]; }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {  // merge pairs of sorted top-2 lists
                const double b1 = __shfl_xor_sync(FULL, a1, o);
                const double b2 = __shfl_xor_sync(FULL, a2, o);
                const double n1 = fmax(a1, b1);
                const double n2 = fmax(fmin(a1, b1), fmax(a2, b2));
                a1 = n1; a2 = n2;
            }
            if (lane == g) my_score = a1 + a2;
        }
        kept = 0u;
        for (int r = 0; r < TG; ++r) {
            double v = (lane < G && !((kept >> lane) & 1u)) ? my_score : -INFINITY;
            int i = (lane < G && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
            warp_argmax(v, i);
            kept |= 1u << i;
        }
    }
    // expert stage: K arg-max picks; lane k keeps the unbiased score of slot k
    double my_s = 0.0;
    int my_id = -1;
    for (int k = 0; k < K; ++k) {
        double bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            const int e = lane + 32 * v;
            if (e < E && !taken[v] && ((kept >> (e / gs)) & 1u) && beats(c[v], e, bv, bi)) {
                bv = c[v];
                bi = e;
            }
        }
        warp_argmax(bv, bi);
        double sv = 0.0;
#pragma unroll
        for (int v = 0; v < VPL; ++v)
            if (lane + 32 * v == bi) { taken[v] = true; sv = s[v]; }
        const int owner = bi & 31;
        sv = __shfl_sync(FULL, sv, owner);
        if (lane == k) { my_s = sv; my_id = bi; }
    }
    double denom = 0.0;
    for (int k = 0; k < K; ++k) denom += __shfl_sync(FULL, my_s, k);
    if (lane < K) {
        ids[static_cast<size_t>(t) * K + lane] = my_id;
        wout[static_cast<size_t>(t) * K + lane] = static_cast<float>((my_s / denom) * rsf);
    }
}

// ---------------------------------------------------------------- a3 group -----------------
// One CTA of 32 warps; warp w owns the contiguous slot range [w n / 32, (w + 1) n / 32).
// Pass 1: each warp counts its range per expert (32 slots at a time, peers by __match_any_sync;
// the leader of each id adds the peer count).  Pass 2: per expert, an exclusive scan over the
// warps and an exclusive scan of the expert totals give every (warp, expert) its first position.
// Pass 3: each warp places its slots in order (rank among the batch's peers plus its running
// cursor).  Stable: a warp's slots keep their order, and warp w's slots of an expert follow those
// of warps < w.  Only warp-level synchronisation inside the passes.
constexpr int GROUP_WARPS = 32;

__global__ void __launch_bounds__(GROUP_WARPS * 32) group_kernel(const int32_t *__restrict__ ids, int n,
                                                                 int E, int32_t *__restrict__ counts,
                                                                 int32_t *__restrict__ offsets,
                                                                 int32_t *__restrict__ perm,
                                                                 int32_t *__restrict__ unique,
                                                                 int32_t *__restrict__ n_unique,
                                                                 int *__restrict__ err) {
    extern __shared__ int sm[];
    int *wc = sm;                // [GROUP_WARPS][E]: counts, then first positions, then cursors
    int *tot = sm + GROUP_WARPS * E;  // [E]
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int s_lo = static_cast<int>(static_cast<long>(n) * warp / GROUP_WARPS);
    const int s_hi = static_cast<int>(static_cast<long>(n) * (warp + 1) / GROUP_WARPS);
    if (tid == 0) bad = 0;
    for (int i = tid; i < GROUP_WARPS * E; i += blockDim.x) wc[i] = 0;
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    int *mine = wc + warp * E;
    for (int base = s_lo; base < s_hi; base += 32) {
        const int s = base + lane;
        const int id = s < s_hi ? ids[s] : -1;
        const bool ok = id >= 0 && id < E;
        if (s < s_hi && !ok) bad = 1;
        const unsigned peers = __match_any_sync(FULL, ok ? id : -1 - lane);
        if (ok && (peers & lt) == 0) mine[id] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {  // exclusive scan over the warps, per expert
        int run = 0;
        for (int w = 0; w < GROUP_WARPS; ++w) {
            const int c = wc[w * E + e];
            wc[w * E + e] = run;
            run += c;
        }
        tot[e] = run;
    }
    __syncthreads();
    // exclusive scans of the totals and of the non-empty flags, by warp 0 (E <= 1024)
    if (warp == 0) {
        const int per = (E + 31) / 32;
        const int b = lane * per;
        int sc = 0, su = 0;
        for (int e = b; e < b + per && e < E; ++e) { sc += tot[e]; su += tot[e] > 0; }
        int ic = sc, iu = su;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(FULL, ic, o), bb = __shfl_up_sync(FULL, iu, o);
            if (lane >= o) { ic += a; iu += bb; }
        }
        int rc = ic - sc, ru = iu - su;
        for (int e = b; e < b + per && e < E; ++e) {
            offsets[e] = rc;
            counts[e] = tot[e];
            if (tot[e] > 0) unique[ru++] = e;
            const int c = tot[e];
            tot[e] = rc;  // first position of expert e
            rc += c;
        }
        if (lane == 31) {
            offsets[E] = ic;
            *n_unique = iu;
            for (int e = iu; e < E; ++e) unique[e] = -1;
        }
    }
    __syncthreads();
    for (int i = tid; i < GROUP_WARPS * E; i += blockDim.x) wc[i] += tot[i % E];
    __syncthreads();
    for (int base = s_lo; base < s_hi; base += 32) {
        const int s = base + lane;
        const int id = s < s_hi ? ids[s] : -1;
        const bool ok = id >= 0 && id < E;
        const unsigned peers = __match_any_sync(FULL, ok ? id : -1 - lane);
        if (ok) perm[mine[id] + __popc(peers & lt)] = s;
        __syncwarp();
        if (ok && (peers & lt) == 0) mine[id] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // slots with a bad id are not placed; the tail of perm is marked
    if (tid == 0 && bad) {
        atomicOr(err, COLI_DEVERR_EXPERT_ID);
        for (int p = offsets[E]; p < n; ++p) perm[p] = -1;
    }
}

}  // namespace

cudaError_t launch_gate(const coli_moe_config &c, const float *Wr, const void *x, int T,
                        float *logits, cudaStream_t st) {
    const int H = c.hidden, E = c.n_experts;
    if (T <= 16) {
        dim3 grid((E + 3) / 4);
        if (c.act == COLI_ACT_F32)
            gate_rows_kernel<COLI_ACT_F32, 8><<<grid, 128, 0, st>>>(Wr, x, T, H, E, logits);
        else
            gate_rows_kernel<COLI_ACT_BF16, 8><<<grid, 128, 0, st>>>(Wr, x, T, H, E, logits);
    } else {
        // clusters of CL CTAs along x, each CTA a CL-th of H (a whole number of 32-wide chunks)
        const int cl = H % (4 * GK) == 0 ? 4 : 2;
        dim3 grid(cl * ((E + GN - 1) / GN), (T + GM - 1) / GM);
        if (cl == 4) {
            if (c.act == COLI_ACT_F32)
                gate_dmma_kernel<COLI_ACT_F32, 4><<<grid, 128, 0, st>>>(Wr, x, T, H, E, logits);
            else
                gate_dmma_kernel<COLI_ACT_BF16, 4><<<grid, 128, 0, st>>>(Wr, x, T, H, E, logits);
        } else {
            if (c.act == COLI_ACT_F32)
                gate_dmma_kernel<COLI_ACT_F32, 2><<<grid, 128, 0, st>>>(Wr, x, T, H, E, logits);
            else
                gate_dmma_kernel<COLI_ACT_BF16, 2><<<grid, 128, 0, st>>>(Wr, x, T, H, E, logits);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_route(const coli_moe_config &c, const float *logits, const float *bias,
                         int T, int32_t *ids, float *w, cudaStream_t st) {
    const int E = c.n_experts;
    dim3 grid((T + 3) / 4);
    const int vpl = (E + 31) / 32;
#define COLI_ROUTE(V)                                                                        \
    route_kernel<V><<<grid, 128, 0, st>>>(logits, bias, T, E, c.top_k, c.n_group,            \
                                          c.topk_group, c.routed_scaling, ids, w)
    if (vpl <= 1) COLI_ROUTE(1);
    else if (vpl <= 2) COLI_ROUTE(2);
    else if (vpl <= 4) COLI_ROUTE(4);
    else if (vpl <= 8) COLI_ROUTE(8);
    else if (vpl <= 16) COLI_ROUTE(16);
    else COLI_ROUTE(32);
#undef COLI_ROUTE
    return cudaGetLastError();
}

cudaError_t launch_group(const coli_moe_config &c, const int32_t *ids, int T, int32_t *counts,
                         int32_t *offsets, int32_t *perm, int32_t *unique, int32_t *n_unique,
                         int *err, cudaStream_t st) {
    const int n = T * c.top_k, E = c.n_experts;
    const size_t smem = static_cast<size_t>(GROUP_WARPS + 1) * E * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    group_kernel<<<1, GROUP_WARPS * 32, smem, st>>>(ids, n, E, counts, offsets, perm, unique, n_unique, err);
    return cudaGetLastError();
}

}  // namespace coli
