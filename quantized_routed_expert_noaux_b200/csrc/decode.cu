// decode.cu -- the fused decode path of the layer for a few tokens (decode and MTP verify).
//
// Two launches, the second one programmatically dependent on the first:
//
//  K1 router_decode_kernel  a1 gate on grid (E/2, T): two Wr rows per CTA, products and sums in
//                           double.  The last CTA to finish a token routes it (a2, noaux_tc,
//                           colibri-strix README "What's implemented"), the last token router
//                           groups the batch (a3, batch-union).  No CTA ever waits on another:
//                           "last arrival" is decided by an atomic ticket.
//  K2 ffn_decode_kernel     a4..a7, persistent, one CTA per SM.  Warp 0 streams weight rows
//                           into a shared-memory ring with bulk asynchronous copies (TMA engine,
//                           mbarrier completion); the other warps dequantise from the ring.
//                           Phase 1 (gate/up) splits every expert's I rows evenly over the CTAs
//                           and writes h = SiLU(g)*u; a grid barrier; phase 2 (down + combine)
//                           gives every CTA a block of output rows over all experts and sums
//                           them in registers in a fixed order: no atomics, deterministic.  The
//                           shared expert comes first, so its rows stream while K1 routes.
//
// Dequantisation (dequant-on-use, same README section): phase 1 multiplies codes by activations
// held as 16-bit block fixed point (per 16-byte chunk of codes, one power-of-two scale) with
// dp2a integer dot products, exact in int32; the activation is exact for every element within a
// factor 2^7 of its chunk's largest magnitude (bf16 has 8 significant bits), smaller elements are
// rounded to 2^-15 of that maximum.  Phase 2 uses float32 with a positional magic-exponent
// decode (codes at their bit position, the activation pre-scaled by the matching power of two).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace coli {

namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int NCW = 16;              // consumer warps
constexpr int NC = NCW * 32;         // consumer threads
constexpr int NT = NC + 32;          // + producer warp
constexpr int PS1 = 8;               // (gate, up) row pairs per phase-1 stage
constexpr int RPT2MAX = 8;           // phase-2 rows per thread over the whole CTA row range
constexpr int CONS_BAR = 1;          // named barrier id of the consumer warps
constexpr long long WAIT_CYCLES = 4000000000LL;  // ~2 s at 1.9 GHz: bound of every spin-wait

// ------------------------------------------------------------------------- PTX helpers -----
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
// try_wait with a suspend-time hint (ns): a waiting warp sleeps instead of spinning, leaving
// issue slots to the warps that compute; it is woken when the phase completes.
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(a), "r"(parity), "r"(20000u) : "memory");
    return ok != 0;
}
// Bounded wait: false when the bound ran out (the caller records the error and gives up).
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    if (mbar_try(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(a, parity)) {
        if (clock64() - t0 > WAIT_CYCLES) return false;
    }
    return true;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar,
                                         uint64_t policy) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(mbar), "l"(policy) : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync %0, %1;" ::"n"(CONS_BAR), "n"(NC) : "memory"); }
__device__ __forceinline__ uint4 lds128(const unsigned char *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float4 ldcg4(const float *p) {
    return __ldcg(reinterpret_cast<const float4 *>(p));
}

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// ------------------------------------------------------------------------- code formats ----
// Codes per 16-byte chunk: int4 32, int8 16, int2 64.
template <int FMT> struct Fmt { static constexpr int CPC = 128 / FMT; };

// Integer dot of one 16-byte chunk of codes with its activation chunk (16-bit pairs laid out by
// prepare_x below).  Returns sum_j q_j * m_j exactly.
template <int FMT>
__device__ __forceinline__ int idot_chunk(const uint4 q, const int *xp, int corr);

template <>
__device__ __forceinline__ int idot_chunk<4>(const uint4 q, const int *xp, int corr) {
    // u = q + 8 per nibble (flip of the sign bit); bytes of lo hold elements 0,2,4,6 of a word,
    // bytes of hi hold 1,3,5,7.  xp holds per word: (m0,m2) (m4,m6) (m1,m3) (m5,m7).
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    int a0 = -corr, a1 = 0, a2 = 0, a3 = 0;  // corr = 8 * sum(m); four independent chains
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t f = w[i] ^ 0x88888888u;
        const uint32_t lo = f & 0x0F0F0F0Fu;
        const uint32_t hi = (f >> 4) & 0x0F0F0F0Fu;
        a0 = __dp2a_lo(xp[4 * i + 0], static_cast<int>(lo), a0);
        a1 = __dp2a_hi(xp[4 * i + 1], static_cast<int>(lo), a1);
        a2 = __dp2a_lo(xp[4 * i + 2], static_cast<int>(hi), a2);
        a3 = __dp2a_hi(xp[4 * i + 3], static_cast<int>(hi), a3);
    }
    return (a0 + a1) + (a2 + a3);
}
template <>
__device__ __forceinline__ int idot_chunk<8>(const uint4 q, const int *xp, int) {
    // signed bytes in natural order; xp holds (m0,m1) (m2,m3) per word
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    int a0 = 0, a1 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a0 = __dp2a_lo(xp[2 * i + 0], static_cast<int>(w[i]), a0);
        a1 = __dp2a_hi(xp[2 * i + 1], static_cast<int>(w[i]), a1);
    }
    return a0 + a1;
}
template <>
__device__ __forceinline__ int idot_chunk<2>(const uint4 q, const int *xp, int corr) {
    // u = q + 2 per 2-bit field; extraction k gives bytes with elements 4j+k (j = byte);
    // xp holds per word and k: (m_k, m_{4+k}) (m_{8+k}, m_{12+k}).
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    int a[4] = {-corr, 0, 0, 0};  // corr = 2 * sum(m)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t f = w[i] ^ 0xAAAAAAAAu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t b = (f >> (2 * k)) & 0x03030303u;
            a[k] = __dp2a_lo(xp[8 * i + 2 * k + 0], static_cast<int>(b), a[k]);
            a[k] = __dp2a_hi(xp[8 * i + 2 * k + 1], static_cast<int>(b), a[k]);
        }
    }
    return (a[0] + a[1]) + (a[2] + a[3]);
}

// Float decode of codes at their bit position.  A code field u sitting at mantissa bits
// [B*pos, B*pos + B) of a float whose exponent makes bit B*pos weigh exactly 1 (biased exponent
// 150 - B*pos) reads as 2^(23 - B*pos) + u; subtracting 2^(23 - B*pos) + BIAS gives the
// two's-complement code q = u - BIAS exactly (u is the code with its sign bit flipped).  Fields
// above bit 19 are first shifted down by SHIFT so that every field stays inside the mantissa.
template <int FMT> struct Fpos;
template <> struct Fpos<4> {  // element k of a word: nibble k at bits 4k
    static constexpr int SHIFT = 12, CUT = 5, BITS = 4, CPW = 8, BIAS = 8;
    static constexpr uint32_t FLIP = 0x88888888u, MASK = 0xFu;
};
template <> struct Fpos<8> {  // element k: byte k at bits 8k
    static constexpr int SHIFT = 16, CUT = 2, BITS = 8, CPW = 4, BIAS = 128;
    static constexpr uint32_t FLIP = 0x80808080u, MASK = 0xFFu;
};
template <> struct Fpos<2> {  // element k: bits 2k
    static constexpr int SHIFT = 10, CUT = 11, BITS = 2, CPW = 16, BIAS = 2;
    static constexpr uint32_t FLIP = 0xAAAAAAAAu, MASK = 0x3u;
};

__device__ __forceinline__ uint64_t pack_b64(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// One word of codes against its four activation pairs: acc += decoded codes * h (packed pairs).
template <int FMT>
__device__ __forceinline__ uint64_t fdot_word(uint32_t w, const uint64_t *hw, uint64_t acc) {
    using F = Fpos<FMT>;
    const uint32_t f0 = w ^ F::FLIP;
    const uint32_t f1 = f0 >> F::SHIFT;
#pragma unroll
    for (int k = 0; k < F::CPW; k += 2) {
        uint32_t bits[2];
        float off[2];
#pragma unroll
        for (int d = 0; d < 2; ++d) {
            const int kk = k + d;
            const int pos = kk < F::CUT ? kk : kk - F::SHIFT / F::BITS;
            const uint32_t src = kk < F::CUT ? f0 : f1;
            bits[d] = (src & (F::MASK << (F::BITS * pos))) | (static_cast<uint32_t>(150 - F::BITS * pos) << 23);
            off[d] = static_cast<float>(1u << (23 - F::BITS * pos)) + static_cast<float>(F::BIAS);
        }
        const uint64_t v = sub_f32x2(pack_b64(bits[0], bits[1]),
                                     pack_b64(__float_as_uint(off[0]), __float_as_uint(off[1])));
        acc = fma_f32x2(v, hw[k >> 1], acc);
    }
    return acc;
}

__device__ __forceinline__ float sum_pair(uint64_t v) {
    return __fadd_rn(__uint_as_float(static_cast<uint32_t>(v)), __uint_as_float(static_cast<uint32_t>(v >> 32)));
}

// Dots of two chunks of codes (two rows) with the same activations, four independent chains.
// hr holds the chunk's activations as float pairs (element 2i in the low half); element k of a
// word accumulates into the low lane for even k and the high lane for odd k; words 0-1 and 2-3
// go to separate pairs, summed at the end.
template <int FMT>
__device__ __forceinline__ void fdot2_chunk(const uint4 q0, const uint4 q1, const uint64_t *hr, float &d0, float &d1) {
    constexpr int HP = Fpos<FMT>::CPW / 2;  // activation pairs per word
    uint64_t a0 = 0ull, b0 = 0ull, a1 = 0ull, b1 = 0ull;
    a0 = fdot_word<FMT>(q0.x, hr + 0 * HP, a0);
    a1 = fdot_word<FMT>(q1.x, hr + 0 * HP, a1);
    b0 = fdot_word<FMT>(q0.z, hr + 2 * HP, b0);
    b1 = fdot_word<FMT>(q1.z, hr + 2 * HP, b1);
    a0 = fdot_word<FMT>(q0.y, hr + 1 * HP, a0);
    a1 = fdot_word<FMT>(q1.y, hr + 1 * HP, a1);
    b0 = fdot_word<FMT>(q0.w, hr + 3 * HP, b0);
    b1 = fdot_word<FMT>(q1.w, hr + 3 * HP, b1);
    d0 = __fadd_rn(sum_pair(a0), sum_pair(b0));
    d1 = __fadd_rn(sum_pair(a1), sum_pair(b1));
}

__device__ __forceinline__ float warp_allsum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

// ------------------------------------------------------------------------- K1 router -------
__device__ __forceinline__ bool beats(double va, int ia, double vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// Route token t with the whole CTA (256 threads) and write ids/weights; smem scratch given.
__device__ void route_token_cta(const DecodeParams &p, int t, double *cs, double *ss, double *gsc,
                                int *kept, int *sel_id, double *sel_s) {
    const int E = p.f.E, K = p.f.K, G = p.G, TG = p.TG;
    const int gs = E / G;
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) {
        const double l = static_cast<double>(__ldcg(p.logits + static_cast<size_t>(t) * E + e));
        const double s = 1.0 / (1.0 + exp(-l));
        ss[e] = s;
        cs[e] = s + static_cast<double>(p.bias[e]);
    }
    __syncthreads();
    if (G > 1 && TG < G) {
        for (int g = tid; g < G; g += blockDim.x) {
            double a1 = -INFINITY, a2 = -INFINITY;
            for (int e = g * gs; e < (g + 1) * gs; ++e) {
                const double v = cs[e];
                if (v > a1) { a2 = a1; a1 = v; }
                else if (v > a2) { a2 = v; }
            }
            gsc[g] = a1 + a2;
        }
        __syncthreads();
        for (int g = tid; g < G; g += blockDim.x) {
            int r = 0;
            for (int h = 0; h < G; ++h) r += beats(gsc[h], h, gsc[g], g);
            kept[g] = r < TG;
        }
    } else {
        for (int g = tid; g < G; g += blockDim.x) kept[g] = 1;
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        if (!kept[e / gs]) continue;
        const double v = cs[e];
        int r = 0;
        for (int g = 0; g < G; ++g) {
            if (!kept[g]) continue;
            for (int f = g * gs; f < (g + 1) * gs; ++f) r += beats(cs[f], f, v, e);
        }
        if (r < K) { sel_id[r] = e; sel_s[r] = ss[e]; }
    }
    __syncthreads();
    if (tid < K) {
        double denom = 0.0;
        for (int k = 0; k < K; ++k) denom += sel_s[k];
        p.ids[static_cast<size_t>(t) * K + tid] = sel_id[tid];
        p.wts[static_cast<size_t>(t) * K + tid] = static_cast<float>((sel_s[tid] / denom) * p.rsf);
    }
}

// Group the n = T*K <= 32 slots of the batch: warp 0 ranks the slots by (expert id, slot) with
// shuffles (a stable sort), the unique list follows from the sorted order; every thread fills the
// per-expert counts and offsets by scanning the n slots.
__device__ void group_batch_cta(const DecodeParams &p, int *sid, int *ssorted) {
    const int E = p.f.E, n = p.f.T * p.f.K;
    const int tid = threadIdx.x;
    if (tid < 32) {
        const int lane = tid;
        const int id = lane < n ? __ldcg(p.ids + lane) : 0x7fffffff;
        sid[lane] = id;
        int r = 0;
        for (int s2 = 0; s2 < 32; ++s2) {
            const int o = __shfl_sync(FULL, id, s2);
            r += (o < id) || (o == id && s2 < lane);
        }
        if (lane < n) {
            p.f_perm[r] = lane;
            ssorted[r] = id;
        }
        __syncwarp();
        const int idr = lane < n ? ssorted[lane] : 0x7fffffff;
        const bool first = lane < n && (lane == 0 || ssorted[lane - 1] != idr);
        const unsigned m = __ballot_sync(FULL, first);
        const int up = __popc(m & ((1u << lane) - 1u));
        if (first) p.f_unique[up] = idr;
        if (lane == 0) {
            *p.f_nuniq = __popc(m);
            p.f_offsets[E] = n;
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        int c = 0, lt = 0;
        for (int s2 = 0; s2 < n; ++s2) {
            const int v = sid[s2];
            c += v == e;
            lt += v < e;
        }
        p.f_counts[e] = c;
        p.f_offsets[e] = lt;
    }
    // unique entries past the last are -1: the number of distinct ids is known to every thread
    int distinct = 0;
    for (int s2 = 0; s2 < n; ++s2) distinct += (s2 == 0 || ssorted[s2 - 1] != ssorted[s2]);
    for (int e = tid; e < E; e += blockDim.x)
        if (e >= distinct) p.f_unique[e] = -1;
}

__global__ void __launch_bounds__(256) router_decode_kernel(DecodeParams p) {
    grid_dep_launch();  // let the FFN kernel start streaming the shared expert
    const int H = p.f.H, E = p.f.E;
    const int t = blockIdx.y;
    const int half = threadIdx.x >> 7, l = threadIdx.x & 127;
    const int e = blockIdx.x * 2 + half;
    __shared__ double red[8];
    // a1: one Wr row per 128 threads, products and sums in double.  Loads are issued in groups
    // of GB so that a thread's whole slice of the row is in flight at once (H <= GB * 512 * 2).
    constexpr int GB = 6;
    double acc = 0.0;
    if (e < E) {
        const float *wrow = p.Wr + static_cast<size_t>(e) * H;
        for (int base = l * 4; base < H; base += GB * 512) {
            float4 wv[GB];
            float xv[GB][4];
#pragma unroll
            for (int g = 0; g < GB; ++g) {
                const int h0 = base + g * 512;
                if (h0 < H) {
                    wv[g] = __ldg(reinterpret_cast<const float4 *>(wrow + h0));
                    if (p.f.act == COLI_ACT_F32) {
                        const float4 f4 = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p.f.x) + static_cast<size_t>(t) * H + h0));
                        xv[g][0] = f4.x; xv[g][1] = f4.y; xv[g][2] = f4.z; xv[g][3] = f4.w;
                    } else {
                        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(p.f.x) + static_cast<size_t>(t) * H + h0));
                        xv[g][0] = __uint_as_float(u.x << 16); xv[g][1] = __uint_as_float(u.x & 0xffff0000u);
                        xv[g][2] = __uint_as_float(u.y << 16); xv[g][3] = __uint_as_float(u.y & 0xffff0000u);
                    }
                } else {
                    wv[g] = make_float4(0.f, 0.f, 0.f, 0.f);
                    xv[g][0] = xv[g][1] = xv[g][2] = xv[g][3] = 0.f;
                }
            }
#pragma unroll
            for (int g = 0; g < GB; ++g) {
                acc = fma(static_cast<double>(wv[g].x), static_cast<double>(xv[g][0]), acc);
                acc = fma(static_cast<double>(wv[g].y), static_cast<double>(xv[g][1]), acc);
                acc = fma(static_cast<double>(wv[g].z), static_cast<double>(xv[g][2]), acc);
                acc = fma(static_cast<double>(wv[g].w), static_cast<double>(xv[g][3]), acc);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (l == 0 && e < E) {
        const double s = red[half * 4 + 0] + red[half * 4 + 1] + red[half * 4 + 2] + red[half * 4 + 3];
        p.logits[static_cast<size_t>(t) * E + e] = static_cast<float>(s);
    }
    // last CTA of token t routes it; last token router groups the batch
    __shared__ int last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned ticket = atomicAdd(p.tok_cnt + t, 1u);
        last = ticket == gridDim.x - 1;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    extern __shared__ unsigned char dyn[];
    double *cs = reinterpret_cast<double *>(dyn);
    double *ss = cs + E;
    double *gsc = ss + E;
    double *sel_s = gsc + 32;
    int *kept = reinterpret_cast<int *>(sel_s + 32);
    int *sel_id = kept + 32;
    route_token_cta(p, t, cs, ss, gsc, kept, sel_id, sel_s);
    __syncthreads();
    if (threadIdx.x == 0) {
        p.tok_cnt[t] = 0u;
        __threadfence();
        const unsigned ticket = atomicAdd(p.route_cnt, 1u);
        last = ticket == gridDim.y - 1;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    int *sid = sel_id + 32;
    int *ssorted = sid + 64;
    group_batch_cta(p, sid, ssorted);
    __syncthreads();
    if (threadIdx.x == 0) {
        *p.route_cnt = 0u;
        __threadfence();
    }
}

// ------------------------------------------------------------------------- K2 FFN ----------
// Phase 1: a stage holds PS (gate row, up row) pairs of one expert; consumer warp w works on pair
// w % PS of the stages whose sequence number is w / PS modulo NCW / PS, reduces its rows with
// shuffles and writes h itself.  Every consumer warp waits on every stage's full barrier and
// arrives on its empty barrier (count NCW), so a stage is refilled only after all its readers
// are done.  Phase 2: a stage holds the CTA's whole block of down rows of one expert; consumer
// thread (p2, c2) owns chunk c2 of rows p2 + P2*m and keeps per-(row, token) partial sums in
// registers across experts; one cross-lane reduction at the end.
template <int FMT, int TMAX>
__global__ void __maxnreg__(96) ffn_decode_kernel(DecodeParams p) {
    constexpr int CPC = Fmt<FMT>::CPC;       // codes per 16-byte chunk
    constexpr int XW = CPC / 2;              // int32 words of 16-bit activations per chunk
    constexpr int XV = XW / 4;               // int4 vectors per chunk
    extern __shared__ __align__(1024) unsigned char sm[];
    const FfnParams &f = p.f;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, b = blockIdx.x;
    const int S = p.S;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm);          // full[S], empty[S]
    int *rt = reinterpret_cast<int *>(sm + p.off_route);         // routing cache
    int4 *xq = reinterpret_cast<int4 *>(sm + p.off_x);            // [T][XV][Lh] (transposed)
    float *xs = reinterpret_cast<float *>(sm + p.off_xs);         // [T][Lh] scale
    int *xc = reinterpret_cast<int *>(sm + p.off_xc);             // [T][Lh] correction
    float *red2 = reinterpret_cast<float *>(sm + p.off_red);      // phase-2 partials
    float4 *hb = reinterpret_cast<float4 *>(sm + p.off_x);        // phase-2 h (aliases x)
    unsigned char *ring = sm + p.off_ring;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    const int Lh = p.Lh, Li = p.Li;
    const int PS = p.R1;                     // pairs per phase-1 stage

    const int i_lo = static_cast<int>(static_cast<long>(f.I) * b / G), i_hi = static_cast<int>(static_cast<long>(f.I) * (b + 1) / G);
    const int j_lo = static_cast<int>(static_cast<long>(f.H) * b / G), j_hi = static_cast<int>(static_cast<long>(f.H) * (b + 1) / G);
    const int n1 = (i_hi - i_lo + PS - 1) / PS;  // phase-1 stages per expert

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), NCW);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- producer --------
        if (lane != 0) return;
        const uint64_t pol = evict_first_policy();
        int seq = 0, U = 0;
        int uniq[32];
        bool have_routing = false, ok = true;
        auto record = [&](int we) -> const uint8_t * {
            if (we < f.S) return f.shared;
            const int e = uniq[we - f.S];
            return (e >= 0 && e < f.E) ? f.experts + static_cast<size_t>(e) * f.stride : nullptr;
        };
        for (int we = 0; ok; ++we) {
            if (we >= f.S && !have_routing) {
                grid_dep_wait();
                U = __ldcg(f.n_unique);
                U = U < 0 ? 0 : (U > 32 ? 32 : U);
                for (int u = 0; u < U; ++u) uniq[u] = __ldcg(f.unique + u);
                have_routing = true;
            }
            if (have_routing && we >= f.S + U) break;
            const uint8_t *rec = record(we);
            for (int k = 0; k < n1 && ok; ++k, ++seq) {
                const int s = seq % S;
                const uint32_t par = (seq / S) & 1;
                if (!mbar_wait(empty_bar(s), par ^ 1)) { ok = false; break; }
                const int r0 = i_lo + k * PS, n = min(PS, i_hi - r0);
                const uint32_t dst = smem_u32(ring + static_cast<size_t>(s) * p.SB);
                if (rec == nullptr) { mbar_arrive(full_bar(s)); continue; }
                const int a0 = r0 & ~3, a1 = (r0 + n + 3) & ~3;
                const uint32_t bytes = 2u * n * static_cast<uint32_t>(f.rb_h) + 2u * 4u * (a1 - a0);
                mbar_expect_tx(full_bar(s), bytes);
                bulk_g2s(dst, rec + static_cast<size_t>(r0) * f.rb_h, n * f.rb_h, full_bar(s), pol);
                bulk_g2s(dst + p.st_up, rec + f.off_wu + static_cast<size_t>(r0) * f.rb_h, n * f.rb_h, full_bar(s), pol);
                bulk_g2s(dst + p.st_sg, rec + f.off_sg + 4 * a0, 4 * (a1 - a0), full_bar(s), pol);
                bulk_g2s(dst + p.st_su, rec + f.off_su + 4 * a0, 4 * (a1 - a0), full_bar(s), pol);
            }
        }
        for (int we = 0; ok && we < f.S + U; ++we, ++seq) {
            const uint8_t *rec = record(we);
            const int s = seq % S;
            const uint32_t par = (seq / S) & 1;
            if (!mbar_wait(empty_bar(s), par ^ 1)) { ok = false; break; }
            const uint32_t dst = smem_u32(ring + static_cast<size_t>(s) * p.SB);
            if (rec == nullptr) { mbar_arrive(full_bar(s)); continue; }
            const int n = j_hi - j_lo;
            const int a0 = j_lo & ~3, a1 = (j_hi + 3) & ~3;
            const uint32_t bytes = n * static_cast<uint32_t>(f.rb_i) + 4u * (a1 - a0);
            mbar_expect_tx(full_bar(s), bytes);
            bulk_g2s(dst, rec + f.off_wd + static_cast<size_t>(j_lo) * f.rb_i, n * f.rb_i, full_bar(s), pol);
            bulk_g2s(dst + p.st_sd, rec + f.off_sd + 4 * a0, 4 * (a1 - a0), full_bar(s), pol);
        }
        if (!ok) atomicOr(f.err, COLI_DEVERR_TIMEOUT);
        return;
    }

    // -------------------------------------------------------------------- consumers --------
    const int ct = threadIdx.x - 32;
    const int cw = ct >> 5;
    const int T = f.T;
    bool ok = true;

    // activations -> 16-bit block fixed point per (token, chunk), transposed for conflict-free
    // reads: int4 vector v of chunk c of token t at xq[(t * XV + v) * Lh + c]
    for (int idx = ct; idx < T * Lh; idx += NC) {
        const int t = idx / Lh, c = idx % Lh;
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(f.x) +
                                                          static_cast<size_t>(t) * f.H + static_cast<size_t>(c) * CPC);
        uint32_t raw[CPC / 2];  // bf16 pairs
#pragma unroll
        for (int i = 0; i < CPC / 8; ++i) {
            const uint4 v = __ldg(src + i);
            raw[4 * i] = v.x; raw[4 * i + 1] = v.y; raw[4 * i + 2] = v.z; raw[4 * i + 3] = v.w;
        }
        auto xval = [&](int j) -> float {
            const uint32_t w2 = raw[j >> 1];
            return __uint_as_float((j & 1) ? (w2 & 0xffff0000u) : (w2 << 16));
        };
        float mx = 0.f;
#pragma unroll
        for (int j = 0; j < CPC; ++j) mx = fmaxf(mx, fabsf(xval(j)));
        int ex = 0;
        if (mx > 0.f) frexpf(mx, &ex);            // mx < 2^ex
        const float up = ldexpf(1.0f, 15 - ex);    // |x * up| < 2^15
        auto mq = [&](int j) -> int { return max(-32767, min(32767, __float2int_rn(xval(j) * up))); };
        auto pk = [](int a, int bb) { return static_cast<int>((static_cast<uint32_t>(a) & 0xffffu) | (static_cast<uint32_t>(bb) << 16)); };
        int w[XW];
        int sum = 0;
        if (FMT == 4) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int m[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) { m[j] = mq(8 * i + j); sum += m[j]; }
                w[4 * i + 0] = pk(m[0], m[2]);
                w[4 * i + 1] = pk(m[4], m[6]);
                w[4 * i + 2] = pk(m[1], m[3]);
                w[4 * i + 3] = pk(m[5], m[7]);
            }
            xc[idx] = 8 * sum;
        } else if (FMT == 8) {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = pk(mq(2 * i), mq(2 * i + 1));
            xc[idx] = 0;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int m[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) { m[j] = mq(16 * i + j); sum += m[j]; }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    w[8 * i + 2 * k + 0] = pk(m[k], m[4 + k]);
                    w[8 * i + 2 * k + 1] = pk(m[8 + k], m[12 + k]);
                }
            }
            xc[idx] = 2 * sum;
        }
#pragma unroll
        for (int v = 0; v < XV; ++v)
            xq[(static_cast<size_t>(t) * XV + v) * Lh + c] = make_int4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        xs[idx] = 1.0f / up;
    }

    // routing cache: [0] U; rBeg/rCnt per work expert; per slot: token, weight, h row
    int *rU = rt;
    int *rBeg = rt + 1;
    int *rCnt = rBeg + 33;
    int *rTok = rCnt + 33;
    float *rW = reinterpret_cast<float *>(rTok + 8 * 33);
    int *rH = reinterpret_cast<int *>(rW + 8 * 33);
    bool have_routing = false;
    auto get_routing = [&]() {
        grid_dep_wait();
        if (cw == 0) {  // lane u handles unique expert u (U <= 32)
            int U = __ldcg(f.n_unique);
            U = U < 0 ? 0 : (U > 32 ? 32 : U);
            int e = -1, b0 = 0, c0 = 0;
            if (lane < U) {
                e = __ldcg(f.unique + lane);
                if (e >= 0 && e < f.E) {
                    b0 = __ldcg(f.offsets + e);
                    c0 = __ldcg(f.offsets + e + 1) - b0;
                    if (b0 < 0 || c0 < 0 || b0 + c0 > T * f.K || c0 > TMAX) { c0 = 0; atomicOr(f.err, COLI_DEVERR_GROUPING); }
                } else {
                    atomicOr(f.err, COLI_DEVERR_EXPERT_ID);
                }
            }
            int pos = c0;  // exclusive scan of the slot counts
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(FULL, pos, o);
                if (lane >= o) pos += v;
            }
            pos -= c0;
            if (lane == 0) *rU = U;
            if (lane < U) {
                rBeg[f.S + lane] = pos;
                rCnt[f.S + lane] = c0;
                for (int q = 0; q < c0; ++q) {
                    const int sl = __ldcg(f.perm + b0 + q);
                    const bool good = sl >= 0 && sl < T * f.K;
                    if (!good) atomicOr(f.err, COLI_DEVERR_GROUPING);
                    rTok[pos + q] = good ? sl / f.K : 0;
                    rW[pos + q] = good ? __ldcg(f.topk_w + sl) : 0.f;
                    rH[pos + q] = good ? b0 + q : 0;
                }
            }
        }
        cons_sync();
        have_routing = true;
    };
    cons_sync();  // activations ready

    // ------------------------------------------------ phase 1: gate/up, h = SiLU(g)*u -----
    // After a timed-out wait a thread keeps walking the same loops and barriers (skipping later
    // waits), so that no consumer is ever left alone at a named barrier.
    const int NJ = Lh / 32;                  // chunks per lane in a row
    const int NGRP = NCW / PS;               // stage groups
    const int my_pair = cw % PS, my_grp = cw / PS;
    int seq = 0, U = 0;
    for (int we = 0;; ++we) {
        if (we >= f.S && !have_routing) { get_routing(); U = *rU; }
        if (have_routing && we >= f.S + U) break;
        const bool shared = we < f.S;
        const int cnt = shared ? T : rCnt[we];
        const int beg = shared ? 0 : rBeg[we];
        for (int k = 0; k < n1; ++k, ++seq) {
            const int s = seq % S;
            const uint32_t par = (seq / S) & 1;
            if (ok && !mbar_wait(full_bar(s), par)) ok = false;
            const int r0 = i_lo + k * PS, n = min(PS, i_hi - r0);
            const bool mine = ok && (seq % NGRP) == my_grp && my_pair < n && my_grp < NGRP;
            if (mine) {
                const unsigned char *st = ring + static_cast<size_t>(s) * p.SB;
                const unsigned char *rg = st + static_cast<size_t>(my_pair) * f.rb_h;
                const unsigned char *ru = st + p.st_up + static_cast<size_t>(my_pair) * f.rb_h;
                float g[TMAX], u[TMAX];
                const int4 *xb[TMAX];
                const float *xsb[TMAX];
                const int *xcb[TMAX];
#pragma unroll
                for (int q = 0; q < TMAX; ++q) {
                    g[q] = 0.f; u[q] = 0.f;
                    const int tok = q < cnt ? (shared ? q : rTok[beg + q]) : 0;
                    xb[q] = xq + static_cast<size_t>(tok) * XV * Lh + lane;
                    xsb[q] = xs + tok * Lh + lane;
                    xcb[q] = xc + tok * Lh + lane;
                }
                const unsigned char *rgl = rg + lane * 16, *rul = ru + lane * 16;
#pragma unroll 2
                for (int j = 0; j < NJ; ++j) {
                    const uint4 qg = lds128(rgl + j * 512);
                    const uint4 qu = lds128(rul + j * 512);
#pragma unroll
                    for (int q = 0; q < TMAX; ++q) {
                        if (q < cnt) {
                            int xr[XW];
#pragma unroll
                            for (int v = 0; v < XV; ++v) {
                                const int4 t4 = xb[q][v * Lh + 32 * j];
                                xr[4 * v] = t4.x; xr[4 * v + 1] = t4.y; xr[4 * v + 2] = t4.z; xr[4 * v + 3] = t4.w;
                            }
                            const float sc = xsb[q][32 * j];
                            const int corr = xcb[q][32 * j];
                            g[q] = __fmaf_rn(static_cast<float>(idot_chunk<FMT>(qg, xr, corr)), sc, g[q]);
                            u[q] = __fmaf_rn(static_cast<float>(idot_chunk<FMT>(qu, xr, corr)), sc, u[q]);
                        }
                    }
                }
                const int a0 = r0 & ~3;
                const float sgv = reinterpret_cast<const float *>(st + p.st_sg)[r0 + my_pair - a0];
                const float suv = reinterpret_cast<const float *>(st + p.st_su)[r0 + my_pair - a0];
#pragma unroll
                for (int q = 0; q < TMAX; ++q) {
                    if (q < cnt) {
                        const float gq = __fmul_rn(warp_allsum(g[q]), sgv);
                        const float uq = __fmul_rn(warp_allsum(u[q]), suv);
                        if (lane == q) {
                            const int hrow = shared ? T * f.K + q : rH[beg + q];
                            f.h[static_cast<size_t>(hrow) * f.I + r0 + my_pair] =
                                __fmul_rn(__fdiv_rn(gq, __fadd_rn(1.0f, expf(-gq))), uq);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));
        }
    }

    // ------------------------------------------------ grid barrier ------------------------
    cons_sync();
    if (ct == 0) {
        __threadfence();
        atomicAdd(p.gbar, 1u);
        const long long t0 = clock64();
        while (ld_acquire(p.gbar) < static_cast<unsigned>(G)) {
            if (clock64() - t0 > WAIT_CYCLES) { atomicOr(f.err, COLI_DEVERR_TIMEOUT); break; }
            __nanosleep(64);
        }
        // the last CTA to leave the barrier zeroes both counters for the next call
        if (atomicAdd(p.gdep, 1u) == static_cast<unsigned>(G) - 1u) {
            *p.gbar = 0u;
            *p.gdep = 0u;
            __threadfence();
        }
    }
    cons_sync();

    // ------------------------------------------------ phase 2: down + combine -------------
    const int p2 = ct / Li, c2 = ct % Li;
    const int P2 = p.P2;
    const int nwr2 = Li / 32;
    constexpr int HV = CPC / 4;              // float4 vectors of h per chunk
    float acc[RPT2MAX][TMAX];
#pragma unroll
    for (int m = 0; m < RPT2MAX; ++m)
#pragma unroll
        for (int q = 0; q < TMAX; ++q) acc[m][q] = 0.f;
    const int nrows = j_hi - j_lo;
    const int a0d = j_lo & ~3;
    const int nwe = f.S + U;
    // h of an expert's slots -> shared memory with cp.async, transposed: float4 vector v of
    // chunk c of slot q at hb[buf][(q * HV + v) * Li + c]
    const size_t hbuf = static_cast<size_t>(TMAX) * HV * Li;  // float4 per buffer
    auto stage_h = [&](int we) {
        const bool shd = we < f.S;
        const int cnt = shd ? T : rCnt[we];
        const int beg = shd ? 0 : rBeg[we];
        float4 *dstb = hb + (we & 1) * hbuf;
        const int per = HV * Li;             // float4 per slot
        for (int idx = ct; idx < cnt * per; idx += NC) {
            const int q = idx / per, r = idx % per;
            const int c = r / HV, v = r % HV;  // source order: chunk-major
            const int hrow = shd ? T * f.K + q : rH[beg + q];
            const uint32_t d = smem_u32(dstb + (static_cast<size_t>(q) * HV + v) * Li + c);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d),
                         "l"(f.h + static_cast<size_t>(hrow) * f.I + static_cast<size_t>(c) * CPC + 4 * v) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (nwe > 0) stage_h(0);
    for (int we = 0; we < nwe; ++we) {
        const bool shared = we < f.S;
        const int cnt = shared ? T : rCnt[we];
        const int beg = shared ? 0 : rBeg[we];
        cons_sync();                               // everyone is done with buffer (we+1)&1
        if (we + 1 < nwe) {
            stage_h(we + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        cons_sync();                               // buffer we&1 is complete
        const float4 *hcur = hb + (we & 1) * hbuf;
        const int s = seq % S;
        const uint32_t par = (seq / S) & 1;
        ++seq;
        if (ok && !mbar_wait(full_bar(s), par)) ok = false;
        if (ok) {
            const unsigned char *st = ring + static_cast<size_t>(s) * p.SB;
            const float *sdp = reinterpret_cast<const float *>(st + p.st_sd) + (j_lo - a0d);
            for (int q = 0; q < cnt; ++q) {
                const int tok = shared ? q : rTok[beg + q];
                const float wq = shared ? 1.0f : rW[beg + q];
                uint64_t hr[CPC / 2];
#pragma unroll
                for (int v = 0; v < HV; ++v) {
                    const ulonglong2 t2 = *reinterpret_cast<const ulonglong2 *>(hcur + (static_cast<size_t>(q) * HV + v) * Li + c2);
                    hr[2 * v] = t2.x; hr[2 * v + 1] = t2.y;
                }
#pragma unroll
                for (int m = 0; m < RPT2MAX; m += 2) {
                    const int row0 = p2 + P2 * m, row1 = row0 + P2;
                    if (row0 < nrows) {
                        const bool has1 = row1 < nrows;
                        const uint4 qd0 = lds128(st + static_cast<size_t>(row0) * f.rb_i + c2 * 16);
                        const uint4 qd1 = has1 ? lds128(st + static_cast<size_t>(row1) * f.rb_i + c2 * 16) : make_uint4(0, 0, 0, 0);
                        const float wsd0 = __fmul_rn(wq, sdp[row0]);
                        const float wsd1 = has1 ? __fmul_rn(wq, sdp[row1]) : 0.f;
                        float d0, d1;
                        fdot2_chunk<FMT>(qd0, qd1, hr, d0, d1);
#pragma unroll
                        for (int t2 = 0; t2 < TMAX; ++t2)
                            if (t2 == tok) {
                                acc[m][t2] = __fmaf_rn(d0, wsd0, acc[m][t2]);
                                acc[m + 1][t2] = __fmaf_rn(d1, wsd1, acc[m + 1][t2]);
                            }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
    }
    if (!ok) atomicOr(f.err, COLI_DEVERR_TIMEOUT);
    // cross-lane reduction of the accumulators, then one store per (token, row)
#pragma unroll
    for (int m = 0; m < RPT2MAX; ++m)
#pragma unroll
        for (int q = 0; q < TMAX; ++q) {
            if (q < T) {
                const float v = warp_allsum(acc[m][q]);
                if (lane == 0) red2[((p2 * RPT2MAX + m) * TMAX + q) * nwr2 + (c2 >> 5)] = v;
            }
        }
    cons_sync();
    for (int fi = ct; fi < P2 * RPT2MAX * T; fi += NC) {
        const int q = fi % T, m = (fi / T) % RPT2MAX, ps = fi / (T * RPT2MAX);
        const int row = ps + P2 * m;
        if (row >= nrows) continue;
        float v = 0.f;
        for (int w = 0; w < nwr2; ++w) v = __fadd_rn(v, red2[((ps * RPT2MAX + m) * TMAX + q) * nwr2 + w]);
        f.out[static_cast<size_t>(q) * f.H + j_lo + row] = v;
    }
}

template <int FMT, int TMAX>
cudaError_t launch_k2(const DecodeParams &p, size_t smem, cudaStream_t st, bool pdl) {
    auto kern = ffn_decode_kernel<FMT, TMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int FMT>
cudaError_t launch_k2_t(const DecodeParams &p, size_t smem, cudaStream_t st, bool pdl) {
    if (p.f.T <= 1) return launch_k2<FMT, 1>(p, smem, st, pdl);
    if (p.f.T <= 2) return launch_k2<FMT, 2>(p, smem, st, pdl);
    return launch_k2<FMT, 4>(p, smem, st, pdl);
}

}  // namespace

// The register allocation of a kernel instantiation bounds its block size: check it fits NT.
template <int FMT, int TMAX>
static bool fits_block() {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, ffn_decode_kernel<FMT, TMAX>) != cudaSuccess) return false;
    return fa.maxThreadsPerBlock >= NT;
}
static bool kernel_fits(int fmt, int T) {
    const int tm = T <= 1 ? 1 : (T <= 2 ? 2 : 4);
#define COLI_FITS(F)                                                        \
    if (fmt == F) return tm == 1 ? fits_block<F, 1>() : (tm == 2 ? fits_block<F, 2>() : fits_block<F, 4>());
    COLI_FITS(4) COLI_FITS(8) COLI_FITS(2)
#undef COLI_FITS
    return false;
}

// Shape rules and the shared-memory plan of the fused decode path.
bool decode_plan(const coli_moe_config &c, int T, DecodePlan *plan) {
    if (T < 1 || T > 4) return false;
    if (c.act != COLI_ACT_BF16) return false;  // 16-bit block fixed point is exact for bf16 only
    if (c.n_experts > 1024 || c.top_k * T > 32 || c.n_group > 32) return false;
    if (c.hidden % 512) return false;
    const int sms = device_sm_count();
    const int rb_h = c.hidden * c.wfmt / 8, rb_i = c.inter * c.wfmt / 8;
    const int Lh = rb_h / 16, Li = rb_i / 16;
    if (rb_h % 16 || rb_i % 16 || Lh % 32 || Li % 32 || NC % Li) return false;
    if (NCW % PS1) return false;
    const int P2 = NC / Li;
    const int rows2 = (c.hidden + sms - 1) / sms;
    if (c.inter < sms || c.hidden < sms) return false;
    if (rows2 > P2 * RPT2MAX) return false;
    const int tmax = T <= 1 ? 1 : (T <= 2 ? 2 : 4);
    if (!kernel_fits(c.wfmt, T)) return false;
    DecodePlan pl;
    pl.grid = sms;
    pl.Lh = Lh; pl.Li = Li; pl.P1 = 0; pl.P2 = P2; pl.R1 = PS1;
    // stage layout (phase 1: gate rows | up rows | sg | su; phase 2: down rows | sd)
    const int scal1 = ((PS1 + 8 + 3) / 4) * 16;
    const int scal2 = ((rows2 + 8 + 3) / 4) * 16;
    pl.st_up = PS1 * rb_h;
    pl.st_sg = 2 * PS1 * rb_h;
    pl.st_su = pl.st_sg + scal1;
    const int sb1 = pl.st_su + scal1;
    pl.st_sd = rows2 * rb_i;
    const int sb2 = pl.st_sd + scal2;
    pl.SB = ((sb1 > sb2 ? sb1 : sb2) + 127) / 128 * 128;
    // shared memory: barriers | routing cache | x (phase 1) or h (phase 2) | x scales |
    // corrections | phase-2 partials | ring
    size_t o = 1024;  // barriers (up to 64 stages)
    pl.off_route = o; o += 4096;
    pl.off_x = o;
    const size_t xbytes = static_cast<size_t>(T) * c.hidden * 2;
    const size_t hbytes = static_cast<size_t>(2) * tmax * c.inter * 4;  // two buffers of TMAX h rows
    o += ((xbytes > hbytes ? xbytes : hbytes) + 127) / 128 * 128;
    pl.off_xs = o; o += static_cast<size_t>(T) * Lh * 4;
    pl.off_xc = o; o += static_cast<size_t>(T) * Lh * 4;
    o = (o + 127) / 128 * 128;
    pl.red1_len = 0;
    const int red2_len = P2 * RPT2MAX * tmax * (Li / 32);
    pl.off_red = o; o += static_cast<size_t>(red2_len) * 4;
    o = (o + 1023) / 1024 * 1024;
    pl.off_ring = o;
    const size_t budget = device_smem_optin() - 1024;
    if (o + 2 * static_cast<size_t>(pl.SB) > budget) return false;
    pl.S = static_cast<int>((budget - o) / pl.SB);
    if (pl.S > 8) pl.S = 8;
    pl.smem = o + static_cast<size_t>(pl.S) * pl.SB;
    *plan = pl;
    return true;
}

static void fill_plan(DecodeParams &p, const DecodePlan &pl) {
    p.grid = pl.grid; p.Lh = pl.Lh; p.Li = pl.Li; p.P1 = pl.P1; p.P2 = pl.P2; p.R1 = pl.R1;
    p.S = pl.S; p.SB = pl.SB; p.st_up = pl.st_up; p.st_sg = pl.st_sg; p.st_su = pl.st_su; p.st_sd = pl.st_sd;
    p.off_route = pl.off_route; p.off_x = pl.off_x; p.off_xs = pl.off_xs; p.off_xc = pl.off_xc;
    p.off_red = pl.off_red; p.off_ring = pl.off_ring; p.red1_len = pl.red1_len;
}

cudaError_t launch_ffn_decode(DecodeParams p, const DecodePlan &pl, cudaStream_t st, bool pdl) {
    fill_plan(p, pl);
    if (p.f.fmt == 4) return launch_k2_t<4>(p, pl.smem, st, pdl);
    if (p.f.fmt == 8) return launch_k2_t<8>(p, pl.smem, st, pdl);
    if (p.f.fmt == 2) return launch_k2_t<2>(p, pl.smem, st, pdl);
    return cudaErrorInvalidValue;
}

cudaError_t launch_router_decode(DecodeParams p, cudaStream_t st) {
    const int E = p.f.E;
    const size_t smem = static_cast<size_t>(E) * 16 + 64 * 8 + (32 + 32 + 64) * 4 + static_cast<size_t>(3 * E + 1) * 4 + 64;
    cudaError_t e = cudaFuncSetAttribute(router_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid((E + 1) / 2, p.f.T);
    router_decode_kernel<<<grid, 256, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace coli
