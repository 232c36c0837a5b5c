// decode.cu -- the fused decode path of the layer for a few tokens (decode and MTP verify).
//
// One persistent launch, one CTA per SM (ffn_decode_kernel):
//
//  phase 0  a1 gate: CTA b computes the logits of experts [b*E/G, (b+1)*E/G) in double from
//           exact double products and arrives on a grid counter.  After the shared expert's
//           gate/up rows, every CTA waits for all logits and routes the batch itself (a2,
//           noaux_tc, colibri-strix README "What's implemented") and groups it (a3, batch-union):
//           the same code on the same inputs, so all CTAs agree bit for bit; CTA 0 writes the
//           routing outputs of the call.  (For coli_moe_ffn the routing arrays are inputs.)
//  phases 1-2 (a4..a7).  Warp 0 streams weight rows
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
// rounded to 2^-15 of that maximum.  Phase 2 takes h as 16-bit fixed point per chunk split in two
// signed bytes and the codes as signed bytes (16q for int4, 64q for int2), so dp4a integer dot
// products are exact; h is rounded to 2^-16 of its chunk's largest magnitude.
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
constexpr int CONS_BAR = 1;          // named barrier id of the consumer warps (2..5: per-token routing)
// routing cache in shared memory (int offsets): U | unique[32] | beg[33] | cnt[33] | tok[32] | w[32] | hrow[32] | sorted slots[32]
constexpr int RT_UNIQ = 1, RT_BEG = 33, RT_CNT = 66, RT_TOK = 99, RT_W = 131, RT_H = 163, RT_SORT = 195;
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
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync %0, %1;" ::"n"(CONS_BAR), "n"(NC) : "memory"); }
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ uint4 lds128(const unsigned char *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float4 ldcg4(const float *p) {
    return __ldcg(reinterpret_cast<const float4 *>(p));
}


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

// Phase 2 activations (h) as 16-bit fixed point per chunk, X = rint(h * 32512 / max|h|), split
// X = 256 * Xh + Xl into two signed bytes; the codes become signed bytes scaled by a power of
// two (the int4 nibble in the high half of a byte is 16q, an int2 field in the top two bits is
// 64q), so one dp4a takes four products of each part exactly.  Slice word order follows the
// byte extraction below (h_slot).  Returns the two exact integer sums.
template <int FMT> struct Ph2 {
    static constexpr int MUL = FMT == 4 ? 16 : (FMT == 2 ? 64 : 1);  // code byte = MUL * q
    static constexpr int XW8 = Fmt<FMT>::CPC / 4;                    // int8x4 words per chunk and part
    static constexpr int XV8 = XW8 / 4;                              // int4 vectors per chunk and part
};
template <int FMT>
__device__ __forceinline__ void idot4_chunk(const uint4 q, const int *xh, const int *xl, int &sh, int &sl);

template <>
__device__ __forceinline__ void idot4_chunk<4>(const uint4 q, const int *xh, const int *xl, int &sh, int &sl) {
    // word i (codes 8i..8i+7): (w << 4) & 0xF0F0F0F0 holds codes 0,2,4,6, w & 0xF0F0F0F0 codes 1,3,5,7
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    int h0 = 0, h1 = 0, l0 = 0, l1 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int ev = static_cast<int>((w[i] << 4) & 0xF0F0F0F0u);
        const int od = static_cast<int>(w[i] & 0xF0F0F0F0u);
        h0 = __dp4a(ev, xh[2 * i], h0);
        l0 = __dp4a(ev, xl[2 * i], l0);
        h1 = __dp4a(od, xh[2 * i + 1], h1);
        l1 = __dp4a(od, xl[2 * i + 1], l1);
    }
    sh = h0 + h1;
    sl = l0 + l1;
}
template <>
__device__ __forceinline__ void idot4_chunk<8>(const uint4 q, const int *xh, const int *xl, int &sh, int &sl) {
    // signed bytes in natural order
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    int h0 = 0, h1 = 0, l0 = 0, l1 = 0;
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
        h0 = __dp4a(static_cast<int>(w[i]), xh[i], h0);
        l0 = __dp4a(static_cast<int>(w[i]), xl[i], l0);
        h1 = __dp4a(static_cast<int>(w[i + 1]), xh[i + 1], h1);
        l1 = __dp4a(static_cast<int>(w[i + 1]), xl[i + 1], l1);
    }
    sh = h0 + h1;
    sl = l0 + l1;
}
template <>
__device__ __forceinline__ void idot4_chunk<2>(const uint4 q, const int *xh, const int *xl, int &sh, int &sl) {
    // word i (codes 16i..16i+15): (w << (6 - 2k)) & 0xC0C0C0C0 holds codes k, 4+k, 8+k, 12+k
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    int h[2] = {0, 0}, l[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int bb = static_cast<int>((w[i] << (6 - 2 * k)) & 0xC0C0C0C0u);
            h[k & 1] = __dp4a(bb, xh[4 * i + k], h[k & 1]);
            l[k & 1] = __dp4a(bb, xl[4 * i + k], l[k & 1]);
        }
    }
    sh = h[0] + h[1];
    sl = l[0] + l[1];
}

// Position of chunk element j in the chunk's int8x4 slice layout (word, byte), matching
// idot4_chunk.
template <int FMT>
__device__ __forceinline__ void h_slot(int j, int &word, int &byte) {
    if (FMT == 4) {
        const int i = j >> 3, k = j & 7;
        word = 2 * i + (k & 1);
        byte = k >> 1;
    } else if (FMT == 8) {
        word = j >> 2;
        byte = j & 3;
    } else {
        const int i = j >> 4, k = j & 15;
        word = 4 * i + (k & 3);
        byte = k >> 2;
    }
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

constexpr int RMAX_BLOCKS = 8;  // E <= 256 on the fused path
struct RouteSmem {
    double btop1[RMAX_BLOCKS], btop2[RMAX_BLOCKS];
    double cval[RMAX_BLOCKS * 8], cs[RMAX_BLOCKS * 8];  // per block: its K <= 8 best
    int cid[RMAX_BLOCKS * 8];
    double sel_s[32];
    int sel_id[32];
    int out_id[8];
    float out_w[8];
};

// Route token t with four consumer warps (w4 = warp index within the four, barrier id bar).
// Experts are taken in blocks of 32 (one per lane); a group is a whole number of blocks (or
// G = 1).  Per block: the two largest biased scores (group score) and the block's K best experts
// by rank among its 32 lanes; warp w4 handles blocks w4, w4 + 4 together so that their loads,
// sigmoids and shuffles overlap.  Warp 0 then ranks the groups, takes the kept blocks' K best
// (at most 32 candidates, one per lane) and ranks them.  Selections, ties and weights are those
// of the per-token definition (largest biased score, lower id on ties, weights from the
// unbiased scores renormalised in slot order, times routed_scaling).  Writes the token's ids and
// weights into r.
__device__ void route_token(const DecodeParams &p, int t, int w4, int lane, int bar, RouteSmem &r) {
    const int E = p.f.E, K = p.f.K, G = p.G, TG = p.TG;
    const int gs = E / G, nb = E / 32, bpg = gs / 32;
    const bool grouped = G > 1 && TG < G;
    constexpr int BPW = RMAX_BLOCKS / 4;  // blocks per warp
    double c[BPW], s[BPW];
    float lf[BPW], bf[BPW];
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
        const int e = (w4 + 4 * j) * 32 + lane;
        const bool on = w4 + 4 * j < nb;
        lf[j] = on ? __ldcg(p.logits + static_cast<size_t>(t) * E + e) : 0.f;
        bf[j] = on ? __ldg(p.bias + e) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
        s[j] = 1.0 / (1.0 + exp(-static_cast<double>(lf[j])));
        c[j] = s[j] + static_cast<double>(bf[j]);
    }
    if (grouped) {
        double a1[BPW], a2[BPW];
#pragma unroll
        for (int j = 0; j < BPW; ++j) { a1[j] = c[j]; a2[j] = -INFINITY; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int j = 0; j < BPW; ++j) {
                const double b1 = __shfl_xor_sync(FULL, a1[j], o);
                const double b2 = __shfl_xor_sync(FULL, a2[j], o);
                const double n1 = fmax(a1[j], b1);
                const double n2 = fmax(fmin(a1[j], b1), fmax(a2[j], b2));
                a1[j] = n1; a2[j] = n2;
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < BPW; ++j)
                if (w4 + 4 * j < nb) { r.btop1[w4 + 4 * j] = a1[j]; r.btop2[w4 + 4 * j] = a2[j]; }
        }
    }
    int rank[BPW];
#pragma unroll
    for (int j = 0; j < BPW; ++j) rank[j] = 0;
#pragma unroll
    for (int o = 0; o < 32; ++o) {
#pragma unroll
        for (int j = 0; j < BPW; ++j) {
            const double oc = __shfl_sync(FULL, c[j], o);
            rank[j] += (oc > c[j] || (oc == c[j] && o < lane)) ? 1 : 0;  // same block: id order = lane order
        }
    }
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
        const int bk = w4 + 4 * j;
        if (bk < nb && rank[j] < K) {
            r.cval[bk * K + rank[j]] = c[j];
            r.cs[bk * K + rank[j]] = s[j];
            r.cid[bk * K + rank[j]] = bk * 32 + lane;
        }
    }
    named_sync(bar, 128);
    if (w4 != 0) return;
    // kept blocks: all, or those of the TG best groups (group g = lane)
    unsigned kmask;
    if (grouped) {
        double gsc = -INFINITY;
        if (lane < G) {
            double a1 = -INFINITY, a2 = -INFINITY;
            for (int bk = lane * bpg; bk < (lane + 1) * bpg; ++bk) {
                const double v[2] = {r.btop1[bk], r.btop2[bk]};
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    if (v[k] > a1) { a2 = a1; a1 = v[k]; }
                    else if (v[k] > a2) { a2 = v[k]; }
                }
            }
            gsc = a1 + a2;
        }
        int rk = 0;
#pragma unroll
        for (int o = 0; o < 32; ++o) {
            const double og = __shfl_sync(FULL, gsc, o);
            rk += (o < G && (og > gsc || (og == gsc && o < lane))) ? 1 : 0;
        }
        const unsigned gmask = __ballot_sync(FULL, lane < G && rk < TG);
        kmask = __ballot_sync(FULL, lane < nb && ((gmask >> ((lane * 32) / gs)) & 1u));
    } else {
        kmask = __ballot_sync(FULL, lane < nb);
    }
    // candidate of this lane: rank k of the kb-th kept block
    double c2 = -INFINITY, s2 = 0.0;
    int id = 0x7fffffff;
    if (lane < __popc(kmask) * K) {
        const int kb = lane / K, k = lane - kb * K;
        unsigned m = kmask;
        for (int i = 0; i < kb; ++i) m &= m - 1u;  // drop the kb lowest kept blocks
        const int bk = __ffs(m) - 1;
        c2 = r.cval[bk * K + k];
        s2 = r.cs[bk * K + k];
        id = r.cid[bk * K + k];
    }
    int rank2 = 0;
#pragma unroll
    for (int o = 0; o < 32; ++o) {
        const double oc = __shfl_sync(FULL, c2, o);
        const int oi = __shfl_sync(FULL, id, o);
        rank2 += beats(oc, oi, c2, id) ? 1 : 0;
    }
    if (rank2 < K) { r.sel_s[rank2] = s2; r.sel_id[rank2] = id; }
    __syncwarp();
    if (lane < K) {
        double denom = 0.0;
        for (int k = 0; k < K; ++k) denom += r.sel_s[k];
        r.out_id[lane] = r.sel_id[lane];
        r.out_w[lane] = static_cast<float>((r.sel_s[lane] / denom) * p.rsf);
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
template <int FMT, int TMAX, int NJ>
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
    unsigned char *ring = sm + p.off_ring;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    const uint32_t route_bar = bar0 + 8u * (2 * S);  // consumers -> producer: routing cache ready
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
        mbar_init(route_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- producer --------
        if (lane != 0) return;
        const uint64_t pol = evict_first_policy();
        int seq = 0, U = 0;
        int uniq[32] = {0};
        bool have_routing = false, ok = true;
        auto record = [&](int we) -> const uint8_t * {
            if (we < f.S) return f.shared;
            const int e = uniq[we - f.S];
            return (e >= 0 && e < f.E) ? f.experts + static_cast<size_t>(e) * f.stride : nullptr;
        };
        for (int we = 0; ok; ++we) {
            if (we >= f.S && !have_routing) {
                if (!mbar_wait(route_bar, 0)) { ok = false; break; }
                const int *rtc = reinterpret_cast<const int *>(sm + p.off_route);
                U = rtc[0];
                for (int u = 0; u < U; ++u) uniq[u] = rtc[RT_UNIQ + u];
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
    int *rBeg = rt + RT_BEG;
    int *rCnt = rt + RT_CNT;
    int *rTok = rt + RT_TOK;
    float *rW = reinterpret_cast<float *>(rt + RT_W);
    int *rH = rt + RT_H;
    bool have_routing = false;
    int *rUniq = rt + RT_UNIQ;             // unique expert ids (for the producer)
    RouteSmem *rsm = reinterpret_cast<RouteSmem *>(sm + p.off_x + static_cast<size_t>(T) * f.H * 2);
    int *sorted_slot = rt + RT_SORT;
    auto get_routing = [&]() {
        const int n = T * f.K;
        if (p.route_here) {
            if (ct == 0) {  // every CTA's logits are written
                const long long t0 = clock64();
                while (ld_acquire(p.gbar) < static_cast<unsigned>(G)) {
                    if (clock64() - t0 > WAIT_CYCLES) { atomicOr(f.err, COLI_DEVERR_TIMEOUT); break; }
                }
            }
            cons_sync();
            // every CTA routes the batch from the logits (same code, same inputs, same result)
            if (cw < 4 * T) route_token(p, cw >> 2, cw & 3, lane, 2 + (cw >> 2), rsm[cw >> 2]);
            cons_sync();
            if (cw == 0) {
                // slot s0 = lane: token s0 / K, rank s0 % K; stable sort of the slots by expert id
                const int s0 = lane;
                const int t0 = s0 < n ? s0 / f.K : 0;
                const int id = s0 < n ? rsm[t0].out_id[s0 - t0 * f.K] : 0x7fffffff;
                const float w0 = s0 < n ? rsm[t0].out_w[s0 - t0 * f.K] : 0.f;
                int rk = 0;
#pragma unroll
                for (int o = 0; o < 32; ++o) {
                    const int oid = __shfl_sync(FULL, id, o);
                    rk += ((oid < id) || (oid == id && o < lane)) ? 1 : 0;
                }
                if (s0 < n) sorted_slot[rk] = s0;
                __syncwarp();
                // position `lane` of the grouped order holds slot sl
                const int sl = lane < n ? sorted_slot[lane] : 0;
                const int idr = __shfl_sync(FULL, id, sl);
                const int tr = __shfl_sync(FULL, t0, sl);
                const float wr = __shfl_sync(FULL, w0, sl);
                const int idp = __shfl_up_sync(FULL, idr, 1);
                const bool first = lane < n && (lane == 0 || idp != idr);
                const unsigned m = __ballot_sync(FULL, first);
                const int U = __popc(m);
                const int up = __popc(m & ((1u << lane) - 1u));
                if (first) {
                    const unsigned rest = lane < 31 ? (m >> (lane + 1)) : 0u;
                    const int nxt = rest ? lane + __ffs(rest) : n;
                    rBeg[f.S + up] = lane;
                    rCnt[f.S + up] = nxt - lane;
                    rUniq[up] = idr;
                }
                if (lane < n) {
                    rTok[lane] = tr;
                    rW[lane] = wr;
                    rH[lane] = lane;
                }
                if (lane == 0) *rU = U;
                if (blockIdx.x == 0) {  // the routing outputs of the call
                    if (s0 < n) {
                        p.ids[s0] = id;
                        p.wts[s0] = w0;
                    }
                    if (lane < n) p.f_perm[lane] = sl;
                    if (first) p.f_unique[up] = idr;
                    if (lane == 0) { *p.f_nuniq = U; p.f_offsets[f.E] = n; }
                }
            }
            cons_sync();
            if (blockIdx.x == 0) {
                const int U = *rU;
                for (int e = ct; e < f.E; e += NC) {
                    int c = 0, lt = 0;
                    for (int s2 = 0; s2 < n; ++s2) {
                        const int v = rsm[s2 / f.K].out_id[s2 % f.K];
                        c += v == e;
                        lt += v < e;
                    }
                    p.f_counts[e] = c;
                    p.f_offsets[e] = lt;
                    if (e >= U) p.f_unique[e] = -1;
                }
            }
        } else if (grid_dep_wait(), cw == 0) {  // routing given: lane u handles unique expert u
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
                rUniq[lane] = e;
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
        if (ct == 0) mbar_arrive(route_bar);
        have_routing = true;
    };
    cons_sync();  // activations ready

    // phase 0 (layer calls): this CTA's share of the router gate, logits[t][e] in double from
    // exact double products, then an arrival on the grid counter (the wait comes later, after
    // the shared expert's rows, in get_routing)
    if (p.route_here) {
        const int e0 = static_cast<int>(static_cast<long>(f.E) * b / G), e1 = static_cast<int>(static_cast<long>(f.E) * (b + 1) / G);
        double *gred = reinterpret_cast<double *>(sm + p.off_red);
        for (int job = e0 * T; job < e1 * T; ++job) {
            const int e = job / T, t = job % T;
            const float *wrow = p.Wr + static_cast<size_t>(e) * f.H;
            const uint16_t *xrow = static_cast<const uint16_t *>(f.x) + static_cast<size_t>(t) * f.H;
            double acc = 0.0;
            constexpr int GLD = 3;  // all of a thread's loads in flight together (H <= 3 * 2048)
            float4 wv[GLD];
            uint2 xv[GLD];
#pragma unroll
            for (int g = 0; g < GLD; ++g) {
                const int h0 = ct * 4 + g * NC * 4;
                const bool in = h0 < f.H;
                wv[g] = in ? __ldg(reinterpret_cast<const float4 *>(wrow + h0)) : make_float4(0.f, 0.f, 0.f, 0.f);
                xv[g] = in ? __ldg(reinterpret_cast<const uint2 *>(xrow + h0)) : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int g = 0; g < GLD; ++g) {
                acc = fma(static_cast<double>(wv[g].x), static_cast<double>(__uint_as_float(xv[g].x << 16)), acc);
                acc = fma(static_cast<double>(wv[g].y), static_cast<double>(__uint_as_float(xv[g].x & 0xffff0000u)), acc);
                acc = fma(static_cast<double>(wv[g].z), static_cast<double>(__uint_as_float(xv[g].y << 16)), acc);
                acc = fma(static_cast<double>(wv[g].w), static_cast<double>(__uint_as_float(xv[g].y & 0xffff0000u)), acc);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
            if (lane == 0) gred[cw] = acc;
            cons_sync();
            if (ct == 0) {
                double sum = 0.0;
                for (int w2 = 0; w2 < NCW; ++w2) sum += gred[w2];
                p.logits[static_cast<size_t>(t) * f.E + e] = static_cast<float>(sum);
            }
            cons_sync();
        }
        if (ct == 0) {
            __threadfence();
            atomicAdd(p.gbar, 1u);
        }
    }

    // ------------------------------------------------ phase 1: gate/up, h = SiLU(g)*u -----
    // After a timed-out wait a thread keeps walking the same loops and barriers (skipping later
    // waits), so that no consumer is ever left alone at a named barrier.
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
#pragma unroll
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
        const unsigned target = static_cast<unsigned>(G) * (p.route_here ? 2u : 1u);
        const long long t0 = clock64();
        while (ld_acquire(p.gbar) < target) {
            if (clock64() - t0 > WAIT_CYCLES) { atomicOr(f.err, COLI_DEVERR_TIMEOUT); break; }
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
    // h of one expert's slots is converted once per CTA into 16-bit fixed point per chunk split
    // in two signed bytes (4 elements per thread, chunk maximum over the chunk's lanes), double
    // buffered; the next expert's h is prefetched into registers while the current one is used.
    const int p2 = ct / Li, c2 = ct % Li;
    const int P2 = p.P2;
    const int nwr2 = Li / 32;
    float acc[RPT2MAX][TMAX];
#pragma unroll
    for (int m = 0; m < RPT2MAX; ++m)
#pragma unroll
        for (int q = 0; q < TMAX; ++q) acc[m][q] = 0.f;
    const int nrows = j_hi - j_lo;
    const int a0d = j_lo & ~3;
    const int nwe = f.S + U;
    // buffer layout (int4 vectors): [buf][slot][part hi/lo][XV8][Li]; per (buf, slot, chunk):
    // one float scale
    constexpr int XW8 = Ph2<FMT>::XW8, XV8 = Ph2<FMT>::XV8;
    int4 *hq = reinterpret_cast<int4 *>(sm + p.off_x);
    const size_t hq_buf = static_cast<size_t>(TMAX) * 2 * XV8 * Li;      // int4 per buffer
    float *hsc = reinterpret_cast<float *>(sm + p.off_xs);                // [buf][slot][Li]
    const int ngrp = f.I / 4;                                              // 4-element groups per slot
    float4 pre[TMAX];
    auto fetch_h = [&](int we) {
        const bool shd = we < f.S;
        const int cnt = shd ? T : rCnt[we];
        const int beg = shd ? 0 : rBeg[we];
#pragma unroll
        for (int q = 0; q < TMAX; ++q) {
            if (q < cnt && ct < ngrp) {
                const int hrow = shd ? T * f.K + q : rH[beg + q];
                pre[q] = ldcg4(f.h + static_cast<size_t>(hrow) * f.I + 4 * ct);
            }
        }
    };
    auto convert_h = [&](int we, int buf) {
        const bool shd = we < f.S;
        const int cnt = shd ? T : rCnt[we];
        constexpr int GPC = CPC / 4;          // threads (4 elements each) per chunk
#pragma unroll
        for (int q = 0; q < TMAX; ++q) {
            if (q < cnt) {
                const bool act = ct < ngrp;
                const float v[4] = {pre[q].x, pre[q].y, pre[q].z, pre[q].w};
                float mx = act ? fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))) : 0.f;
#pragma unroll
                for (int o = GPC / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
                const float inv = mx > 0.f ? __fdiv_rn(32512.0f, mx) : 0.f;
                if (act) {
                    const int cc = (4 * ct) / CPC;                          // chunk of these elements
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const int j = (4 * ct + e2) % CPC;
                        const int X = max(-32512, min(32512, __float2int_rn(__fmul_rn(v[e2], inv))));
                        const int xh = (X + 128) >> 8;                      // in [-127, 127]
                        const int xl = X - 256 * xh;                        // in [-128, 127]
                        int word, byte;
                        h_slot<FMT>(j, word, byte);
                        int8_t *ph = reinterpret_cast<int8_t *>(hq + buf * hq_buf + ((static_cast<size_t>(q) * 2 + 0) * XV8 + (word >> 2)) * Li + cc);
                        int8_t *pl = reinterpret_cast<int8_t *>(hq + buf * hq_buf + ((static_cast<size_t>(q) * 2 + 1) * XV8 + (word >> 2)) * Li + cc);
                        ph[4 * (word & 3) + byte] = static_cast<int8_t>(xh);
                        pl[4 * (word & 3) + byte] = static_cast<int8_t>(xl);
                    }
                    if ((ct % GPC) == 0)
                        hsc[(buf * TMAX + q) * Li + cc] = __fdiv_rn(mx, 32512.0f * Ph2<FMT>::MUL);
                }
            }
        }
    };
    if (nwe > 0) {
        fetch_h(0);
        convert_h(0, 0);
    }
    cons_sync();
    for (int we = 0; we < nwe; ++we) {
        const bool shared = we < f.S;
        const int cnt = shared ? T : rCnt[we];
        const int beg = shared ? 0 : rBeg[we];
        const int buf = we & 1;
        if (we + 1 < nwe) fetch_h(we + 1);
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
                int xh[XW8], xl[XW8];
#pragma unroll
                for (int v = 0; v < XV8; ++v) {
                    const int4 a4 = hq[buf * hq_buf + ((static_cast<size_t>(q) * 2 + 0) * XV8 + v) * Li + c2];
                    const int4 b4 = hq[buf * hq_buf + ((static_cast<size_t>(q) * 2 + 1) * XV8 + v) * Li + c2];
                    xh[4 * v] = a4.x; xh[4 * v + 1] = a4.y; xh[4 * v + 2] = a4.z; xh[4 * v + 3] = a4.w;
                    xl[4 * v] = b4.x; xl[4 * v + 1] = b4.y; xl[4 * v + 2] = b4.z; xl[4 * v + 3] = b4.w;
                }
                const float hs = hsc[(buf * TMAX + q) * Li + c2];
#pragma unroll
                for (int m = 0; m < RPT2MAX; ++m) {
                    const int row = p2 + P2 * m;
                    if (row < nrows) {
                        const uint4 qd = lds128(st + static_cast<size_t>(row) * f.rb_i + c2 * 16);
                        int sh, sl;
                        idot4_chunk<FMT>(qd, xh, xl, sh, sl);
                        const float d = __fmul_rn(__fmaf_rn(static_cast<float>(sh), 256.0f, static_cast<float>(sl)), hs);
                        const float wsd = __fmul_rn(wq, sdp[row]);
#pragma unroll
                        for (int t2 = 0; t2 < TMAX; ++t2)
                            if (t2 == tok) acc[m][t2] = __fmaf_rn(d, wsd, acc[m][t2]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
        if (we + 1 < nwe) convert_h(we + 1, buf ^ 1);
        cons_sync();
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

template <int FMT, int TMAX, int NJ>
cudaError_t launch_k2(const DecodeParams &p, size_t smem, cudaStream_t st) {
    auto kern = ffn_decode_kernel<FMT, TMAX, NJ>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<p.grid, NT, smem, st>>>(p);
    return cudaGetLastError();
}

template <int FMT, int NJ>
cudaError_t launch_k2_t(const DecodeParams &p, size_t smem, cudaStream_t st) {
    if (p.f.T <= 1) return launch_k2<FMT, 1, NJ>(p, smem, st);
    if (p.f.T <= 2) return launch_k2<FMT, 2, NJ>(p, smem, st);
    return launch_k2<FMT, 4, NJ>(p, smem, st);
}

// The instantiated (format, chunks per lane) pairs: GLM-5.2 shapes (hidden 6144) in the three
// containers and the OLMoE shape (hidden 2048) in int4.
template <int FMT, int NJ>
static bool fits_block_t(int T) {
    cudaFuncAttributes fa;
    cudaError_t e;
    if (T <= 1) e = cudaFuncGetAttributes(&fa, ffn_decode_kernel<FMT, 1, NJ>);
    else if (T <= 2) e = cudaFuncGetAttributes(&fa, ffn_decode_kernel<FMT, 2, NJ>);
    else e = cudaFuncGetAttributes(&fa, ffn_decode_kernel<FMT, 4, NJ>);
    return e == cudaSuccess && fa.maxThreadsPerBlock >= NT;
}

static bool kernel_fits(int fmt, int nj, int T) {
    if (fmt == 4 && nj == 6) return fits_block_t<4, 6>(T);
    if (fmt == 4 && nj == 2) return fits_block_t<4, 2>(T);
    if (fmt == 8 && nj == 12) return fits_block_t<8, 12>(T);
    if (fmt == 2 && nj == 3) return fits_block_t<2, 3>(T);
    return false;
}

static cudaError_t launch_k2_any(const DecodeParams &p, size_t smem, cudaStream_t st) {
    const int nj = p.Lh / 32;
    if (p.f.fmt == 4 && nj == 6) return launch_k2_t<4, 6>(p, smem, st);
    if (p.f.fmt == 4 && nj == 2) return launch_k2_t<4, 2>(p, smem, st);
    if (p.f.fmt == 8 && nj == 12) return launch_k2_t<8, 12>(p, smem, st);
    if (p.f.fmt == 2 && nj == 3) return launch_k2_t<2, 3>(p, smem, st);
    return cudaErrorInvalidValue;
}

}  // namespace

// Shape rules and the shared-memory plan of the fused decode path.
bool decode_plan(const coli_moe_config &c, int T, DecodePlan *plan) {
    if (T < 1 || T > 4) return false;
    if (c.act != COLI_ACT_BF16) return false;  // 16-bit block fixed point is exact for bf16 only
    if (c.n_experts > 1024 || c.top_k * T > 32 || c.n_group > 32) return false;
    if (c.hidden % 512 || c.hidden > 3 * NC * 4) return false;
    // router blocks of 32 experts: groups are whole blocks, at most 32 candidates, K <= 8
    if (c.n_experts % 32 || c.n_experts > 32 * RMAX_BLOCKS || c.top_k > 8) return false;
    {
        const int gs = c.n_experts / c.n_group;
        const bool grouped = c.n_group > 1 && c.topk_group < c.n_group;
        if (grouped && gs % 32) return false;
        const int kept_blocks = grouped ? c.topk_group * gs / 32 : c.n_experts / 32;
        if (kept_blocks * c.top_k > 32) return false;
    }
    if (c.inter > 4 * NC) return false;  // phase-2 conversion: 4 elements per consumer thread
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
    if (!kernel_fits(c.wfmt, Lh / 32, T)) return false;
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
    const size_t xbytes = static_cast<size_t>(T) * c.hidden * 2 + static_cast<size_t>(T) * sizeof(RouteSmem);
    const size_t hbytes = static_cast<size_t>(2) * tmax * c.inter * 4;  // two buffers of TMAX h rows
    o += ((xbytes > hbytes ? xbytes : hbytes) + 127) / 128 * 128;
    // x scales / corrections (phase 1) or h scales / corrections (phase 2)
    const size_t xsb = static_cast<size_t>(T) * Lh * 4, hsb = static_cast<size_t>(2) * tmax * Li * 4;
    pl.off_xs = o; o += (xsb > hsb ? xsb : hsb);
    pl.off_xc = o; o += (xsb > 2 * hsb ? xsb : 2 * hsb);
    o = (o + 127) / 128 * 128;
    pl.red1_len = 0;
    const int red2_len = P2 * RPT2MAX * tmax * (Li / 32);
    pl.off_red = o; o += (static_cast<size_t>(red2_len) * 4 > NCW * 8 ? static_cast<size_t>(red2_len) * 4 : NCW * 8);
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

cudaError_t launch_ffn_decode(DecodeParams p, const DecodePlan &pl, cudaStream_t st) {
    fill_plan(p, pl);
    return launch_k2_any(p, pl.smem, st);
}

}  // namespace coli
