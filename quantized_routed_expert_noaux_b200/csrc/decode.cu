// decode.cu -- the fused decode path of the layer for a few tokens (decode and MTP verify).
//
// One persistent cooperative launch, one CTA per SM, one producer warp and 16 consumer warps
// (ffn_decode_kernel):
//
//  start    every consumer thread loads its slice of the activations and of this CTA's router
//           rows at once.  a1 gate: the CTA's logits (experts [b*E/G, (b+1)*E/G)) are summed in
//           double from exact double products and published with an arrival on a grid counter.
//           The activations become 24-bit fixed point per token row (scale 2^(e-22) with
//           max|x| < 2^e), exact for every bf16 element within 2^15 of the row's maximum, held
//           as three signed byte slices in the layout of the tensor-core B operand.
//  routing  every CTA waits for all logits and routes the batch itself (a2, noaux_tc,
//           colibri-strix README "What's implemented") and groups it (a3, batch-union): the
//           same code on the same inputs, so all CTAs agree bit for bit; CTA 0 writes the
//           routing outputs of the call.  (For coli_moe_ffn the routing arrays are inputs.)
//  phase 1  (a4, and a6 for the shared expert) gate/up rows stream through a shared-memory ring
//           (bulk asynchronous copies by the producer warp, mbarrier completion).  A tile is 8
//           gate rows and the same 8 up rows of one expert; two groups of 8 warps take tiles in
//           turn, each warp a slice of K, with int8 tensor-core MMAs (mma.sync m16n8k32,
//           int32 accumulation over all of K: exact) of the unpacked codes against every
//           token's three slices.  A group's partial sums meet in shared memory; one warp
//           forms g and u per (row, token) and writes h = SiLU(g) * u in float32.  The shared
//           expert's tiles, issued at launch, are multiplied right after routing; the routed
//           tiles are dealt over the CTAs as one flat list (tile tau to CTA tau mod G).
//  barrier  bounded grid barrier (every h row complete).
//  convert  each 128-element chunk of every work expert's h is converted once (chunk q by CTA
//           q mod G) into 24-bit fixed point per (chunk, token), three byte slices in the MMA B
//           layout, written to the workspace; a release-add counts it on the expert's
//           readiness counter.
//  phase 2  (a5, a7) each CTA owns H/G output rows of every expert.  A down stage carries the
//           CTA's block of down rows and, once the producer has seen the expert's readiness
//           count complete, the expert's converted h (two bulk copies).  Warp w multiplies its
//           64-byte column chunk of the rows with the chunk's fragments on the tensor cores and
//           accumulates w * sd * dot per (row, token) in float registers over the experts in a
//           fixed order (shared expert first, then the unique ids ascending).  One cross-warp
//           reduction at the end, no atomics: deterministic, and batch-union output equals
//           per-token output bit for bit.
//  counters the workspace header holds a phase word and two counter sets; a call uses the set
//           the phase names, and CTA 0, past the grid barrier, zeroes the other set and flips
//           the phase, so a completed call leaves the header ready for the next one.
//
// Dequantisation (dequant-on-use, same README section): the codes enter the MMA as signed
// bytes scaled by a power of two (the int4 nibble in the high half of a byte is 16q, an int2
// field in the top two bits 64q); the row scale and the activation scale are applied once per
// dot product in the epilogue.
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
constexpr int GW = 8;                // warps of a phase-1 group
constexpr int NGRP = NCW / GW;       // phase-1 groups
constexpr int MAXTOK = 4;            // tokens of the fused path
constexpr int MAXWE = 33;            // work experts: the shared one + up to 32 unique routed
// named barriers: 0 __syncthreads, 1 all consumers, 2.. group full, 4.. group reduction free
constexpr int BAR_CONS = 1, BAR_GFULL = 2, BAR_GFREE = 4;
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
__device__ __forceinline__ void mbar_arrive_cnt(uint32_t a, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
// more bytes expected in the current phase, without an arrival (the arrival comes later)
__device__ __forceinline__ void mbar_add_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
// try_wait with a suspend-time hint (ns): a waiting warp sleeps instead of spinning.
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(a), "r"(parity), "r"(20000u) : "memory");
    return ok != 0;
}
// Bounded wait: false when the bound ran out (the caller records the error and gives up).
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, long long bound) {
    if (mbar_try(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(a, parity)) {
        if (clock64() - t0 > bound) return false;
    }
    return true;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar,
                                         uint64_t policy) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(mbar), "l"(policy) : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t evict_last_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void named_arrive(int id, int n) { asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void cons_sync() { named_sync(BAR_CONS, NC); }
// arrival on a grid counter that publishes every write made before it (by this thread, and by
// the CTA's threads that met it at a barrier just before)
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// orders this thread's generic-proxy global accesses with async-proxy ones (bulk copies)
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// D (16x8 int32) += A (16x32 int8) * B (32x8 int8).  Fragments (thread = 4 * group + tig):
// a0 / a2 row `group`, a1 / a3 row `group + 8`; a0, a1 hold k = 4 tig + j, a2, a3 hold
// k = 16 + 4 tig + j (byte j); b0 / b1 hold the same k of column `group`; d0, d1 row `group`
// columns 2 tig, 2 tig + 1; d2, d3 row `group + 8`.
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------------- code formats ----
// A 64-byte chunk of a row holds CPC codes; each of the 4 threads of a quad loads 16 bytes of
// it and feeds MPC MMAs (k = 32 each).  The codes become signed bytes MUL * q.  Inside a chunk,
// MMA m, thread tig, A register a0 byte j holds code pos0(tig, m, j) and a2 byte j code
// pos0 + OFS2 (the B slices follow the same positions, so the dot products are unchanged).
template <int FMT> struct Fmt;
template <> struct Fmt<4> {
    static constexpr int CPC = 128, MPC = 4, MUL = 16;
    // word m of a thread's 16 bytes holds codes 32 tig + 8 m + (0..7); even codes -> a0, odd -> a2
    __device__ static __forceinline__ void unpack(const uint4 q, int m, uint32_t &lo, uint32_t &hi) {
        const uint32_t w = m == 0 ? q.x : (m == 1 ? q.y : (m == 2 ? q.z : q.w));
        lo = (w << 4) & 0xF0F0F0F0u;
        hi = w & 0xF0F0F0F0u;
    }
    // element p of a chunk -> (tig, m, half, byte)
    __device__ static __forceinline__ void place(int p, int &tig, int &m, int &half, int &byte) {
        tig = p >> 5;
        m = (p >> 3) & 3;
        byte = (p >> 1) & 3;
        half = p & 1;
    }
};
template <> struct Fmt<2> {
    static constexpr int CPC = 256, MPC = 8, MUL = 64;
    // word i of a thread's 16 bytes holds codes 64 tig + 16 i + 4 j + k (byte j, field k); MMA
    // 2i takes fields 0 (a0) and 1 (a2), MMA 2i + 1 fields 2 and 3
    __device__ static __forceinline__ void unpack(const uint4 q, int m, uint32_t &lo, uint32_t &hi) {
        const int i = m >> 1;
        const uint32_t w = i == 0 ? q.x : (i == 1 ? q.y : (i == 2 ? q.z : q.w));
        const int k0 = 2 * (m & 1);
        lo = (w << (6 - 2 * k0)) & 0xC0C0C0C0u;
        hi = (w << (4 - 2 * k0)) & 0xC0C0C0C0u;
    }
    __device__ static __forceinline__ void place(int p, int &tig, int &m, int &half, int &byte) {
        tig = p >> 6;
        const int i = (p >> 4) & 3, k = p & 3;
        m = 2 * i + (k >> 1);
        half = k & 1;
        byte = (p >> 2) & 3;
    }
};

// Byte offset, inside one column's block of a chunk (4 tig x 8 MPC bytes), of B byte `byte` of
// register `half` of MMA m for thread tig.  16-byte units are permuted per column so that the
// 8 threads of a quarter warp (two columns x four tig) read 8 distinct bank groups.
template <int FMT>
__device__ __forceinline__ int b_off(int col, int tig, int m, int half, int byte) {
    constexpr int MPC = Fmt<FMT>::MPC;
    const int u = m >> 1;  // 16-byte unit of the thread's 8 MPC bytes
    int su;
    if (MPC == 4) su = u ^ (col & 1);
    else su = u ^ (tig >> 1) ^ ((col & 1) << 1);
    return tig * 8 * MPC + su * 16 + (m & 1) * 8 + half * 4 + byte;
}
// The thread's B registers of one chunk for MMAs 2u and 2u + 1 (one 16-byte unit): b0, b1 of
// MMA 2u, then b0, b1 of MMA 2u + 1.
template <int FMT>
__device__ __forceinline__ uint4 load_b2(const unsigned char *colblk, int col, int tig, int u) {
    return *reinterpret_cast<const uint4 *>(colblk + b_off<FMT>(col, tig, 2 * u, 0, 0));
}

// Three signed byte slices of a 24-bit fixed-point value: X = 65536 s2 + 256 s1 + s0.
__device__ __forceinline__ void slices3(int X, int &s0, int &s1, int &s2) {
    s0 = static_cast<int>(static_cast<int8_t>(X & 0xff));
    const int r = (X - s0) >> 8;
    s1 = static_cast<int>(static_cast<int8_t>(r & 0xff));
    s2 = (r - s1) >> 8;
}

// ------------------------------------------------------------------------- routing ---------
__device__ __forceinline__ bool beats(double va, int ia, double vb, int ib) {
    return static_cast<bool>(static_cast<int>(va > vb) | (static_cast<int>(va == vb) & static_cast<int>(ia < ib)));
}

constexpr int RMAX_BLOCKS = 8;  // E <= 256 on the fused path: blocks of 32 experts
struct RouteToken {             // per token, shared memory
    double cval[RMAX_BLOCKS][8], cs[RMAX_BLOCKS][8];  // per block: its best max(K, 2) experts
    int cid[RMAX_BLOCKS][8];
    double sel_s[8];
    int sel_id[8];
};
struct RouteCache {             // the routing of the call, shared memory
    int U;                      // unique routed experts
    int uniq[32];               // their ids, ascending
    int slot[MAXWE][MAXTOK];    // h row of (work expert, token), -1 when not routed
    float wgt[MAXWE][MAXTOK];   // combine weight of (work expert, token), 0 when not routed
    int ids[MAXTOK][8];         // per token: selected ids, slot order
    float w[MAXTOK][8];         //            and weights
    int sorted[32];             // grouped order of the slots
    int sid[32], stok[32];      // per grouped position: expert id and token of its slot
    float sw[32];               //                       and its weight
    float xscale[MAXTOK];       // activation scale of each token row, 2^(e - 22)
    int err;
};

// Step A: the best max(K, 2) of one 32-expert block of token t (lane = expert in the block).
// Ranks within a warp come from broadcast reads of the warp's values in shared-memory scratch
// (`scr`, 32 doubles) rather than shuffles.
__device__ void route_block(const DecodeParams &p, int t, int blk, int lane, RouteToken &r, double *scr) {
    const int E = p.f.E, K = p.f.K;
    const int e = blk * 32 + lane;
    const float lf = __ldcg(p.logits + static_cast<size_t>(t) * E + e);
    const float bf = __ldg(p.bias + e);
    const double s = 1.0 / (1.0 + exp(-static_cast<double>(lf)));
    const double c = s + static_cast<double>(bf);
    scr[lane] = c;
    __syncwarp();
    int rank = 0;
#pragma unroll
    for (int o = 0; o < 32; ++o) {
        const double oc = scr[o];
        rank += static_cast<int>(oc > c) | (static_cast<int>(oc == c) & static_cast<int>(o < lane));  // id order = lane order
    }
    __syncwarp();  // the scratch is reused by the warp's next job only after every lane read it
    const int keep = K > 2 ? K : 2;
    if (rank < keep) {
        r.cval[blk][rank] = c;
        r.cs[blk][rank] = s;
        r.cid[blk][rank] = e;
    }
}

// Step B: group stage, selection and weights of token t (one warp).  Selections, ties and
// weights are those of the per-token definition: largest biased score first, lower id on
// ties; groups score the sum of their two largest biased scores, lower group on ties; weights
// from the unbiased scores renormalised in slot order, times routed_scaling.
__device__ void route_select(const DecodeParams &p, int t, int lane, RouteToken &r, RouteCache &rc, double *scr) {
    const int E = p.f.E, K = p.f.K, G = p.G, TG = p.TG;
    const int nb = E / 32;
    const bool grouped = G > 1 && TG < G;
    unsigned kmask;
    if (grouped) {
        const int bpg = (E / G) / 32;
        double gsc = -INFINITY;
        if (lane < G) {
            double a1 = -INFINITY, a2 = -INFINITY;
            for (int bk = lane * bpg; bk < (lane + 1) * bpg; ++bk) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const double v = r.cval[bk][k];
                    if (v > a1) { a2 = a1; a1 = v; }
                    else if (v > a2) { a2 = v; }
                }
            }
            gsc = a1 + a2;
        }
        int rk = 0;
        for (int o = 0; o < G; ++o) {
            const double og = __shfl_sync(FULL, gsc, o);
            rk += static_cast<int>(og > gsc) | (static_cast<int>(og == gsc) & static_cast<int>(o < lane));
        }
        const unsigned gmask = __ballot_sync(FULL, lane < G && rk < TG);
        kmask = __ballot_sync(FULL, lane < nb && ((gmask >> (lane / bpg)) & 1u));
    } else {
        kmask = nb >= 32 ? FULL : ((1u << nb) - 1u);
    }
    // candidate of this lane: rank k of the kb-th kept block
    double c2 = -INFINITY, s2 = 0.0;
    int id = 0x7fffffff;
    if (lane < __popc(kmask) * K) {
        const int kb = lane / K, k = lane - kb * K;
        unsigned m = kmask;
        for (int i = 0; i < kb; ++i) m &= m - 1u;  // drop the kb lowest kept blocks
        const int bk = __ffs(m) - 1;
        c2 = r.cval[bk][k];
        s2 = r.cs[bk][k];
        id = r.cid[bk][k];
    }
    int *scri = reinterpret_cast<int *>(scr + 32);
    scr[lane] = c2;
    scri[lane] = id;
    __syncwarp();
    int rank2 = 0;
#pragma unroll
    for (int o = 0; o < 32; ++o) rank2 += beats(scr[o], scri[o], c2, id) ? 1 : 0;
    if (rank2 < K) { r.sel_s[rank2] = s2; r.sel_id[rank2] = id; }
    __syncwarp();
    if (lane < K) {
        double denom = 0.0;
        for (int k = 0; k < K; ++k) denom += r.sel_s[k];
        rc.ids[t][lane] = r.sel_id[lane];
        rc.w[t][lane] = static_cast<float>((r.sel_s[lane] / denom) * p.rsf);
    }
}

// The order of a CTA's jobs once the batch is routed, walked identically by the producer and the
// consumers.  Routed tile tau (tau = 0 .. U*NRB - 1; work expert S + tau / NRB, row block
// tau % NRB) belongs to CTA tau mod G, so every CTA takes its tiles of expert 0 first, then of
// expert 1, and so on, and at any moment the CTAs read neighbouring tiles (measured on B200:
// contiguous ranges per CTA are 8% slower at one token and 40% at four).  The down projection of work expert S + u (job kind 2; u = -1 is the
// shared expert) follows the CTA's tiles of every expert up to u + lag.
struct JobIter {
    int j = 0;   // next tile of this CTA
    int u = 0;   // next down projection (-S: the shared expert's)
};
__device__ __forceinline__ int next_job(JobIter &it, int b, int G, int NRB, int U, int S, int lag,
                                        int &we, int &rb) {
    const unsigned tau = static_cast<unsigned>(b) + static_cast<unsigned>(G) * it.j;  // < 2^31
    const bool more = tau < static_cast<unsigned>(U) * static_cast<unsigned>(NRB);
    const int te = more ? static_cast<int>(tau / static_cast<unsigned>(NRB)) : 0x7fffffff;
    if (it.u < U && te > it.u + lag) {
        we = S + it.u;
        ++it.u;
        return 2;
    }
    if (!more) return 0;
    we = S + te;
    rb = static_cast<int>(tau - static_cast<unsigned>(te) * static_cast<unsigned>(NRB));
    ++it.j;
    return 1;
}

// ------------------------------------------------------------------------- the kernel ------
// Shared-memory regions (byte offsets from the plan): barriers | routing cache | per-token
// routing scratch | gate partials | group reduction buffers | activation slices (phase 1)
// aliased with the h slices and the final reduction (phase 2) | ring.
// Ring stages: phase 1 holds one tile (8 gate rows | the same 8 up rows | their scales), each
// matrix's rows one contiguous copy; phase 2 holds the CTA's block of down rows of one expert
// (one contiguous copy) and their scales.  Few large copies: a single producer thread issues
// them at a rate far below that of the TMA engine's data path.
template <int FMT, int TT, int GS>
__global__ void __launch_bounds__(NT, 1) ffn_decode_kernel(DecodeParams p) {
    using F = Fmt<FMT>;
    constexpr int CPC = F::CPC, MPC = F::MPC;
    constexpr int MAXT = TT;                          // tokens of this instantiation (T <= TT)
    constexpr int NB = (3 * TT + 7) / 8;              // 8-column MMA blocks (3 slices per token)
    constexpr int EG = FMT == 4 ? 8 : 16;             // activations converted together (whole B words)
    extern __shared__ __align__(1024) unsigned char sm[];
    const FfnParams &f = p.f;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, b = blockIdx.x;
    const int T = f.T, S = p.S;
    const long long bound = p.wait_cycles;
    // This call's counter set (the previous call left it zero and flipped the phase to it)
    const unsigned phase = __ldcg(p.phase) & 1u;
    unsigned *const gbar = p.gbar + 8 * phase;         // logits and grid-barrier arrivals
    unsigned *const ready = p.ready + 40 * phase;      // converted h chunks per work expert
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm);
    RouteCache &rc = *reinterpret_cast<RouteCache *>(sm + p.off_route);
    RouteToken *rtok = reinterpret_cast<RouteToken *>(sm + p.off_rtok);
    unsigned char *xb = sm + p.off_x;                  // activation slices, B layout
    int4 *red1 = reinterpret_cast<int4 *>(sm + p.off_red1);
    double *gpart = reinterpret_cast<double *>(sm + p.off_gate);
    float *xmax = reinterpret_cast<float *>(gpart + NCW * 2 * MAXTOK);  // [NCW][MAXTOK]
    unsigned char *ring = sm + p.off_ring;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    const uint32_t route_bar = bar0 + 8u * (2 * S);  // consumers -> producer: routing cache ready

    // geometry
    const int rb_h = static_cast<int>(f.rb_h), rb_i = static_cast<int>(f.rb_i);
    const int NRB = f.I / 8;                           // tiles (8 row pairs) per expert
    const int j_lo = static_cast<int>(static_cast<long>(f.H) * b / G), j_hi = static_cast<int>(static_cast<long>(f.H) * (b + 1) / G);
    const int nrows = j_hi - j_lo;
    const int a0d = j_lo & ~3;
    const int sh_lo = f.S ? static_cast<int>(static_cast<long>(NRB) * b / G) : 0;
    const int sh_hi = f.S ? static_cast<int>(static_cast<long>(NRB) * (b + 1) / G) : 0;
    const int nsh = sh_hi - sh_lo;                     // shared-expert tiles of this CTA
    const int sc1 = GS ? 8 * f.nsh * 4 : 32;           // bytes of one matrix's scales in a tile stage
    // converted h: per (work expert, chunk of K) the chunk's B block (3 T columns of 32 MPC bytes)
    // and the tokens' 4 scales; a down job's fragments are its expert's nch chunks, contiguous
    const int nch = rb_i / 64;
    const int fch = 3 * T * 32 * MPC + 16;
    unsigned char *frag = sm + p.off_frag;             // S slots of fslot bytes, one per ring stage

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), NCW);  // phase 1: 8 warps x 2; phase 2: the active warps
        }
        mbar_init(route_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- producer --------
        if (lane != 0) return;
        const uint64_t pol = evict_first_policy();
        const uint64_t keep = evict_last_policy();
        int seq = 0, U = 0;
        bool ok = true;
        auto record = [&](int we) -> const uint8_t * {
            if (we < f.S) return f.shared;
            const int e = rc.uniq[we - f.S];
            return (e >= 0 && e < f.E) ? f.experts + static_cast<size_t>(e) * f.stride : nullptr;
        };
        auto stage1 = [&](const uint8_t *rec, int rb) {
            const int r0 = rb * 8;
            const int s = seq % S;
            const uint32_t par = (seq / S) & 1;
            if (!mbar_wait(empty_bar(s), par ^ 1, bound)) { ok = false; return; }
            ++seq;  // counts filled stages only (the drain waits for the last fill of each slot)
            if (rec == nullptr) { mbar_arrive(full_bar(s)); return; }
            const uint32_t dst = smem_u32(ring + static_cast<size_t>(s) * p.SB);
            mbar_expect_tx(full_bar(s), 16u * rb_h + 2u * sc1);
            const size_t so = GS ? static_cast<size_t>(r0) * f.nsh * 4 : static_cast<size_t>(4 * r0);
            bulk_g2s(dst, rec + static_cast<size_t>(r0) * rb_h, 8 * rb_h, full_bar(s), pol);
            bulk_g2s(dst + 8 * rb_h, rec + f.off_wu + static_cast<size_t>(r0) * rb_h, 8 * rb_h, full_bar(s), pol);
            bulk_g2s(dst + 16 * rb_h, rec + f.off_sg + so, sc1, full_bar(s), pol);
            bulk_g2s(dst + 16 * rb_h + sc1, rec + f.off_su + so, sc1, full_bar(s), pol);
        };
        // phase 1: the shared expert's tiles, then (once routed) the flat list of routed tiles
        for (int l = 0; l < nsh && ok; ++l) stage1(f.shared, sh_lo + l);
        if (f.S && ok)  // the shared expert's down rows go to L2 while the batch is routed
            bulk_prefetch_l2(f.shared + f.off_wd + static_cast<size_t>(j_lo) * rb_i, static_cast<uint32_t>(nrows) * rb_i);
        if (ok && !mbar_wait(route_bar, 0, bound)) ok = false;
        if (ok) U = rc.U;
        // a down-projection stage: the CTA's block of one work expert's down rows and their scales
        const int a1 = (j_hi + 3) & ~3;
        const uint32_t sdb = GS ? static_cast<uint32_t>(nrows) * f.nsi * 4 : 4u * (a1 - a0d);
        // A down stage carries the CTA's block of one work expert's down rows and their scales,
        // and in a second part (its fragment slot) the expert's converted h.  Stages issued before
        // the expert's chunks are all converted (counted on its readiness counter) expect the
        // rows' bytes only; their fragments and the arrival follow once this thread has seen the
        // count complete.
        const uint32_t fbytes = static_cast<uint32_t>(nch * fch);
        auto frag_copy = [&](int we, int s) {
            bulk_g2s(smem_u32(frag + static_cast<size_t>(s) * p.fslot),
                     reinterpret_cast<const unsigned char *>(p.dsl) + static_cast<size_t>(we) * DEC_CH * fch, fbytes, full_bar(s), keep);
        };
        auto converted = [&](int we) {  // bounded wait until every chunk of we is converted
            const long long t0 = clock64();
            while (ld_acquire(ready + we) < static_cast<unsigned>(nch)) {
                if (clock64() - t0 > bound) { ok = false; break; }
            }
            fence_proxy_async_global();  // the converters' generic stores, before the bulk copy
            return ok;
        };
        bool published = false;
        int seq0 = -1, npend = 0;
        auto publish = [&]() {  // complete the pending stages as their experts' h is converted
            for (int j = 0; j < npend; ++j) {
                const int s = (seq0 + j) % S;
                if (ok && converted(j)) {
                    mbar_expect_tx(full_bar(s), fbytes);
                    frag_copy(j, s);
                } else {
                    mbar_arrive(full_bar(s));
                }
            }
            npend = 0;
            published = true;
        };
        auto stage2 = [&](int we) {
            const uint8_t *rec = record(we);
            if (seq0 < 0) seq0 = seq;
            if (!published && seq - seq0 == S) publish();  // the ring is full of waiting stages
            if (!ok) return;
            const int s = seq % S;
            const uint32_t par = (seq / S) & 1;
            if (!mbar_wait(empty_bar(s), par ^ 1, bound)) { ok = false; return; }
            ++seq;
            const uint32_t rows = rec ? static_cast<uint32_t>(nrows) * rb_i + sdb : 0u;
            if (published && !converted(we)) { mbar_arrive(full_bar(s)); return; }
            if (published) mbar_expect_tx(full_bar(s), rows + fbytes);
            else mbar_add_tx(full_bar(s), rows);
            const uint32_t dst = smem_u32(ring + static_cast<size_t>(s) * p.SB);
            const uint64_t pl = we < f.S ? keep : pol;
            if (rec) {
                bulk_g2s(dst, rec + f.off_wd + static_cast<size_t>(j_lo) * rb_i, static_cast<uint32_t>(nrows) * rb_i, full_bar(s), pl);
                bulk_g2s(dst + p.st_sd, rec + f.off_sd + (GS ? static_cast<size_t>(j_lo) * f.nsi * 4 : static_cast<size_t>(4 * a0d)),
                         sdb, full_bar(s), pl);
            }
            if (published) frag_copy(we, s);
            else ++npend;
        };
        JobIter it;
        it.u = -f.S;
        while (ok) {
            int we = 0, rb = 0;
            const int kind = next_job(it, b, G, NRB, U, f.S, p.lag, we, rb);
            if (kind == 0) break;
            if (kind == 1) stage1(record(we), rb);
            else stage2(we);
        }
        if (ok && !published && npend > 0) publish();
        if (!ok) {  // complete the stages still waiting for an arrival (their copies drain below)
            for (int j = 0; j < npend; ++j) mbar_arrive(full_bar((seq0 + j) % S));
            atomicOr(f.err, COLI_DEVERR_TIMEOUT);
        }
        // Drain: the last fill of every ring slot has landed before this thread (and with it the
        // CTA) exits, also when a wait ran out and the consumers gave up on the stage.
        for (int s = 0; s < S && s < seq; ++s) {
            const int q = s + S * ((seq - 1 - s) / S);  // last sequence number held by slot s
            if (!mbar_wait(full_bar(s), (q / S) & 1, bound)) atomicOr(f.err, COLI_DEVERR_TIMEOUT);
        }
        return;
    }

    // -------------------------------------------------------------------- consumers --------
    const int ct = threadIdx.x - 32;
    const int cw = ct >> 5;
    const int g8 = lane >> 2, tig = lane & 3;
    const int NCOL = 3 * T;
    const int colblk = 4 * 8 * MPC;                   // bytes of one column's block of a chunk
    bool ok = true;

    for (int i = ct; i < MAXWE * MAXTOK; i += NC) {
        (&rc.slot[0][0])[i] = -1;
        (&rc.wgt[0][0])[i] = 0.f;
    }

    // ---- start: activations and the gate ----
    // thread ct owns the groups of EG activations q = ct + NC r of every token
    const int e0 = static_cast<int>(static_cast<long>(f.E) * b / G), e1 = static_cast<int>(static_cast<long>(f.E) * (b + 1) / G);
    const int ne = p.route_here ? e1 - e0 : 0;        // router rows of this CTA (<= 2)
    const int NQ = f.H / EG;
    auto load_x = [&](int t, int q, uint32_t (&w)[EG / 2]) {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(f.x) + static_cast<size_t>(t) * f.H + q * EG);
#pragma unroll
        for (int i = 0; i < EG / 8; ++i) {
            const uint4 v = __ldg(src + i);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    };
    auto bf = [](const uint32_t (&w)[EG / 2], int k) -> float {
        return __uint_as_float((k & 1) ? (w[k >> 1] & 0xffff0000u) : (w[k >> 1] << 16));
    };
    constexpr int RQ = FMT == 4 ? 2 : 1;              // activation groups per thread (NQ <= RQ * NC)
    {
        // every load is issued before any arithmetic: the activations of all tokens and this
        // CTA's router rows, held in registers through the conversion below
        uint32_t xw[MAXT][RQ][EG / 2];
        float wv[2][RQ][EG];
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            const int q = ct + NC * r;
            const bool in = q < NQ;
#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                if (t < T && in) {
                    load_x(t, q, xw[t][r]);
                } else {
#pragma unroll
                    for (int i = 0; i < EG / 2; ++i) xw[t][r][i] = 0u;
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int i = 0; i < EG / 4; ++i) {
                    const float4 v = (j < ne && in) ? __ldg(reinterpret_cast<const float4 *>(p.Wr + static_cast<size_t>(e0 + j) * f.H + q * EG) + i)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                    wv[j][r][4 * i] = v.x; wv[j][r][4 * i + 1] = v.y; wv[j][r][4 * i + 2] = v.z; wv[j][r][4 * i + 3] = v.w;
                }
        }
        // gate partial dot products (exact double products, double sums) and row maxima
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            double a0 = 0.0, a1 = 0.0;
            float mx = 0.f;
#pragma unroll
            for (int r = 0; r < RQ; ++r)
#pragma unroll
                for (int k = 0; k < EG; ++k) {
                    const float xv = bf(xw[t][r], k);
                    mx = fmaxf(mx, fabsf(xv));
                    a0 = fma(static_cast<double>(wv[0][r][k]), static_cast<double>(xv), a0);
                    a1 = fma(static_cast<double>(wv[1][r][k]), static_cast<double>(xv), a1);
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
                a0 += __shfl_xor_sync(FULL, a0, o);
                a1 += __shfl_xor_sync(FULL, a1, o);
            }
            if (lane == 0) {
                xmax[cw * MAXTOK + t] = mx;
                gpart[cw * 2 * MAXTOK + t] = a0;
                gpart[cw * 2 * MAXTOK + MAXTOK + t] = a1;
            }
        }
        cons_sync();
        if (ct < ne * T) {  // one logit per thread of warp 0: the 16 warps' partials in order
            const int j = ct / T, t = ct % T;
            double sum = 0.0;
            for (int w2 = 0; w2 < NCW; ++w2) sum += gpart[w2 * 2 * MAXTOK + j * MAXTOK + t];
            p.logits[static_cast<size_t>(t) * f.E + e0 + j] = static_cast<float>(sum);
            __threadfence();
        }
        if (cw == 0 && p.route_here) {
            __syncwarp();
            if (lane == 0) atomicAdd(gbar, 1u);
        }
        // activation slices: X = rint(x * 2^(22 - e)), max|x| < 2^e, written as whole B words
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            if (t < T) {
                float m = 0.f;
                for (int w2 = 0; w2 < NCW; ++w2) m = fmaxf(m, xmax[w2 * MAXTOK + t]);
                int ex = 0;
                if (m > 0.f) frexpf(m, &ex);
                const float up = ldexpf(1.0f, 22 - ex);
                if (ct == 0) rc.xscale[t] = ldexpf(1.0f, ex - 22);
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    const int q = ct + NC * r;
                    if (q >= NQ) continue;
                    uint32_t sl[3][EG];  // slice bytes of the EG elements
#pragma unroll
                    for (int k = 0; k < EG; ++k) {
                        int s0, s1, s2;
                        slices3(__float2int_rn(bf(xw[t][r], k) * up), s0, s1, s2);
                        sl[0][k] = static_cast<uint32_t>(s0) & 0xffu;
                        sl[1][k] = static_cast<uint32_t>(s1) & 0xffu;
                        sl[2][k] = static_cast<uint32_t>(s2) & 0xffu;
                    }
                    const int h0 = q * EG, kc = h0 / CPC, p0 = h0 % CPC;
#pragma unroll
                    for (int s = 0; s < 3; ++s) {
                        const int col = 3 * t + s;
                        unsigned char *blk = xb + (static_cast<size_t>(kc) * NCOL + col) * colblk;
                        if (FMT == 4) {  // elements p0 + 2j (+1) -> byte j of register half 0 (1)
                            const int tg = p0 >> 5, m2 = (p0 >> 3) & 3;
#pragma unroll
                            for (int hf = 0; hf < 2; ++hf) {
                                const uint32_t word = sl[s][hf] | (sl[s][2 + hf] << 8) | (sl[s][4 + hf] << 16) | (sl[s][6 + hf] << 24);
                                *reinterpret_cast<uint32_t *>(blk + b_off<FMT>(col, tg, m2, hf, 0)) = word;
                            }
                        } else {         // elements p0 + 4j + k -> byte j of field k's register
                            const int tg = p0 >> 6, i4 = (p0 >> 4) & 3;
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint32_t word = sl[s][k] | (sl[s][4 + k] << 8) | (sl[s][8 + k] << 16) | (sl[s][12 + k] << 24);
                                *reinterpret_cast<uint32_t *>(blk + b_off<FMT>(col, tg, 2 * i4 + (k >> 1), k & 1, 0)) = word;
                            }
                        }
                    }
                }
            }
        }
    }
    if (!p.route_here) {
        // routing given (coli_moe_ffn): warp 0, lane u handles unique expert u
        if (cw == 0) {
            int U = __ldcg(f.n_unique);
            U = U < 0 ? 0 : (U > 32 ? 32 : U);
            if (lane < U) {
                const int e = __ldcg(f.unique + lane);
                rc.uniq[lane] = e;
                if (e >= 0 && e < f.E) {
                    const int b0 = __ldcg(f.offsets + e);
                    int c0 = __ldcg(f.offsets + e + 1) - b0;
                    if (b0 < 0 || c0 < 0 || b0 + c0 > T * f.K || c0 > T) { c0 = 0; atomicOr(f.err, COLI_DEVERR_GROUPING); }
                    for (int qq = 0; qq < c0; ++qq) {
                        const int sl = __ldcg(f.perm + b0 + qq);
                        if (sl < 0 || sl >= T * f.K) { atomicOr(f.err, COLI_DEVERR_GROUPING); continue; }
                        const int tok = sl / f.K;
                        rc.slot[f.S + lane][tok] = b0 + qq;
                        rc.wgt[f.S + lane][tok] = __ldcg(f.topk_w + sl);
                    }
                } else {
                    atomicOr(f.err, COLI_DEVERR_EXPERT_ID);
                }
            }
            if (lane == 0) rc.U = U;
        }
    }
    if (f.S && ct < T) {
        rc.slot[0][ct] = T * f.K + ct;
        rc.wgt[0][ct] = 1.0f;
    }
    cons_sync();  // activation slices and (given routing) the routing cache ready

    // ---- routing of the batch by every CTA (layer calls) ----
    auto route_batch = [&]() {
        if (ct == 0) {  // every CTA's logits are written
            const long long t0 = clock64();
            const unsigned target = static_cast<unsigned>(G) + p.gate_extra;
            while (ld_acquire(gbar) < target) {
                if (clock64() - t0 > bound) { atomicOr(f.err, COLI_DEVERR_TIMEOUT); break; }
            }
        }
        cons_sync();
        const int nb = f.E / 32;
        // the group reduction buffers are idle until the first tile: per-warp scratch of 48 doubles
        double *scr = reinterpret_cast<double *>(red1) + cw * 48;
        for (int job = cw; job < T * nb; job += NCW) route_block(p, job / nb, job % nb, lane, rtok[job / nb], scr);
        cons_sync();
        if (cw < T) route_select(p, cw, lane, rtok[cw], rc, scr);
        cons_sync();
        if (cw == 0) {
            // slot s = t K + k; stable sort of the slots by expert id (ranks from broadcast reads
            // of the selected ids: no shuffles, whose cost here varies tenfold with code layout)
            const int n = T * f.K, K = f.K;
            const int t0 = lane < n ? lane / K : 0;
            const int id = lane < n ? rc.ids[t0][lane - t0 * K] : 0x7fffffff;
            const float w0 = lane < n ? rc.w[t0][lane - t0 * K] : 0.f;
            int rk = 0;
#pragma unroll
            for (int t2 = 0; t2 < MAXT; ++t2)
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) {
                    if (t2 < T && k2 < K) {
                        const int oid = rc.ids[t2][k2], o = t2 * K + k2;
                        rk += static_cast<int>(oid < id) | (static_cast<int>(oid == id) & static_cast<int>(o < lane));
                    }
                }
            if (lane < n) {
                rc.sorted[rk] = lane;
                rc.sid[rk] = id;
                rc.stok[rk] = t0;
                rc.sw[rk] = w0;
            }
            __syncwarp();
            const int sl = lane < n ? rc.sorted[lane] : 0;  // position `lane` holds slot sl
            const int idr = lane < n ? rc.sid[lane] : 0x7fffffff;
            const int tr = lane < n ? rc.stok[lane] : 0;
            const float wr = lane < n ? rc.sw[lane] : 0.f;
            const int idp = lane > 0 && lane < n ? rc.sid[lane - 1] : -1;
            const bool first = lane < n && (lane == 0 || idp != idr);
            const unsigned m = __ballot_sync(FULL, first);
            const int U = __popc(m);
            const int u = __popc(m & ((2u << lane) - 1u)) - 1;  // unique index of position lane
            if (first) rc.uniq[u] = idr;
            if (lane < n) {
                if (idr < 0 || idr >= f.E) atomicOr(f.err, COLI_DEVERR_EXPERT_ID);
                rc.slot[f.S + u][tr] = lane;
                rc.wgt[f.S + u][tr] = wr;
            }
            if (lane == 0) rc.U = U;
            if (blockIdx.x == 0) {  // the routing outputs of the call
                if (lane < n) {
                    p.ids[lane] = id;
                    p.wts[lane] = w0;
                    p.f_perm[lane] = sl;
                }
                if (first) p.f_unique[u] = idr;
                if (lane == 0) { *p.f_nuniq = U; p.f_offsets[f.E] = n; }
            }
        }
        cons_sync();
        if (blockIdx.x == 0) {
            const int n = T * f.K, U = rc.U;
            for (int e = ct; e < f.E; e += NC) {
                int c = 0, lt = 0;
                for (int s2 = 0; s2 < n; ++s2) {
                    const int v = rc.ids[s2 / f.K][s2 % f.K];
                    c += v == e;
                    lt += v < e;
                }
                p.f_counts[e] = c;
                p.f_offsets[e] = lt;
                if (e >= U) p.f_unique[e] = -1;
            }
        }
    };

    // One MMA of the chunk's codes against B, into the per-row sum D or, for the group-scaled
    // container, split by group: a thread's codes lie in group tig >> 1 of the 64-byte chunk, so
    // group g's MMA takes the A registers of lanes with tig >> 1 == g and zeros elsewhere.
    auto mma_chunk = [&](int (&D)[4], int (&D1)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                         uint32_t b0, uint32_t b1) {
        if (GS) {
            const bool g1 = (tig >> 1) != 0;
            mma_s8(D, g1 ? 0u : a0, g1 ? 0u : a1, g1 ? 0u : a2, g1 ? 0u : a3, b0, b1);
            mma_s8(D1, g1 ? a0 : 0u, g1 ? a1 : 0u, g1 ? a2 : 0u, g1 ? a3 : 0u, b0, b1);
        } else {
            mma_s8(D, a0, a1, a2, a3, b0, b1);
        }
    };

    // ------------------------------------------------ jobs: gate/up tiles and down projections
    // After a timed-out wait a warp keeps walking the same jobs and barriers (skipping later waits
    // and MMAs), so that no consumer is ever left alone at a named barrier, and releases no more
    // ring stages: the producer then runs out of its own bounded waits, and its drain makes sure
    // no copy is still landing in shared memory when the CTA exits.
    const int grp = cw / GW, wg = cw % GW;
    const int cpw1 = rb_h / 64 / GW;                  // chunks of a row per warp
    // down projection: warp cw owns the 64-byte chunk cw of every down row of the CTA's block
    constexpr int CPL = CPC / 32;                     // h elements per lane of a chunk
    constexpr int RT2 = 3;                            // 16-row tiles of the CTA's output rows
    const int nch2 = rb_i / 64;
    const int nact = nch2 < NCW ? nch2 : NCW;         // warps with a chunk
    const bool active2 = cw < nch2;
    float acc[RT2][NB][4];                            // down-projection sums (zeroed after the tiles)
    int my_tiles = 0;

    // Chunk c (CPC elements) of work expert we's h (all of h is written: after the grid barrier):
    // per token 24-bit fixed point with one scale (three byte slices), each 32-bit word stored
    // straight into the chunk's block in the workspace at its place in the MMA B fragment layout
    // (no shared-memory staging: the fragment slots, which the producer may fill with other
    // experts' converted h at any time after the barrier, share the span that staging would
    // use).  Lane l holds elements l * CPL + k; two neighbouring lanes fill each 32-bit B word
    // (one shuffle).
    auto convert_chunk = [&](int we, int c) {
        unsigned char *const gblk = reinterpret_cast<unsigned char *>(p.dsl) + static_cast<size_t>(we * DEC_CH + c) * fch;
        float hv[MAXT][CPL];
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            const int slot = t < T ? rc.slot[we][t] : -1;
#pragma unroll
            for (int k = 0; k < CPL; k += 4) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (slot >= 0)
                    v = __ldcg(reinterpret_cast<const float4 *>(f.h + static_cast<size_t>(slot) * f.I + c * CPC + lane * CPL + k));
                hv[t][k] = v.x; hv[t][k + 1] = v.y; hv[t][k + 2] = v.z; hv[t][k + 3] = v.w;
            }
        }
        const bool odd = lane & 1;
        const int tg = lane >> 3;
        float scl[MAXT];
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            scl[t] = 0.f;
            if (t >= T) continue;
            float m = 0.f;
#pragma unroll
            for (int k = 0; k < CPL; ++k) m = fmaxf(m, fabsf(hv[t][k]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
            int ex = 0;
            if (m > 0.f) frexpf(m, &ex);
            const float up = ldexpf(1.0f, 22 - ex);
            scl[t] = ldexpf(1.0f, ex - 22);
            uint32_t by[3][CPL];  // slice bytes
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                int s0, s1, s2;
                slices3(__float2int_rn(hv[t][k] * up), s0, s1, s2);
                by[0][k] = static_cast<uint32_t>(s0) & 0xffu;
                by[1][k] = static_cast<uint32_t>(s1) & 0xffu;
                by[2][k] = static_cast<uint32_t>(s2) & 0xffu;
            }
#pragma unroll
            for (int sidx = 0; sidx < 3; ++sidx) {
                const int col = 3 * t + sidx;
                unsigned char *blk = gblk + col * colblk;
                if (FMT == 4) {
                    // elements 4l + {0, 2} -> bytes 2(l&1) + {0, 1} of half 0; 4l + {1, 3} of half 1
                    const uint32_t h0 = by[sidx][0] | (by[sidx][2] << 8), h1 = by[sidx][1] | (by[sidx][3] << 8);
                    const uint32_t got = __shfl_xor_sync(FULL, odd ? h0 : h1, 1);
                    const uint32_t word = odd ? (got | (h1 << 16)) : (h0 | (got << 16));
                    const int m2 = (lane >> 1) & 3;
                    __stcg(reinterpret_cast<unsigned int *>(blk + b_off<FMT>(col, tg, m2, odd ? 1 : 0, 0)), word);
                } else {
                    // elements 8l + kk + {0, 4} -> bytes 2(l&1) + {0, 1} of field kk's register;
                    // the even lane stores fields 0, 1 and the odd lane fields 2, 3
                    const int i4 = (lane >> 1) & 3;
                    uint32_t hw[4];
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) hw[kk] = by[sidx][kk] | (by[sidx][4 + kk] << 8);
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const uint32_t got = __shfl_xor_sync(FULL, odd ? hw[e2] : hw[2 + e2], 1);
                        const int kk = odd ? 2 + e2 : e2;
                        const uint32_t word = odd ? (got | (hw[kk] << 16)) : (hw[kk] | (got << 16));
                        __stcg(reinterpret_cast<unsigned int *>(blk + b_off<FMT>(col, tg, 2 * i4 + (kk >> 1), kk & 1, 0)), word);
                    }
                }
            }
        }
        // then the tokens' scales (16 bytes) after the block
        uint4 *dst = reinterpret_cast<uint4 *>(gblk);
        const int n16 = NCOL * colblk / 16;
        if (lane == 0) {
            float4 sv = make_float4(0.f, 0.f, 0.f, 0.f);
            sv.x = scl[0];
            if (MAXT > 1) sv.y = scl[MAXT > 1 ? 1 : 0];
            if (MAXT > 2) sv.z = scl[MAXT > 2 ? 2 : 0];
            if (MAXT > 3) sv.w = scl[MAXT > 3 ? 3 : 0];
            __stcg(reinterpret_cast<float4 *>(dst + n16), sv);
        }
        fence_proxy_async_global();  // the block is read by the producers' bulk copies
        __syncwarp();  // every lane's stores precede lane 0's release; the block may be reused
        if (lane == 0) red_release_add(ready + we, 1u);  // one more chunk of we converted
    };

    // A gate/up tile (taken by one group of 8 warps): every warp multiplies its chunks of the 8
    // gate and 8 up rows with all tokens' activation slices, the group reduces the partial sums,
    // and its first warp forms and publishes h = SiLU(g)*u of the 8 rows.
    auto gate_up_tile = [&](int we, int rb, int s, uint32_t par) {
        int D[NB][4], D2[NB][4];  // per-row scales: exact int32 sums over all of K (two chains)
        float Dg[NB][4];          // group scales: float sums of (group sum x group scale)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) { D[nb][i] = 0; D2[nb][i] = 0; Dg[nb][i] = 0.f; }
        if (ok && !mbar_wait(full_bar(s), par, bound)) ok = false;
        ok = __all_sync(FULL, ok);  // warp-uniform: the MMAs below need every lane
        const unsigned char *st = ring + static_cast<size_t>(s) * p.SB;
        const float *sgs = reinterpret_cast<const float *>(st + 16 * rb_h);       // gate rows' scales
        const float *sus = reinterpret_cast<const float *>(st + 16 * rb_h + sc1);  // up rows' scales
        if (ok) {
            for (int cc = 0; cc < cpw1; ++cc) {
                const int c = wg * cpw1 + cc;                    // 64-byte chunk of the row
                const uint4 qa = *reinterpret_cast<const uint4 *>(st + g8 * rb_h + 64 * c + 16 * tig);
                const uint4 qb = *reinterpret_cast<const uint4 *>(st + (8 + g8) * rb_h + 64 * c + 16 * tig);
                const unsigned char *xk = xb + static_cast<size_t>(c) * NCOL * colblk;
                int Dc[NB][4], Dc1[NB][4];  // group-scaled container: this chunk's two groups
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int i = 0; i < 4; ++i) { Dc[nb][i] = 0; Dc1[nb][i] = 0; }
#pragma unroll
                for (int u = 0; u < MPC / 2; ++u) {
                    uint4 bv[NB];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        const int col = nb * 8 + g8;
                        bv[nb] = col < NCOL ? load_b2<FMT>(xk + col * colblk, col, tig, u) : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int mm = 0; mm < 2; ++mm) {
                        uint32_t a0, a2, a1, a3;
                        F::unpack(qa, 2 * u + mm, a0, a2);
                        F::unpack(qb, 2 * u + mm, a1, a3);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            if (GS) mma_chunk(Dc[nb], Dc1[nb], a0, a1, a2, a3, mm ? bv[nb].z : bv[nb].x, mm ? bv[nb].w : bv[nb].y);
                            else mma_s8((NB == 1 && mm) ? D2[nb] : D[nb], a0, a1, a2, a3, mm ? bv[nb].z : bv[nb].x, mm ? bv[nb].w : bv[nb].y);
                        }
                    }
                }
                if (GS) {  // groups 2c and 2c + 1 of rows g8 (gate) and g8 + 8 (up)
                    const float ga0 = sgs[g8 * f.nsh + 2 * c], ga1 = sgs[g8 * f.nsh + 2 * c + 1];
                    const float ua0 = sus[g8 * f.nsh + 2 * c], ua1 = sus[g8 * f.nsh + 2 * c + 1];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            Dg[nb][i] = __fmaf_rn(static_cast<float>(Dc1[nb][i]), ga1, __fmaf_rn(static_cast<float>(Dc[nb][i]), ga0, Dg[nb][i]));
                            Dg[nb][2 + i] = __fmaf_rn(static_cast<float>(Dc1[nb][2 + i]), ua1, __fmaf_rn(static_cast<float>(Dc[nb][2 + i]), ua0, Dg[nb][2 + i]));
                        }
                    }
                }
            }
        }
        // group reduction of the partial sums, then one warp forms h
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) D[nb][i] += D2[nb][i];
        if (my_tiles > 0 && wg != 0) named_sync(BAR_GFREE + grp, GW * 32);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
            red1[((grp * GW + wg) * NB + nb) * 32 + lane] =
                GS ? make_int4(__float_as_int(Dg[nb][0]), __float_as_int(Dg[nb][1]), __float_as_int(Dg[nb][2]), __float_as_int(Dg[nb][3]))
                   : make_int4(D[nb][0], D[nb][1], D[nb][2], D[nb][3]);
        named_sync(BAR_GFULL + grp, GW * 32);
        if (wg == 0) {
            const int pr = lane & 7, t = lane >> 3;  // row pair, token
            const int slot = t < T ? rc.slot[we][t] : -1;
            double gsum = 0.0, usum = 0.0;
            if (ok && slot >= 0) {
#pragma unroll
                for (int sidx = 0; sidx < 3; ++sidx) {
                    const int col = 3 * t + sidx, nb = col >> 3, c8 = col & 7;
                    const int ln = pr * 4 + (c8 >> 1), ix = c8 & 1;
                    const double wsl = sidx == 0 ? 1.0 : (sidx == 1 ? 256.0 : 65536.0);
                    if (GS) {  // the partials already carry the weights' group scales
                        float gs = 0.f, us = 0.f;
                        for (int w2 = 0; w2 < GW; ++w2) {
                            const float *v = reinterpret_cast<const float *>(&red1[((grp * GW + w2) * NB + nb) * 32 + ln]);
                            gs = __fadd_rn(gs, v[ix]);
                            us = __fadd_rn(us, v[2 + ix]);
                        }
                        gsum += wsl * gs;
                        usum += wsl * us;
                    } else {   // exact: int32 per slice, combined exactly in double (|sum| < 2^53)
                        int gs = 0, us = 0;
                        for (int w2 = 0; w2 < GW; ++w2) {
                            const int *v = reinterpret_cast<const int *>(&red1[((grp * GW + w2) * NB + nb) * 32 + ln]);
                            gs += v[ix];
                            us += v[2 + ix];
                        }
                        gsum += wsl * gs;
                        usum += wsl * us;
                    }
                }
            }
            __syncwarp();
            named_arrive(BAR_GFREE + grp, GW * 32);  // partials read: the group's next tile may go on
            if (ok && slot >= 0) {
                const double xs = static_cast<double>(rc.xscale[t]) / F::MUL;
                const double gsc = GS ? 1.0 : static_cast<double>(sgs[pr]);
                const double usc = GS ? 1.0 : static_cast<double>(sus[pr]);
                const float gq = static_cast<float>(gsum * xs * gsc);
                const float uq = static_cast<float>(usum * xs * usc);
                f.h[static_cast<size_t>(slot) * f.I + rb * 8 + pr] = __fmul_rn(__fdiv_rn(gq, __fadd_rn(1.0f, expf(-gq))), uq);
            }
        }
        // the stage (rows and scales) is released once the epilogue has read the scales
        __syncwarp();
        if (ok && lane == 0) mbar_arrive_cnt(empty_bar(s), NCW / GW);
        ++my_tiles;
    };

    // The down projection of work expert we for this warp's chunk (all warps): the warp's chunk
    // of h as B fragments and scales (loaded one job ahead), and once the stage has landed the
    // CTA's down rows multiplied with them into the per-row accumulators.
    // B fragments and column factors of job we from the fragment slot of its (landed) stage s
    auto prep_frag = [&](int we, int s, uint32_t (&bfr)[MPC][NB][2], float (&fcol)[NB][2]) {
        if (active2) {
            const unsigned char *fr = frag + static_cast<size_t>(s) * p.fslot + cw * fch;
#pragma unroll
            for (int u = 0; u < MPC / 2; ++u)
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int col = nb * 8 + g8;
                    const uint4 v = col < NCOL ? load_b2<FMT>(fr + col * colblk, col, tig, u) : make_uint4(0u, 0u, 0u, 0u);
                    bfr[2 * u][nb][0] = v.x;
                    bfr[2 * u][nb][1] = v.y;
                    bfr[2 * u + 1][nb][0] = v.z;
                    bfr[2 * u + 1][nb][1] = v.w;
                }
            const float *scl = reinterpret_cast<const float *>(fr + NCOL * colblk);
            // column factor: combine weight x chunk scale x slice weight (powers of two but the weight)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int col = nb * 8 + 2 * tig + i, t = col / 3;
                    const float base = t < T ? rc.wgt[we][t] * scl[t] / F::MUL : 0.f;
                    fcol[nb][i] = base * (col % 3 == 0 ? 1.0f : (col % 3 == 1 ? 256.0f : 65536.0f));
                }
        }
    };
    // The down projection of job we once its stage (rows, scales, fragments) has landed.
    auto down_job = [&](int we, int s, uint32_t par) {
        if (ok && active2 && !mbar_wait(full_bar(s), par, bound)) ok = false;
        ok = __all_sync(FULL, ok);
        if (ok && active2) {
            uint32_t bfr[MPC][NB][2];
            float fcol[NB][2];
            prep_frag(we, s, bfr, fcol);
            const unsigned char *st = ring + static_cast<size_t>(s) * p.SB;
            const float *sdp = reinterpret_cast<const float *>(st + p.st_sd) + (j_lo - a0d);
            const float *sdg = reinterpret_cast<const float *>(st + p.st_sd);  // [nrows][nsi]
            // all row tiles' codes first, then independent MMA chains: per row tile the even and
            // odd k-steps (per-row scales) or the two groups (group scales)
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            uint4 qa[RT2], qb[RT2];
#pragma unroll
            for (int rt = 0; rt < RT2; ++rt) {
                const int ra = rt * 16 + g8, rbw = ra + 8;
                qa[rt] = ra < nrows ? *reinterpret_cast<const uint4 *>(st + ra * rb_i + 64 * cw + 16 * tig) : z;
                qb[rt] = rbw < nrows ? *reinterpret_cast<const uint4 *>(st + rbw * rb_i + 64 * cw + 16 * tig) : z;
            }
            int D[RT2][NB][4], D1[RT2][NB][4];
#pragma unroll
            for (int rt = 0; rt < RT2; ++rt)
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int i = 0; i < 4; ++i) { D[rt][nb][i] = 0; D1[rt][nb][i] = 0; }
#pragma unroll
            for (int m = 0; m < MPC; ++m)
#pragma unroll
                for (int rt = 0; rt < RT2; ++rt) {
                    uint32_t a0, a2, a1, a3;
                    F::unpack(qa[rt], m, a0, a2);
                    F::unpack(qb[rt], m, a1, a3);
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        if (GS) mma_chunk(D[rt][nb], D1[rt][nb], a0, a1, a2, a3, bfr[m][nb][0], bfr[m][nb][1]);
                        else mma_s8((NB == 1 && (m & 1)) ? D1[rt][nb] : D[rt][nb], a0, a1, a2, a3, bfr[m][nb][0], bfr[m][nb][1]);
                    }
                }
#pragma unroll
            for (int rt = 0; rt < RT2; ++rt) {
                const int ra = rt * 16 + g8, rbw = ra + 8;
                float sda, sdb, sda1 = 0.f, sdb1 = 0.f;
                if (GS) {  // groups 2 cw and 2 cw + 1 of rows ra and rbw
                    sda = ra < nrows ? sdg[ra * f.nsi + 2 * cw] : 0.f;
                    sda1 = ra < nrows ? sdg[ra * f.nsi + 2 * cw + 1] : 0.f;
                    sdb = rbw < nrows ? sdg[rbw * f.nsi + 2 * cw] : 0.f;
                    sdb1 = rbw < nrows ? sdg[rbw * f.nsi + 2 * cw + 1] : 0.f;
                } else {
                    sda = ra < nrows ? sdp[ra] : 0.f;
                    sdb = rbw < nrows ? sdp[rbw] : 0.f;
                }
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    if (GS) {
                        acc[rt][nb][0] = __fmaf_rn(static_cast<float>(D[rt][nb][0]), sda * fcol[nb][0], acc[rt][nb][0]);
                        acc[rt][nb][1] = __fmaf_rn(static_cast<float>(D[rt][nb][1]), sda * fcol[nb][1], acc[rt][nb][1]);
                        acc[rt][nb][2] = __fmaf_rn(static_cast<float>(D[rt][nb][2]), sdb * fcol[nb][0], acc[rt][nb][2]);
                        acc[rt][nb][3] = __fmaf_rn(static_cast<float>(D[rt][nb][3]), sdb * fcol[nb][1], acc[rt][nb][3]);
                        acc[rt][nb][0] = __fmaf_rn(static_cast<float>(D1[rt][nb][0]), sda1 * fcol[nb][0], acc[rt][nb][0]);
                        acc[rt][nb][1] = __fmaf_rn(static_cast<float>(D1[rt][nb][1]), sda1 * fcol[nb][1], acc[rt][nb][1]);
                        acc[rt][nb][2] = __fmaf_rn(static_cast<float>(D1[rt][nb][2]), sdb1 * fcol[nb][0], acc[rt][nb][2]);
                        acc[rt][nb][3] = __fmaf_rn(static_cast<float>(D1[rt][nb][3]), sdb1 * fcol[nb][1], acc[rt][nb][3]);
                    } else {  // the two chains' int32 sums add exactly
                        acc[rt][nb][0] = __fmaf_rn(static_cast<float>(D[rt][nb][0] + D1[rt][nb][0]), sda * fcol[nb][0], acc[rt][nb][0]);
                        acc[rt][nb][1] = __fmaf_rn(static_cast<float>(D[rt][nb][1] + D1[rt][nb][1]), sda * fcol[nb][1], acc[rt][nb][1]);
                        acc[rt][nb][2] = __fmaf_rn(static_cast<float>(D[rt][nb][2] + D1[rt][nb][2]), sdb * fcol[nb][0], acc[rt][nb][2]);
                        acc[rt][nb][3] = __fmaf_rn(static_cast<float>(D[rt][nb][3] + D1[rt][nb][3]), sdb * fcol[nb][1], acc[rt][nb][3]);
                    }
                }
            }
        }
        __syncwarp();
        if (ok && active2 && lane == 0) mbar_arrive_cnt(empty_bar(s), NCW / nact);
    };

    // Bounded grid barrier k: the arrivals count on after the logits'.
    auto grid_barrier = [&](unsigned k) {
        cons_sync();
        if (ct == 0) {
            red_release_add(gbar, 1u);
            const unsigned target = static_cast<unsigned>(G) * ((p.route_here ? 1u : 0u) + k) + p.gate_extra;
            const long long t0 = clock64();
            while (ld_acquire(gbar) < target) {
                if (clock64() - t0 > bound) { atomicOr(f.err, COLI_DEVERR_TIMEOUT); break; }
            }
            if (b == 0) {  // every CTA read the phase before arriving: hand the other set to the next call
                unsigned *const ogbar = p.gbar + 8 * (phase ^ 1u);
                unsigned *const oready = p.ready + 40 * (phase ^ 1u);
                *ogbar = 0u;
                for (int i = 0; i < MAXWE; ++i) oready[i] = 0u;
                *p.phase = phase ^ 1u;
            }
        }
        cons_sync();
    };

    // The jobs, in the order next_job gives (the producer walks the same order): the shared
    // expert's tiles of this CTA, the routing, the routed tiles (alternating between the two
    // groups), then the down projections (every warp takes each).
    int seq = 0, lam = 0, kind = 0, we = 0, rb = 0;
    auto tile = [&](int we1, int rb1) {
        const int s = seq % S;
        const uint32_t par = (seq / S) & 1;
        ++seq;
        const bool mine = (lam % NGRP) == grp;
        ++lam;
        if (mine) gate_up_tile(we1, rb1, s, par);
    };
    // the batch is routed first, so the routed tiles start streaming while the shared expert's
    // (already in the ring) are multiplied (measured on B200: 45.5 against 48.0 us at one token)
    if (p.route_here) route_batch();
    if (ct == 0) mbar_arrive(route_bar);
    for (int l = 0; l < nsh; ++l) tile(0, sh_lo + l);
    JobIter it;
    it.u = -f.S;
    while ((kind = next_job(it, b, G, NRB, rc.U, f.S, p.lag, we, rb)) == 1) tile(we, rb);
    if (my_tiles > 0 && wg != 0) named_sync(BAR_GFREE + grp, GW * 32);  // the last arrival

    // Down projections: once every CTA's h is written (grid barrier), each h chunk is converted
    // once (chunk q by CTA q mod G, warp q / G) and counted on its expert's readiness counter;
    // the producer completes each down stage with the expert's converted h once the count is
    // full, and every CTA multiplies its block of down rows with it.
    if (kind == 2) {
        grid_barrier(1u);
        const int nq = (f.S + rc.U) * nch2;
        for (int q = b + G * cw; q < nq; q += G * NCW) convert_chunk(q / nch2, q % nch2);
    }
#pragma unroll
    for (int rt = 0; rt < RT2; ++rt)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[rt][nb][i] = 0.f;
    // The down jobs are the work experts in order (the shared one first).
    if (kind == 2) {
        const int nwe = f.S + rc.U;
        int s = seq % S;
        uint32_t par = (seq / S) & 1;
        for (int we2 = 0; we2 < nwe; ++we2) {
            down_job(we2, s, par);
            if (++s == S) { s = 0; par ^= 1u; }
        }
    }

    if (!ok) atomicOr(f.err, COLI_DEVERR_TIMEOUT);
    // cross-warp reduction (every job is done: the ring is reused)
    cons_sync();
    float *red2 = reinterpret_cast<float *>(ring);  // [warp][rt][nb][lane][4]
    if (active2) {
#pragma unroll
        for (int rt = 0; rt < RT2; ++rt)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                reinterpret_cast<float4 *>(red2)[((cw * RT2 + rt) * NB + nb) * 32 + lane] =
                    make_float4(acc[rt][nb][0], acc[rt][nb][1], acc[rt][nb][2], acc[rt][nb][3]);
    }
    cons_sync();
    for (int fi = ct; fi < nrows * T; fi += NC) {
        const int r = fi / T, t = fi % T;
        const int rt = r >> 4, rr = r & 15, gg = rr & 7, hi = rr >> 3;
        float pv[NCW][3];  // every term first, then the sum in the fixed order
#pragma unroll
        for (int w2 = 0; w2 < NCW; ++w2)
#pragma unroll
            for (int sidx = 0; sidx < 3; ++sidx) {
                const int col = 3 * t + sidx, nb = col >> 3, c8 = col & 7;
                const int ln = gg * 4 + (c8 >> 1), ix = 2 * hi + (c8 & 1);
                pv[w2][sidx] = w2 < nact ? red2[(((w2 * RT2 + rt) * NB + nb) * 32 + ln) * 4 + ix] : 0.f;
            }
        float v = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NCW; ++w2)
#pragma unroll
            for (int sidx = 0; sidx < 3; ++sidx)
                if (w2 < nact) v = __fadd_rn(v, pv[w2][sidx]);
        f.out[static_cast<size_t>(t) * f.H + j_lo + r] = v;
    }
}

template <int FMT, int TT, int GS>
cudaError_t launch_k(const DecodeParams &p, size_t smem, cudaStream_t st) {
    auto kern = ffn_decode_kernel<FMT, TT, GS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // cooperative: the CTAs wait on one another's logits and h tiles, so every CTA must be
    // resident at once; the launch waits for the whole grid to fit (or fails) instead of leaving
    // CTAs spinning for SMs held elsewhere
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int FMT, int GS>
cudaError_t launch_t(const DecodeParams &p, size_t smem, cudaStream_t st) {
    if (p.f.T <= 1) return launch_k<FMT, 1, GS>(p, smem, st);
    if (p.f.T <= 2) return launch_k<FMT, 2, GS>(p, smem, st);
    return launch_k<FMT, 4, GS>(p, smem, st);
}

static cudaError_t launch_any(const DecodeParams &p, size_t smem, cudaStream_t st) {
    if (p.f.fmt == 4 && p.f.group == 64) return launch_t<4, 64>(p, smem, st);
    if (p.f.group) return cudaErrorInvalidValue;
    if (p.f.fmt == 4) return launch_t<4, 0>(p, smem, st);
    if (p.f.fmt == 2) return launch_t<2, 0>(p, smem, st);
    return cudaErrorInvalidValue;
}

}  // namespace

// Shape rules and the shared-memory plan of the fused decode path.
bool decode_plan(const coli_moe_config &c, int T, DecodePlan *plan) {
    if (T < 1 || T > MAXTOK) return false;
    if (c.act != COLI_ACT_BF16) return false;
    if (c.wfmt != COLI_W_INT4 && c.wfmt != COLI_W_INT2) return false;
    const int gsz = c.group_size;                     // 0 or 64 (int4 only)
    if (gsz && (c.wfmt != COLI_W_INT4 || gsz != 64)) return false;
    // router: blocks of 32 experts; groups are whole blocks; at most 32 candidates, K <= 8
    if (c.n_experts % 32 || c.n_experts > 32 * RMAX_BLOCKS || c.top_k > 8 || c.n_group > 32) return false;
    {
        const int epg = c.n_experts / c.n_group;
        const bool grouped = c.n_group > 1 && c.topk_group < c.n_group;
        if (grouped && epg % 32) return false;
        const int kept_blocks = grouped ? c.topk_group * epg / 32 : c.n_experts / 32;
        if (kept_blocks * c.top_k > 32) return false;
    }
    if (c.top_k * T > 32) return false;
    const int bits = c.wfmt;
    const int cpc = bits == 4 ? 128 : 256, eg = bits == 4 ? 8 : 16;
    const int rb_h = c.hidden * bits / 8, rb_i = c.inter * bits / 8;
    // phase 1: each of a group's 8 warps takes whole 64-byte chunks of a row
    if (c.hidden % cpc || c.hidden % eg || rb_h % (GW * 64) || c.inter % 8) return false;
    // phase 2: one 64-byte chunk of the down rows per warp, at most 16
    if (rb_i % 64 || NCW % (rb_i / 64) || c.inter % cpc) return false;
    // activations: at most two groups of eg per consumer thread (int4), one (int2)
    if (c.hidden / eg > (bits == 4 ? 2 : 1) * NC) return false;
    const int sms = device_sm_count();
    const int rows2 = (c.hidden + sms - 1) / sms;
    if (rows2 > 48) return false;
    if ((c.n_experts + sms - 1) / sms > 2) return false;  // at most two router rows per CTA
    const int NB = 3 * T <= 8 ? 1 : 2;
    const int mpc = bits == 4 ? 4 : 8;
    const size_t colblk = 4 * 8 * mpc;
    DecodePlan pl = {};
    pl.grid = sms;
    const int nsh = gsz ? c.hidden / gsz : 1, nsi = gsz ? c.inter / gsz : 1;
    const int sb1 = 16 * rb_h + 2 * (gsz ? 8 * nsh * 4 : 32);          // tile rows + their scales
    pl.st_sd = ((rows2 * rb_i) + 15) / 16 * 16;
    const int sb2 = pl.st_sd + (gsz ? rows2 * nsi * 4 : ((rows2 + 6 + 3) / 4) * 16);
    pl.SB = ((sb1 > sb2 ? sb1 : sb2) + 127) / 128 * 128;
    size_t o = 1024;                                  // mbarriers (up to 60 stages)
    pl.off_route = o; o += (sizeof(RouteCache) + 127) / 128 * 128;
    // One span for what lives in turn: the group reduction buffers and the activation slices
    // (gate/up tiles), then the down stages' fragment slots (one per ring stage).  Then the per-token routing
    // scratch and the gate partials (until the batch is routed), then the ring; the final
    // cross-warp reduction reuses the ring once every stage is consumed.
    const size_t r1bytes = (static_cast<size_t>(NGRP) * GW * NB * 32 * 16 + 127) / 128 * 128;
    const size_t xbytes = static_cast<size_t>(c.hidden / cpc) * 3 * T * colblk;
    const size_t abytes = (xbytes + 127) / 128 * 128;
    pl.fslot = static_cast<int>((static_cast<size_t>(rb_i / 64) * (3 * T * colblk + 16) + 127) / 128 * 128);
    const size_t tbytes = (static_cast<size_t>(T) * sizeof(RouteToken) + 127) / 128 * 128;
    const size_t gbytes = (static_cast<size_t>(NCW) * 2 * MAXTOK * 8 + NCW * MAXTOK * 4 + 127) / 128 * 128;
    const size_t budget = device_smem_optin() - 1024;
    pl.off_red1 = o;
    pl.off_frag = o;
    pl.off_x = o + r1bytes;
    pl.S = 0;
    for (int S = 60; S >= 2; --S) {
        size_t span = r1bytes + abytes;
        const size_t fr = static_cast<size_t>(S) * pl.fslot;
        span = span > fr ? span : fr;
        const size_t ring = o + span + tbytes + gbytes;
        if (ring + static_cast<size_t>(S) * pl.SB <= budget) {
            pl.S = S;
            pl.off_rtok = o + span;
            pl.off_gate = pl.off_rtok + tbytes;
            pl.off_ring = ring;
            break;
        }
    }
    if (pl.S < 2) return false;
    o = pl.off_ring;
    const size_t rbytes = static_cast<size_t>(NCW) * 3 * NB * 32 * 16;
    if (rbytes > static_cast<size_t>(pl.S) * pl.SB) return false;
    // The down projections follow all the CTA's tiles (they need every CTA's h, converted once).
    pl.lag = 1 << 20;
    pl.smem = o + static_cast<size_t>(pl.S) * pl.SB;
    *plan = pl;
    return true;
}

static void fill_plan(DecodeParams &p, const DecodePlan &pl) {
    p.grid = pl.grid; p.S = pl.S; p.SB = pl.SB; p.st_sd = pl.st_sd; p.lag = pl.lag; p.fslot = pl.fslot;
    p.off_route = pl.off_route; p.off_rtok = pl.off_rtok; p.off_gate = pl.off_gate; p.off_red1 = pl.off_red1;
    p.off_x = pl.off_x; p.off_frag = pl.off_frag; p.off_ring = pl.off_ring;
}

cudaError_t launch_ffn_decode(DecodeParams p, const DecodePlan &pl, cudaStream_t st) {
    fill_plan(p, pl);
    if (p.wait_cycles <= 0) p.wait_cycles = WAIT_CYCLES;
    return launch_any(p, pl.smem, st);
}

}  // namespace coli
