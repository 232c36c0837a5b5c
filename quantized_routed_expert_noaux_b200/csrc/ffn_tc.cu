// ffn_tc.cu -- a4..a7 on the 5th-generation tensor cores for batches with many tokens per
// expert (prefill, long verify batches): batch-union grouped GEMMs in exact integer arithmetic.
//
// Batch-union MoE with dequant-on-use (colibri-strix README, "What's implemented"); packed int4
// expert rows with per-row scales (JustVugg/colibri README, expert format).  Swap-AB: 128 weight
// rows of one expert are the MMA's M side and up to 128 of the expert's tokens its N side, so a
// weight tile is fetched once per 128 routed tokens.
//
// Arithmetic
//   weights      int4 code q -> the signed byte 16*q (the nibble in the high half of a byte): exact.
//   activations  each B row (a token's x for gate/up, a slot's h for down) becomes 16-bit fixed
//                point X = rint(v * 32512 / max|v|), split X = 256*Xh + Xl into two signed bytes
//                that are two consecutive B rows, so one MMA yields both partial dot products.
//   MMA          tcgen05.mma kind::i8, int32 accumulators in tensor memory: exact.
//   epilogue     dot = (256*Dh + Dl) * max|v| / (32512*16), times the weight row's scale; SwiGLU
//                (gate/up) or the weighted combine into out with float atomics (down).
// The approximations are the two 16-bit roundings (x, h; 2^-16 of the row maximum) and float32
// epilogue arithmetic.
//
// Two persistent CTAs per SM, warp-specialised, tiles (chunk of <= 96 tokens of one expert x one
// block of weight rows) taken round-robin over all CTAs:
//   warp 8      A producer: per k-block of 128, the packed A tile (128 rows x 64 B, 64-byte
//               swizzle; one 4-D box holds the gate and the up rows) into the A ring, whose stages
//               the converters release as soon as they have read them.
//   warp 10     B producer: the k-block's B rows (boxes of 128/64/32/16 rows of 128 B, 128-byte
//               swizzle) into the B ring, released by the MMAs' completion; one lane per box.
//   warps 0-3   converters: one thread per weight row unpacks its 64 bytes into 128 signed bytes
//               and stores them with tcgen05.st into a TMEM A stage; the MMA reads A from tensor
//               memory, so unpacked weights never pass through shared memory.
//   warp 9      MMA issuer (one elected lane, operands computed warp-uniformly): 4 x tcgen05.mma
//               (K = 32, N <= 192) per k-block into the CTA's TMEM accumulator.
//   warps 4-7   epilogue: tcgen05.ld of the accumulator and the output arithmetic; the tile's
//               per-token scales, tokens and weights are staged in shared memory first.
// TMEM (256 columns per CTA, half of the SM's): the accumulator at columns [0, 192), two 32-column
// A stages at [192, 256).  One accumulator per CTA: while a CTA's epilogue drains it, the SM's
// other CTA keeps the tensor pipe busy (measured on B200 against one CTA per SM with two
// accumulators, eight epilogue warps and deeper rings: 4% faster on the 2048-token Zipf layer
// and on the full-chunk 32-expert layer; the per-k-block cost of one CTA is latency that rings,
// MMA sizes and copy sizes did not move).
// Inside every group of 8 k the order is permuted to (0,2,4,6,1,3,5,7) on both operands: the
// unpacking yields the even and the odd codes of a word as separate words, and the activation
// bytes are written in the same order, so every dot product is unchanged.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace coli {

namespace {

constexpr int KB = 128;                       // k per ring stage
// Tokens per chunk: N = 192 (hi and lo row per token).  (64-token chunks, which leave room for
// eight TMEM A stages instead of four, measured slower on the 2048-token Zipf layer: 2.45 against
// 2.20 ms per step, the extra tiles costing more than the deeper A pipeline saves.)
constexpr int MAXTOK = 96;
constexpr int NA_MAX = 8;                     // A ring stages (at most; per container below)
constexpr int NB = 3;                         // B ring stages
constexpr int B_MAX = 2 * MAXTOK * KB;        // B rows of one stage: 24 KB
constexpr int NBOX = 4;                       // B box heights 16 << i rows
constexpr int W_CONV = 4, W_EPI0 = 4, N_EPI = 4, W_PRODA = 8, W_MMA = 9, W_PRODB = 10;
constexpr int TC_THREADS = 11 * 32;
constexpr int CTAS_PER_SM = 2;
constexpr uint32_t TMEM_COLS = 256;           // per CTA
constexpr uint32_t A_COL0 = 2 * MAXTOK;       // TMEM column of A stage 0
constexpr int NTS = (TMEM_COLS - 2 * MAXTOK) / 32;  // 32-column TMEM A stages after the accumulator
static_assert(NTS >= 2, "no room for TMEM A stages");
static_assert(W_EPI0 % 4 == 0 && N_EPI == 4 && N_EPI * 32 >= MAXTOK, "epilogue warp q reaches TMEM lanes 32q..32q+31");
constexpr long long WAIT_CYCLES = 4000000000LL;  // ~2 s at 1.9 GHz: bound of every wait
constexpr float QMAX = 32512.0f;              // |X| <= 32512 keeps Xh = (X + 128) >> 8 in [-127, 127]
// Weight containers: bytes of one row's k-block (RB), A ring stages (32 KB of A per CTA), the
// code's multiplier (the signed byte the MMA sees is MUL * q: int4 16q, int2 64q, int8 q).
template <int FMT> struct TcFmt;
template <> struct TcFmt<4> { static constexpr int RB = KB / 2, NA = 4; static constexpr float MUL = 16.0f; };
template <> struct TcFmt<8> { static constexpr int RB = KB, NA = 2; static constexpr float MUL = 1.0f; };
template <> struct TcFmt<2> { static constexpr int RB = KB / 4, NA = 8; static constexpr float MUL = 64.0f; };
template <int FMT>
constexpr size_t tc_smem() {
    return static_cast<size_t>(TcFmt<FMT>::NA) * 128 * TcFmt<FMT>::RB + static_cast<size_t>(NB) * B_MAX + 1024;
}
constexpr int EPI_BAR = 1;                    // named barrier of the epilogue warps

// kind::i8 instruction descriptor: D s32 (bits 4-5 = 2), A and B signed 8-bit (bits 7-9, 10-12
// = 1), both K-major, M = 128 (bits 24-28 = M >> 4); N >> 3 goes to bits 17-22.
constexpr uint32_t IDESC_I8 = (2u << 4) | (1u << 7) | (1u << 10) | ((128u >> 4) << 24);

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
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(a), "r"(parity), "r"(20000u) : "memory");
    return ok != 0;
}
// Non-blocking test of a phase.
__device__ __forceinline__ bool mbar_test(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(a), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait; false when the bound ran out or another role has already given up.  A phase
// that has already completed is taken with the non-blocking test.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, volatile int *abort, int *err) {
    if (mbar_test(a, parity)) return true;
    if (*abort) return false;
    if (mbar_try(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(a, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > WAIT_CYCLES) {
            *abort = 1;
            atomicOr(err, COLI_DEVERR_TIMEOUT);
            return false;
        }
    }
    return true;
}
// Wait used only while giving up: bounded, records nothing.
__device__ __forceinline__ void mbar_drain(uint32_t a, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try(a, parity))
        if (clock64() - t0 > WAIT_CYCLES) return;
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *m, int c0, int c1, int c2, int c3,
                                            uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, int c0, int c1, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand with 128-byte swizzle: 8-row groups
// 1024 bytes apart (stride-dimension offset), leading-dimension offset unused (1), version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}
// D[tmem] (+)= A[tmem] * B[smem]^T, kind::i8, M = 128, K = 32.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}
// 32 consecutive 32-bit columns of this thread's TMEM lane, and the wait for their completion in
// the same asm statement: tcgen05.st may read its source registers until tcgen05.wait::st, so
// the compiler must not reuse them before the wait.
__device__ __forceinline__ void tmem_st32_wait(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// 32 consecutive 32-bit columns of this thread's TMEM lane; the wait is in the same asm statement,
// so the destination registers are not read before the load has written them.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, int *v) {
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                   "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = static_cast<int>(r[i]);
}
// Barrier of the epilogue warps that also ORs a predicate over them: every warp takes the same
// decision (used to give up together, so no warp is left waiting at the barrier).
__device__ __forceinline__ bool epi_sync_or(bool pred) {
    uint32_t r;
    asm volatile("{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, %2, %3, p; selp.u32 %0, 1, 0, q; }"
                 : "=r"(r) : "r"(static_cast<uint32_t>(pred)), "n"(EPI_BAR), "n"(N_EPI * 32) : "memory");
    return r != 0;
}

__device__ __forceinline__ int round16(int v) { return (v + 15) & ~15; }
// TMEM column of A stage j: the gaps [2 * MAXTOK, 256) and [256 + 2 * MAXTOK, 512).
__device__ __forceinline__ uint32_t a_col(int j) { return A_COL0 + 32u * static_cast<uint32_t>(j); }
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{ .reg .pred P; elect.sync _|P, 0xffffffff; selp.b32 %0, 1, 0, P; }" : "=r"(pred));
    return pred != 0;
}

// ------------------------------------------------------------------ activation quantisation --
// Position p of every 16 consecutive k holds element ord<FMT>(p): the order in which the
// converters lay out the unpacked weight codes (int4: a word's even codes, then its odd ones;
// int2: codes 0, 4, 8, 12 of a word, then 1, 5, 9, 13, ...; int8: as stored).
template <int FMT>
__device__ __forceinline__ constexpr int ord16(int p) {
    return FMT == 4 ? (p & 8) + 2 * (p & 3) + ((p >> 2) & 1) : (FMT == 2 ? 4 * (p & 3) + (p >> 2) : p);
}
// 16 consecutive values -> 16 hi bytes and 16 lo bytes of X = rint(v * inv), in that order.
template <int FMT>
__device__ __forceinline__ void quant16(const float *v, float inv, uint4 &hi, uint4 &lo) {
    uint32_t h[4] = {0u, 0u, 0u, 0u}, l[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        int x = __float2int_rn(v[ord16<FMT>(p)] * inv);
        x = max(-32512, min(32512, x));
        const int xh = (x + 128) >> 8;
        const int xl = x - 256 * xh;
        h[p >> 2] |= (static_cast<uint32_t>(xh) & 0xFFu) << (8 * (p & 3));
        l[p >> 2] |= (static_cast<uint32_t>(xl) & 0xFFu) << (8 * (p & 3));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <typename In>
__device__ __forceinline__ void load8(const In *row, int j, float *v);
template <>
__device__ __forceinline__ void load8<float>(const float *row, int j, float *v) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(row) + 2 * j);
    const float4 b = __ldg(reinterpret_cast<const float4 *>(row) + 2 * j + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t *row, int j, float *v) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(row) + j);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

struct QuantArgs {
    const void *src;     // x [T][len] (bf16 or f32) or h [slots][len] (f32)
    int len, slots, TK, K;
    const int32_t *perm;     // x only: slot -> (token, k)
    const float *topk_w;     // x only
    int8_t *q;               // [2*slots][len]: hi row, lo row
    float *scale;            // [slots]: max|v| / (32512 * MUL)
    int *tok_of;             // x only: [slots]
    float *w_of;             // x only: [slots]
    int *err;
};

// One warp per slot.  GATHER: the row is x of the slot's token (grouped order of the batch
// union), and the slot's token and combine weight are recorded for the down GEMM.
template <typename In, bool GATHER, int FMT>
__device__ __forceinline__ void quant_slot(const QuantArgs &a, int pos, int lane) {
    const In *row;
    if (GATHER) {
        int tok;
        float w;
        if (pos < a.TK) {
            const int s = a.perm[pos];
            if (s >= 0 && s < a.TK) {
                tok = s / a.K;
                w = a.topk_w[s];
            } else {
                if (lane == 0) atomicOr(a.err, COLI_DEVERR_GROUPING);
                tok = 0;
                w = 0.f;
            }
        } else {
            tok = pos - a.TK;
            w = 1.0f;
        }
        if (lane == 0) {
            a.tok_of[pos] = tok;
            a.w_of[pos] = w;
        }
        row = static_cast<const In *>(a.src) + static_cast<size_t>(tok) * a.len;
    } else {
        row = static_cast<const In *>(a.src) + static_cast<size_t>(pos) * a.len;
    }
    const int n8 = a.len / 8;
    float amax = 0.f;
    for (int j = lane; j < n8; j += 32) {
        float v[8];
        load8<In>(row, j, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float inv = amax > 0.f ? QMAX / amax : 0.f;
    if (lane == 0) a.scale[pos] = amax / (QMAX * TcFmt<FMT>::MUL);
    uint4 *qh = reinterpret_cast<uint4 *>(a.q + static_cast<size_t>(2 * pos) * a.len);
    uint4 *ql = reinterpret_cast<uint4 *>(a.q + static_cast<size_t>(2 * pos + 1) * a.len);
    for (int j = lane; j < n8 / 2; j += 32) {
        float v[16];
        load8<In>(row, 2 * j, v);
        load8<In>(row, 2 * j + 1, v + 8);
        uint4 hi, lo;
        quant16<FMT>(v, inv, hi, lo);
        qh[j] = hi;
        ql[j] = lo;
    }
}

// Chunk table: one entry per (work expert, block of <= 128 tokens), routed experts in unique-id
// order then the shared expert.  Entry = {expert id or -1 (shared), first slot, tokens, 0}.
__device__ void build_chunks(const FfnParams &f, int4 *chunks, int *n_chunks, int max_chunks) {
    __shared__ int s_scan[256];
    __shared__ int s_carry;
    const int tid = threadIdx.x;
    int U = *f.n_unique;
    U = U < 0 ? 0 : (U > f.E ? f.E : U);
    const int W = U + f.S;
    const int TK = f.T * f.K;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base < W; base += 256) {
        const int u = base + tid;
        int e = -1, pos0 = 0, cnt = 0;
        if (u < U) {
            e = f.unique[u];
            if (e >= 0 && e < f.E) {
                pos0 = f.offsets[e];
                cnt = f.offsets[e + 1] - pos0;
                if (pos0 < 0 || cnt < 0 || pos0 + cnt > TK) {
                    atomicOr(f.err, COLI_DEVERR_GROUPING);
                    cnt = 0;
                }
            } else {
                atomicOr(f.err, COLI_DEVERR_EXPERT_ID);
            }
        } else if (u < W) {
            e = -1;
            pos0 = TK;
            cnt = f.T;
        }
        // per-expert dispatch: experts with at most tc_nmin tokens are the GEMV kernels'
        const int nc = cnt > f.tc_nmin ? (cnt + MAXTOK - 1) / MAXTOK : 0;
        s_scan[tid] = nc;
        __syncthreads();
        for (int o = 1; o < 256; o <<= 1) {  // inclusive Hillis-Steele scan
            const int v = tid >= o ? s_scan[tid - o] : 0;
            __syncthreads();
            s_scan[tid] += v;
            __syncthreads();
        }
        int c = s_carry + s_scan[tid] - nc;
        for (int i = 0; i < nc && c < max_chunks; ++i, ++c)
            chunks[c] = make_int4(e, pos0 + i * MAXTOK, min(MAXTOK, cnt - i * MAXTOK), 0);
        __syncthreads();
        if (tid == 255) s_carry += s_scan[255];
        __syncthreads();
    }
    if (tid == 0) *n_chunks = min(s_carry, max_chunks);
}

struct PrepArgs {
    QuantArgs qa;
    FfnParams f;
    int4 *chunks;
    int *n_chunks;
    int max_chunks;
    float4 *out4;        // out, zeroed here (the down GEMM accumulates into it)
    size_t out_n4;
};

// x quantisation in grouped slot order + chunk table (last block) + zeroing of out.
template <typename In, int FMT>
__global__ void __launch_bounds__(256) tc_prep_kernel(const PrepArgs a) {
    const int slot_blocks = (a.qa.slots + 7) / 8;
    const size_t gt = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t nthreads = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t i = gt; i < a.out_n4; i += nthreads) a.out4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (static_cast<int>(blockIdx.x) >= slot_blocks) {
        build_chunks(a.f, a.chunks, a.n_chunks, a.max_chunks);
        return;
    }
    const int pos = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (pos < a.qa.slots) quant_slot<In, true, FMT>(a.qa, pos, threadIdx.x & 31);
}

template <int FMT>
__global__ void __launch_bounds__(256) tc_quant_h_kernel(const QuantArgs a) {
    const int pos = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (pos < a.slots) quant_slot<float, false, FMT>(a, pos, threadIdx.x & 31);
}

struct GemmArgs {
    FfnParams f;
    const int4 *chunks;
    const int *n_chunks;
    int max_chunks;
    const float *bscale;     // per slot B-row scale
    const int *tok_of;
    const float *w_of;
    float *hbuf;             // [slots][I]
};

// Tensor maps of one GEMM: packed weight rows (routed records, shared record) as 4-D byte
// tensors {row bytes, rows, matrices, records}, and the quantised B rows with four box heights.
struct TcMaps {
    CUtensorMap a, as;
    CUtensorMap b[NBOX];
};

// PHASE 1: gate/up.  A = 64 gate rows + the same 64 up rows of one expert (TMEM lanes 32q..32q+15
//          gate rows 16q.., lanes 32q+16.. the matching up rows), B = quantised x; epilogue
//          h = SiLU(g) * u into hbuf (float32).
// PHASE 2: down.  A = 128 rows of Wd, B = quantised h; epilogue out[token] += w * y.
template <int PHASE, int FMT>
__global__ void __launch_bounds__(TC_THREADS, CTAS_PER_SM)
tc_gemm_kernel(const __grid_constant__ TcMaps maps, const GemmArgs p) {
    constexpr int NA = TcFmt<FMT>::NA, RB = TcFmt<FMT>::RB;
    constexpr int A_RAW = 128 * RB;  // A tile of one k-block: 128 rows of RB bytes
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ __align__(8) uint64_t bars[2 * NA_MAX + 2 * NB + 2 * NTS + 3];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float s_bs[2][MAXTOK], s_w[2][MAXTOK];
    __shared__ int s_tk[2][MAXTOK];
    uint64_t *afull = bars, *aempty = afull + NA, *bfull = aempty + NA, *bempty = bfull + NB;
    uint64_t *tfull = bempty + NB, *tempty = tfull + NTS;
    uint64_t *dfull = tempty + NTS, *dempty = dfull + 1, *drain = dempty + 1;
    volatile int *abort = &s_abort;

    const FfnParams &f = p.f;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int MROWS = PHASE == 1 ? 64 : 128;  // weight rows of one matrix per tile
    const int MB = (PHASE == 1 ? f.I : f.H) / MROWS;
    const int KT = (PHASE == 1 ? f.H : f.I) / KB;
    int nch = *p.n_chunks;
    nch = nch < 0 ? 0 : (nch > p.max_chunks ? p.max_chunks : nch);
    const int ntiles = nch * MB;

    if (warp == 0) tmem_alloc(smem_u32(&s_tmem), TMEM_COLS);
    if (threadIdx.x == 32) {
        for (int i = 0; i < NA; ++i) {
            mbar_init(smem_u32(&afull[i]), 1);
            mbar_init(smem_u32(&aempty[i]), W_CONV * 32);
        }
        for (int i = 0; i < NB; ++i) {
            mbar_init(smem_u32(&bfull[i]), 1);
            mbar_init(smem_u32(&bempty[i]), 1);
        }
        for (int i = 0; i < NTS; ++i) {
            mbar_init(smem_u32(&tfull[i]), W_CONV * 32);
            mbar_init(smem_u32(&tempty[i]), 1);
        }
        mbar_init(smem_u32(dfull), 1);
        mbar_init(smem_u32(dempty), N_EPI * 32);
        mbar_init(smem_u32(drain), 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;

    unsigned char *sa = sm;                                        // A ring
    unsigned char *sb = sm + static_cast<size_t>(NA) * A_RAW;      // B ring
    if (warp == W_PRODA || warp == W_PRODB) {
        // ------------------------------------------------------------------ TMA producers
        // A warp, lane 0: the A box.  B warp, lane i < 4: the box of 128 >> i rows when bit 3 - i
        // of nrows/16 is set.
        const bool is_a = warp == W_PRODA;
        const int nst = is_a ? NA : NB;
        uint64_t *fullb = is_a ? afull : bfull, *emptyb = is_a ? aempty : bempty;
        uint32_t it = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int4 c = p.chunks[t / MB];
            const int m = t % MB;
            const int n16 = round16(2 * c.z) / 16;
            const CUtensorMap *ta = c.x >= 0 ? &maps.a : &maps.as;
            const int ez = c.x >= 0 ? c.x : 0;
            for (int kb = 0; kb < KT; ++kb, ++it) {
                const int s = it % nst;
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&emptyb[s]), ((it / nst) & 1) ^ 1, abort, f.err)))
                    goto prod_done;
                const uint32_t fb = smem_u32(&fullb[s]);
                if (lane == 0) mbar_expect_tx(fb, is_a ? A_RAW : n16 * 16 * KB);
                __syncwarp();
                if (is_a) {
                    if (lane == 0) tma_load_4d(smem_u32(sa + s * A_RAW), ta, kb * RB, m * MROWS, 0, ez, fb);
                } else if (lane < NBOX) {
                    const int bit = NBOX - 1 - lane;
                    if ((n16 >> bit) & 1) {
                        const int row0 = 16 * ((n16 >> (bit + 1)) << (bit + 1));  // rows of the larger boxes
                        tma_load_2d(smem_u32(sb + s * B_MAX + row0 * KB), &maps.b[bit], kb * KB, 2 * c.y + row0, fb);
                    }
                }
            }
        }
    prod_done:
        if (*abort && lane == 0) {
            // let the copies already issued land before the CTA's shared memory is released
            for (uint32_t k = it > static_cast<uint32_t>(nst) ? it - nst : 0; k < it; ++k)
                mbar_drain(smem_u32(&fullb[k % nst]), (k / nst) & 1);
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        // the whole warp runs the loop (uniform operands); one elected lane issues
        uint32_t it = 0, tl = 0;
        // B descriptor of stage s, k-step kk: the start-address field (bits 0-13, address >> 4)
        // advances by B_MAX >> 4 per stage and by 2 per 32-byte k-step
        const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sb));
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tl) {
            const int4 c = p.chunks[t / MB];
            const int nrows = round16(2 * c.z);
            const uint32_t idesc = IDESC_I8 | (static_cast<uint32_t>(nrows >> 3) << 17);
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(dempty), (tl & 1) ^ 1, abort, f.err)))
                goto mma_done;
            tc_fence_after();
            const uint32_t dt = tbase;
            for (int kb = 0; kb < KT; ++kb, ++it) {
                const int s = it % NB, ts = it % NTS;
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bfull[s]), (it / NB) & 1, abort, f.err)))
                    goto mma_done;
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&tfull[ts]), (it / NTS) & 1, abort, f.err)))
                    goto mma_done;
                tc_fence_after();
                const uint64_t bd = bdesc0 + static_cast<uint64_t>(s * (B_MAX >> 4));
                const uint32_t a0 = tbase + a_col(ts);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < KB / 32; ++kk)
                        mma_i8(dt, a0 + kk * 8, bd + 2 * kk, idesc, (kb | kk) != 0);
                    mma_commit(smem_u32(&bempty[s]));
                    mma_commit(smem_u32(&tempty[ts]));
                }
                __syncwarp();
            }
            if (elect_one()) mma_commit(smem_u32(dfull));
            __syncwarp();
        }
    mma_done:
        // every MMA issued so far has completed once this commit arrives
        if (elect_one()) mma_commit(smem_u32(drain));
        __syncwarp();
        mbar_drain(smem_u32(drain), 0);
    } else if (warp < W_CONV) {
        // ------------------------------------------------------------------ converters
        const int q = warp;
        const int rho = PHASE == 1 ? (lane < 16 ? 16 * q + lane : 64 + 16 * q + (lane - 16)) : 32 * q + lane;
        // RB-byte swizzle of the A tile: 16-byte chunk c of row r sits at c ^ ((r * RB >> 7) & (RB / 16 - 1))
        const int swz = ((rho * RB) >> 7) & (RB / 16 - 1);
        const uint32_t ta = tbase + (static_cast<uint32_t>(32 * q) << 16);
        uint32_t it = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            for (int kb = 0; kb < KT; ++kb, ++it) {
                const int s = it % NA, ts = it % NTS;
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&afull[s]), (it / NA) & 1, abort, f.err)))
                    goto conv_done;
                const unsigned char *row = sa + s * A_RAW + rho * RB;
                uint4 v[RB / 16];
#pragma unroll
                for (int cch = 0; cch < RB / 16; ++cch) v[cch] = *reinterpret_cast<const uint4 *>(row + ((cch ^ swz) << 4));
                mbar_arrive(smem_u32(&aempty[s]));
                uint32_t o[32];
#pragma unroll
                for (int cch = 0; cch < RB / 16; ++cch) {
                    const uint32_t w4[4] = {v[cch].x, v[cch].y, v[cch].z, v[cch].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (FMT == 8) {         // the codes as they are
                            o[4 * cch + i] = w4[i];
                        } else if (FMT == 4) {  // a word's codes 0,2,4,6 then 1,3,5,7, as 16q
                            o[8 * cch + 2 * i] = (w4[i] << 4) & 0xF0F0F0F0u;
                            o[8 * cch + 2 * i + 1] = w4[i] & 0xF0F0F0F0u;
                        } else {                // codes 0,4,8,12, then 1,5,9,13, ..., as 64q
#pragma unroll
                            for (int j = 0; j < 4; ++j) o[16 * cch + 4 * i + j] = (w4[i] << (6 - 2 * j)) & 0xC0C0C0C0u;
                        }
                    }
                }
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&tempty[ts]), ((it / NTS) & 1) ^ 1, abort, f.err)))
                    goto conv_done;
                tc_fence_after();
                tmem_st32_wait(ta + a_col(ts), o);
                tc_fence_before();
                mbar_arrive(smem_u32(&tfull[ts]));
            }
        }
    conv_done:;
    } else {
        // ------------------------------------------------------------------ epilogue
        const int q = warp - W_EPI0;  // TMEM lane quarter (warp % 4)
        const int et = threadIdx.x - W_EPI0 * 32;  // 0 .. 127 (>= MAXTOK)
        uint32_t tl = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tl) {
            const int4 c = p.chunks[t / MB];
            const int m = t % MB;
            const int n = c.z, pos0 = c.y;
            const int ngrp = (round16(2 * n) + 31) / 32;  // groups of 32 columns = 16 tokens
            const uint8_t *rec = c.x >= 0 ? f.experts + static_cast<size_t>(c.x) * f.stride : f.shared;
            const int pb = tl & 1;
            // per-token data of the tile (double-buffered by tile parity; the barrier below also
            // orders every warp's reads of tile tl - 2 before these writes)
            if (et < n) {
                s_bs[pb][et] = p.bscale[pos0 + et];
                if (PHASE == 2) {
                    s_w[pb][et] = p.w_of[pos0 + et];
                    s_tk[pb][et] = p.tok_of[pos0 + et];
                }
            }
            if (epi_sync_or(*abort != 0)) break;
            // warp-uniform: tcgen05.ld below is a warp-collective instruction
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(dfull), tl & 1, abort, f.err)))
                continue;  // given up: every epilogue warp leaves at the next barrier
            tc_fence_after();
            const uint32_t dt = tbase + (static_cast<uint32_t>(32 * q) << 16);
            if (PHASE == 1) {
                const bool gate = lane < 16;
                const int irow = m * 64 + 16 * q + (lane & 15);
                const float sc = reinterpret_cast<const float *>(rec + (gate ? f.off_sg : f.off_su))[irow];
                for (int g = 0; g < ngrp; ++g) {
                    int v[32];
                    tmem_ld32(dt + 32 * g, v);
                    float d[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        d[j] = sc * fmaf(256.0f, static_cast<float>(v[2 * j]), static_cast<float>(v[2 * j + 1]));
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        // gate lanes keep tokens 0-7 of the group, up lanes tokens 8-15
                        const float keep = gate ? d[i] : d[8 + i];
                        const float other = __shfl_xor_sync(0xffffffffu, gate ? d[8 + i] : d[i], 16);
                        const int j = 16 * g + (gate ? i : 8 + i);
                        if (j < n) {
                            const float bs = s_bs[pb][j];
                            const float gv = (gate ? keep : other) * bs;
                            const float uv = (gate ? other : keep) * bs;
                            p.hbuf[static_cast<size_t>(pos0 + j) * f.I + irow] = gv / (1.0f + expf(-gv)) * uv;
                        }
                    }
                }
            } else {
                const int r = m * 128 + 32 * q + lane;
                const float sd = reinterpret_cast<const float *>(rec + f.off_sd)[r];
                for (int g = 0; g < ngrp; ++g) {
                    int v[32];
                    tmem_ld32(dt + 32 * g, v);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int jj = 16 * g + j;
                        if (jj < n) {
                            const float y = fmaf(256.0f, static_cast<float>(v[2 * j]), static_cast<float>(v[2 * j + 1])) *
                                            (sd * s_bs[pb][jj]);
                            atomicAdd(f.out + static_cast<size_t>(s_tk[pb][jj]) * f.H + r, s_w[pb][jj] * y);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(dempty));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------- host: tensor maps --
// The driver's tensor-map encoder, looked up through the runtime so that the library has no
// link-time dependency on the driver library (it loads on machines without one).
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool encode_u8(CUtensorMap *m, const void *base, cuuint32_t rank, const cuuint64_t *dims,
               const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle sw) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};  // rank <= 5
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed weight rows of a set of records as a 4-D byte tensor {row bytes, rows, matrices,
// records}; the box takes `box_rows` rows of `box_mats` consecutive matrices.
bool weight_map(CUtensorMap *m, const uint8_t *base, size_t row_bytes, size_t rows, size_t mats, size_t nrec,
                size_t rec_stride, cuuint32_t box_rows, cuuint32_t box_mats, int fmt) {
    const cuuint64_t dims[4] = {row_bytes, rows, mats, nrec};
    const cuuint64_t strides[3] = {row_bytes, rows * row_bytes, rec_stride};
    const cuuint32_t rb = static_cast<cuuint32_t>(KB * fmt / 8);  // one k-block of a row: 32/64/128 bytes
    const cuuint32_t box[4] = {rb, box_rows, box_mats, 1};
    const CUtensorMapSwizzle sw = rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : (rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    return encode_u8(m, base, 4, dims, strides, box, sw);
}

// Quantised B rows {len bytes, 2 * slots rows}, boxes of `box_rows` rows.
bool act_map(CUtensorMap *m, const int8_t *base, size_t len, size_t rows, cuuint32_t box_rows) {
    const cuuint64_t dims[2] = {len, rows};
    const cuuint64_t strides[1] = {len};
    const cuuint32_t box[2] = {KB, box_rows};
    return encode_u8(m, base, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool act_maps(TcMaps *m, const int8_t *base, size_t len, size_t rows) {
    for (int i = 0; i < NBOX; ++i)
        if (!act_map(&m->b[i], base, len, rows, 16u << i)) return false;
    return true;
}

}  // namespace

int tc_max_chunks(const coli_moe_config &c, int T) {
    const long n = static_cast<long>(T) * c.top_k;
    const long routed = (n + MAXTOK - 1) / MAXTOK + (n < c.n_experts ? n : c.n_experts);
    const long shared = c.n_shared ? (T + MAXTOK - 1) / MAXTOK : 0;
    return static_cast<int>(routed + shared);
}

bool tc_shape_ok(const coli_moe_config &c) {
    // m-blocks of 64 (gate/up) and 128 (down) rows, k-blocks of 128, int32 accumulators exact
    // for K <= 65536 (|MUL q * X| <= 128 * 128 = 2^14 per product: 16q for int4, 64q for int2,
    // q for int8); per-row scales only: the int32 accumulation runs over all of K
    return (c.wfmt == COLI_W_INT4 || c.wfmt == COLI_W_INT8 || c.wfmt == COLI_W_INT2) && c.group_size == 0 &&
           c.hidden % 128 == 0 && c.inter % 128 == 0 && c.hidden <= 65536 && c.inter <= 65536;
}

namespace {

template <int FMT>
cudaError_t launch_tc_fmt(const FfnParams &f, const TcBuffers &b, cudaStream_t st) {
    const int TK = f.T * f.K;
    const int slots = TK + f.T * f.S;
    cudaError_t e;
    // 1. x quantisation in slot order, chunk table, out = 0
    PrepArgs pa;
    pa.qa.src = f.x;
    pa.qa.len = f.H;
    pa.qa.slots = slots;
    pa.qa.TK = TK;
    pa.qa.K = f.K;
    pa.qa.perm = f.perm;
    pa.qa.topk_w = f.topk_w;
    pa.qa.q = b.xq;
    pa.qa.scale = b.sx;
    pa.qa.tok_of = b.tok_of;
    pa.qa.w_of = b.w_of;
    pa.qa.err = f.err;
    pa.f = f;
    pa.chunks = b.chunks;
    pa.n_chunks = b.n_chunks;
    pa.max_chunks = b.max_chunks;
    pa.out4 = reinterpret_cast<float4 *>(f.out);
    pa.out_n4 = static_cast<size_t>(f.T) * f.H / 4;
    const int prep_blocks = (slots + 7) / 8 + 1;
    if (f.act == COLI_ACT_BF16)
        tc_prep_kernel<uint16_t, FMT><<<prep_blocks, 256, 0, st>>>(pa);
    else
        tc_prep_kernel<float, FMT><<<prep_blocks, 256, 0, st>>>(pa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // tensor maps (host-side encodings of the operands' shapes; no device work)
    TcMaps m1, m2;
    const size_t rbh = f.rb_h, rbi = f.rb_i, I = f.I, H = f.H;
    const size_t rec_bytes = f.off_sd + H * 4;
    const size_t rec_pad = (rec_bytes + 255) & ~static_cast<size_t>(255);
    bool ok = weight_map(&m1.a, f.experts, rbh, I, 2, f.E, f.stride, 64, 2, FMT) &&
              weight_map(&m2.a, f.experts + f.off_wd, rbi, H, 1, f.E, f.stride, 128, 1, FMT) &&
              act_maps(&m1, b.xq, H, 2 * static_cast<size_t>(slots)) &&
              act_maps(&m2, b.hq, I, 2 * static_cast<size_t>(slots));
    if (ok && f.S) {
        ok = weight_map(&m1.as, f.shared, rbh, I, 2, 1, rec_pad, 64, 2, FMT) &&
             weight_map(&m2.as, f.shared + f.off_wd, rbi, H, 1, 1, rec_pad, 128, 1, FMT);
    } else {
        m1.as = m1.a;
        m2.as = m2.a;
    }
    if (!ok) return cudaErrorInvalidValue;

    constexpr size_t TC_SMEM = tc_smem<FMT>();
    e = cudaFuncSetAttribute(tc_gemm_kernel<1, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(TC_SMEM));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_gemm_kernel<2, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(TC_SMEM));
    if (e != cudaSuccess) return e;

    GemmArgs g;
    g.f = f;
    g.chunks = b.chunks;
    g.n_chunks = b.n_chunks;
    g.max_chunks = b.max_chunks;
    g.tok_of = b.tok_of;
    g.w_of = b.w_of;
    g.hbuf = b.hbuf;
    const int grid = CTAS_PER_SM * device_sm_count();

    // 2. gate/up GEMM -> h (float32); the small experts' h by the GEMV kernel
    g.bscale = b.sx;
    tc_gemm_kernel<1, FMT><<<grid, TC_THREADS, TC_SMEM, st>>>(m1, g);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (f.gemv_nmax > 0 && (e = launch_ffn_gemv_gateup(f, st)) != cudaSuccess) return e;

    // 3. h quantisation
    QuantArgs qh = pa.qa;
    qh.src = b.hbuf;
    qh.len = f.I;
    qh.q = b.hq;
    qh.scale = b.sh;
    tc_quant_h_kernel<FMT><<<(slots + 7) / 8, 256, 0, st>>>(qh);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // 4. the small experts' down projections (atomic adds into out, zeroed by the prep kernel),
    //    then the down GEMM + weighted combine into out
    if (f.gemv_nmax > 0 && (e = launch_ffn_gemv_down(f, st)) != cudaSuccess) return e;
    g.bscale = b.sh;
    tc_gemm_kernel<2, FMT><<<grid, TC_THREADS, TC_SMEM, st>>>(m2, g);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_tc(const FfnParams &f, const TcBuffers &b, cudaStream_t st) {
    if (f.fmt == 8) return launch_tc_fmt<8>(f, b, st);
    if (f.fmt == 2) return launch_tc_fmt<2>(f, b, st);
    return launch_tc_fmt<4>(f, b, st);
}

}  // namespace coli
