// ffn_mma.cu -- a4..a7 on the 5th-generation tensor cores for batches with many tokens per
// expert (prefill, long MTP-verify batches).
//
// Batch-union grouped GEMM (colibri-strix README, "What's implemented": batch-union MoE,
// dequant-on-use).  Swap-AB: the 128 weight rows of a tile are the MMA's M dimension and the
// expert's tokens (gathered by the grouping) its N dimension, so one weight tile is read once per
// 128 tokens routed to the expert.
//
//   GEMM1 (per expert, 128 intermediate rows x 128 tokens): D_g = Qg X^T, D_u = Qu X^T in two
//         TMEM accumulators; epilogue h = SiLU(sg * D_g) * (su * D_u), rounded to bf16.
//   GEMM2 (per expert, 128 output rows x 128 tokens): D = Qd H^T; epilogue out[t] += w * sd * D
//         with coalesced float atomics (out starts at zero; the shared expert is one more
//         expert with weight 1).
//
// Codes are dequantised in registers to exact bf16 values (|q| <= 128) and stored into the
// 128-byte-swizzled K-major shared-memory layout the MMA reads; the per-row scales factor out
// of the dot product and are applied in the epilogue.  Products are exact, accumulation is
// float32 in TMEM; the only rounding beyond float32 is h to bf16 before GEMM2.
//
// Pipeline: two shared-memory stages; while the MMAs of k-step k run (issued by one thread,
// completion tracked by tcgen05.commit on a per-stage mbarrier), the CTA dequantises k-step k+1,
// whose global loads were issued one step earlier into registers.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace coli {

namespace {

constexpr int BM = 128;             // weight rows per tile (MMA M)
constexpr int BN = 128;             // tokens per tile (MMA N)
constexpr int BK = 64;              // K per stage: one 128-byte swizzle row of bf16
constexpr int MMA_THREADS = 256;
constexpr long long WAIT_CYCLES = 4000000000LL;
constexpr int TILE_BYTES = BM * BK * 2;  // 16 KB bf16 tile

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count));
}
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(a), "r"(parity), "r"(20000u) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    if (mbar_try(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(a, parity))
        if (clock64() - t0 > WAIT_CYCLES) return false;
    return true;
}
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// ---------------------------------------------------------------- tcgen05 primitives ------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart
// (stride-dimension offset 1024 B), leading-dimension offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major both), float32 D, M = 128, N = BN.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(BM >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, bool accumulate) {
    const uint32_t acc = accumulate ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(IDESC), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------- dequantisation ----------
// Eight int4 codes (one 32-bit word, element k at bits 4k) -> eight exact bf16 values in order.
// With u = q + 8: bf16 bits 0x4300 | u encode 128 + u exactly; subtracting 136 leaves q.
__device__ __forceinline__ uint4 int4x8_to_bf16(uint32_t w) {
    const uint32_t f = w ^ 0x88888888u;
    const uint32_t p0 = (f & 0x0000000Fu) | ((f << 12) & 0x000F0000u) | 0x43004300u;
    const uint32_t p1 = ((f >> 8) & 0x0000000Fu) | ((f << 4) & 0x000F0000u) | 0x43004300u;
    const uint32_t p2 = ((f >> 16) & 0x0000000Fu) | ((f >> 4) & 0x000F0000u) | 0x43004300u;
    const uint32_t p3 = ((f >> 24) & 0x0000000Fu) | ((f >> 12) & 0x000F0000u) | 0x43004300u;
    const __nv_bfloat162 off = __floats2bfloat162_rn(136.0f, 136.0f);
    uint4 r;
    __nv_bfloat162 t;
    t = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&p0), off); r.x = *reinterpret_cast<uint32_t *>(&t);
    t = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&p1), off); r.y = *reinterpret_cast<uint32_t *>(&t);
    t = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&p2), off); r.z = *reinterpret_cast<uint32_t *>(&t);
    t = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&p3), off); r.w = *reinterpret_cast<uint32_t *>(&t);
    return r;
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

struct TileInfo {
    const uint8_t *rec;
    int cnt;   // tokens in the tile
    bool ok;
};

template <int PHASE>
__global__ void __launch_bounds__(MMA_THREADS, 1) mma_ffn_kernel(MmaParams p) {
    constexpr int NA = PHASE == 1 ? 2 : 1;                // A tiles per stage (gate + up, or down)
    constexpr int STAGE = NA * TILE_BYTES + BN * BK * 2;  // A tile(s) + B tile
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t mbar[2];
    __shared__ uint32_t tmem_base;
    __shared__ int s_tok[BN];
    __shared__ float s_w[BN];
    __shared__ int s_hrow[BN];
    const FfnParams &f = p.f;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int y = blockIdx.y;
    if (y >= *p.ntiles) return;
    const int mt = blockIdx.x;
    const int we = p.tile_u[y], n0 = p.tile_n0[y], cnt = p.tile_cnt[y];
    const bool shared = we >= p.n_routed_slots;  // work expert index past the routed ones
    // expert record
    const uint8_t *rec = nullptr;
    int slot_base = 0;
    if (shared) {
        rec = f.shared;
    } else {
        const int e = f.unique[we];
        if (e < 0 || e >= f.E) {
            if (tid == 0) atomicOr(f.err, COLI_DEVERR_EXPERT_ID);
            return;
        }
        rec = f.experts + static_cast<size_t>(e) * f.stride;
        slot_base = f.offsets[e];
    }
    if (tid < BN) {
        int tok = -1, hrow = 0;
        float w = 0.f;
        if (tid < cnt) {
            if (shared) {
                tok = n0 + tid;
                w = 1.0f;
                hrow = f.T * f.K + tok;
            } else {
                const int pos = slot_base + n0 + tid;
                const int s = (pos >= 0 && pos < f.T * f.K) ? f.perm[pos] : -1;
                if (s >= 0 && s < f.T * f.K) {
                    tok = s / f.K;
                    w = f.topk_w[s];
                    hrow = pos;
                } else {
                    atomicOr(f.err, COLI_DEVERR_GROUPING);
                }
            }
        }
        s_tok[tid] = tok;
        s_w[tid] = w;
        s_hrow[tid] = hrow;
    }
    if (warp == 0) tmem_alloc(smem_u32(&tmem_base), NA * BN);
    if (tid == 0) {
        mbar_init(smem_u32(&mbar[0]), 1);
        mbar_init(smem_u32(&mbar[1]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;

    const int K = PHASE == 1 ? f.H : f.I;                 // reduction length
    const size_t rbA = PHASE == 1 ? f.rb_h : f.rb_i;      // bytes per weight row
    const int KT = K / BK;
    // A rows: PHASE 1 thread t -> matrix t / 128 (gate, up), row t % 128, all 64 codes;
    //         PHASE 2 thread t < 128 -> row t.
    const int a_mat = tid / BM, a_row = tid % BM;
    const bool a_act = PHASE == 1 || tid < BM;
    const uint8_t *a_src = rec + (PHASE == 1 ? (a_mat ? f.off_wu : 0) : f.off_wd) +
                           static_cast<size_t>(mt * BM + a_row) * rbA;
    // B rows: thread t -> row t / 2, half t % 2 (32 elements = 64 bytes)
    const int b_row = tid >> 1, b_half = tid & 1;
    const int b_tok = s_tok[b_row];
    const uint16_t *b_src = nullptr;
    if (b_tok >= 0) {
        b_src = PHASE == 1 ? static_cast<const uint16_t *>(f.x) + static_cast<size_t>(b_tok) * f.H
                           : reinterpret_cast<const uint16_t *>(p.hb) + static_cast<size_t>(s_hrow[b_row]) * f.I;
    }
    uint4 ra[2], rb[4];
    auto load_k = [&](int kt) {
        if (a_act) {
            const uint8_t *src = a_src + static_cast<size_t>(kt) * (BK / 2);
            ra[0] = ld_stream(src);
            ra[1] = ld_stream(src + 16);
        }
        if (b_src) {
            const uint4 *src = reinterpret_cast<const uint4 *>(b_src + static_cast<size_t>(kt) * BK + b_half * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) rb[i] = __ldg(src + i);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) rb[i] = make_uint4(0, 0, 0, 0);
        }
    };
    auto store_k = [&](unsigned char *st) {
        if (a_act) {
            unsigned char *at = st + a_mat * TILE_BYTES;
            const uint32_t words[8] = {ra[0].x, ra[0].y, ra[0].z, ra[0].w, ra[1].x, ra[1].y, ra[1].z, ra[1].w};
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(at + sw128(a_row, c)) = int4x8_to_bf16(words[c]);
        }
        unsigned char *bt = st + NA * TILE_BYTES;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4 *>(bt + sw128(b_row, b_half * 4 + i)) = rb[i];
    };

    bool ok = true;
    load_k(0);
    for (int kt = 0; kt < KT; ++kt) {
        const int s = kt & 1;
        unsigned char *st = sm + s * STAGE;
        // the MMAs that last read this stage (k-step kt - 2) must be done before it is rewritten
        if (kt >= 2 && ok && !mbar_wait(smem_u32(&mbar[s]), ((kt - 2) >> 1) & 1)) ok = false;
        store_k(st);
        if (kt + 1 < KT) load_k(kt + 1);
        fence_async_smem();
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(st), b0 = smem_u32(st + NA * TILE_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
                const uint64_t bd = smem_desc(b0 + kk * 32);
                mma_bf16(tbase, smem_desc(a0 + kk * 32), bd, kt > 0 || kk > 0);
                if (PHASE == 1) mma_bf16(tbase + BN, smem_desc(a0 + TILE_BYTES + kk * 32), bd, kt > 0 || kk > 0);
            }
            mma_commit(smem_u32(&mbar[s]));
        }
    }
    // all MMAs are complete once the last commit has arrived
    if (ok && !mbar_wait(smem_u32(&mbar[(KT - 1) & 1]), ((KT - 1) >> 1) & 1)) ok = false;
    tc_fence_after();
    if (!ok) {
        if (tid == 0) atomicOr(f.err, COLI_DEVERR_TIMEOUT);
    } else {
        // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. +31 (its rows), columns
        // [64 * (w / 4), +64) (its tokens)
        const int row = 32 * (warp & 3) + lane;
        const int c0 = 64 * (warp >> 2);
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const int grow = mt * BM + row;  // row of the weight matrix
        if (PHASE == 1) {
            const float sg = reinterpret_cast<const float *>(rec + f.off_sg)[grow];
            const float su = reinterpret_cast<const float *>(rec + f.off_su)[grow];
            __nv_bfloat16 *hb = p.hb;
            for (int cc = 0; cc < 64; cc += 16) {
                float g[16], u[16];
                tmem_ld16(tbase + lane_off + c0 + cc, g);
                tmem_ld16(tbase + lane_off + BN + c0 + cc, u);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int n = c0 + cc + i;
                    if (s_tok[n] >= 0) {
                        const float gg = sg * g[i];
                        const float hv = (gg / (1.0f + expf(-gg))) * (su * u[i]);
                        hb[static_cast<size_t>(s_hrow[n]) * f.I + grow] = __float2bfloat16_rn(hv);
                    }
                }
            }
        } else {
            const float sd = reinterpret_cast<const float *>(rec + f.off_sd)[grow];
            for (int cc = 0; cc < 64; cc += 16) {
                float d[16];
                tmem_ld16(tbase + lane_off + c0 + cc, d);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int n = c0 + cc + i;
                    const int tok = s_tok[n];
                    if (tok >= 0) atomicAdd(f.out + static_cast<size_t>(tok) * f.H + grow, s_w[n] * (sd * d[i]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, NA * BN);
}

// Tile table: one entry per (work expert, block of BN tokens); routed experts first in
// unique-id order, then the shared expert.
__global__ void mma_tiles_kernel(MmaParams p) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const FfnParams &f = p.f;
    int U = *f.n_unique;
    U = U < 0 ? 0 : (U > f.E ? f.E : U);
    int n = 0;
    for (int u = 0; u < U + f.S; ++u) {
        int cnt;
        if (u < U) {
            const int e = f.unique[u];
            cnt = (e >= 0 && e < f.E) ? f.offsets[e + 1] - f.offsets[e] : 0;
            if (cnt < 0) cnt = 0;
        } else {
            cnt = f.T;
        }
        for (int n0 = 0; n0 < cnt && n < p.ntiles_max; n0 += BN, ++n) {
            p.tile_u[n] = u < U ? u : p.n_routed_slots;
            p.tile_n0[n] = n0;
            p.tile_cnt[n] = min(BN, cnt - n0);
        }
    }
    *p.ntiles = n;
}

}  // namespace

int mma_tiles_max(const coli_moe_config &c, int T) {
    const long n = static_cast<long>(T) * c.top_k;
    const long routed = (n + BN - 1) / BN + (n < c.n_experts ? n : c.n_experts);
    const long shared = c.n_shared ? (T + BN - 1) / BN : 0;
    return static_cast<int>(routed + shared);
}

bool mma_shape_ok(const coli_moe_config &c) {
    return c.wfmt == COLI_W_INT4 && c.act == COLI_ACT_BF16 && c.hidden % BM == 0 && c.inter % BM == 0 &&
           c.hidden % BK == 0 && c.inter % BK == 0;
}

cudaError_t launch_ffn_mma(MmaParams p, cudaStream_t st) {
    // the routed experts occupy work-expert indices [0, E); the shared expert is index E
    p.n_routed_slots = p.f.E;
    mma_tiles_kernel<<<1, 32, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(p.f.out, 0, static_cast<size_t>(p.f.T) * p.f.H * sizeof(float), st);
    if (e != cudaSuccess) return e;
    const size_t smem1 = 2 * (2 * TILE_BYTES + BN * BK * 2) + 1024;
    const size_t smem2 = 2 * (1 * TILE_BYTES + BN * BK * 2) + 1024;
    e = cudaFuncSetAttribute(mma_ffn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem1));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(mma_ffn_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem2));
    if (e != cudaSuccess) return e;
    mma_ffn_kernel<1><<<dim3(p.f.I / BM, p.ntiles_max), MMA_THREADS, smem1, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    mma_ffn_kernel<2><<<dim3(p.f.H / BM, p.ntiles_max), MMA_THREADS, smem2, st>>>(p);
    return cudaGetLastError();
}

}  // namespace coli
