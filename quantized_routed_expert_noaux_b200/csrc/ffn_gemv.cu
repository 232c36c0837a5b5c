// ffn_gemv.cu -- a4..a7 on CUDA cores for decode-sized batches (few tokens per expert).
//
// The expert half of the layer is bound by HBM bandwidth here: every unique expert's codes
// are streamed once (batch-union, colibri-strix README "What's implemented") and dequantised in
// registers (dequant-on-use, same section).  Layout of the work:
//
//   * a CTA owns P "row slots" of L lanes; lane c of a row slot always reads the c-th 16-byte
//     chunk of a weight row, so the matching slice of the activation vector is converted once
//     per (expert, token) and reused across R rows held in flight;
//   * gate/up kernel: passes of P*R rows of one expert (routed experts in unique-id order, then
//     the shared expert), dealt round-robin over a fixed grid; it writes h = SiLU(g) * u;
//   * down kernel: each CTA owns a contiguous block of output rows and walks every unique
//     expert (then the shared one) for them, so out[t, j] is summed in one place, in a fixed
//     order, with no atomics.  The combine weight and the row scale are applied there.
//
// Codes are turned into floats with the "magic exponent" construction: OR-ing an unsigned
// code u < 2^23 into the mantissa of 2^23 gives the float 2^23 + u exactly, and one subtraction
// removes the offset; the two's-complement code q = u - bias is recovered by XOR-ing the sign
// bit first.  Accumulation is float32 (products of a small integer and a bf16/f32 value are
// exact in float32).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace coli {

namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int GU_THREADS = 384;  // gate/up CTA (L * P)
constexpr int DN_THREADS = 256;  // down CTA

// Per-format decode constants: codes per 32-bit word, mask, sign-flip pattern, magic offset.
template <int FMT> struct Codes;
template <> struct Codes<4> {
    static constexpr int CPW = 8, BITS = 4;
    static constexpr uint32_t MASK = 0xFu, FLIP = 0x88888888u;
    static constexpr float OFFSET = 8388616.0f;  // 2^23 + 8
};
template <> struct Codes<8> {
    static constexpr int CPW = 4, BITS = 8;
    static constexpr uint32_t MASK = 0xFFu, FLIP = 0x80808080u;
    static constexpr float OFFSET = 8388736.0f;  // 2^23 + 128
};
template <> struct Codes<2> {
    static constexpr int CPW = 16, BITS = 2;
    static constexpr uint32_t MASK = 0x3u, FLIP = 0xAAAAAAAAu;
    static constexpr float OFFSET = 8388610.0f;  // 2^23 + 2
};

template <int FMT>
__device__ __forceinline__ float code_at(uint32_t flipped, int k) {
    const uint32_t u = (flipped >> (Codes<FMT>::BITS * k)) & Codes<FMT>::MASK;
    return __uint_as_float(0x4B000000u | u) - Codes<FMT>::OFFSET;
}

// Streaming 16-byte load: read-only path, no L1 allocation (each weight byte is used once).
__device__ __forceinline__ uint4 ld_stream(const uint8_t *p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// NC (number of columns) activations starting at column col of token row t, as float32.
template <int ACT, int NC>
__device__ __forceinline__ void load_x(const void *x, int H, int t, int col, float *xr) {
    if (ACT == COLI_ACT_F32) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) +
                                                           static_cast<size_t>(t) * H + col);
#pragma unroll
        for (int i = 0; i < NC / 4; ++i) {
            const float4 f = __ldg(p + i);
            xr[4 * i] = f.x; xr[4 * i + 1] = f.y; xr[4 * i + 2] = f.z; xr[4 * i + 3] = f.w;
        }
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) +
                                                         static_cast<size_t>(t) * H + col);
#pragma unroll
        for (int i = 0; i < NC / 8; ++i) {
            const uint4 u = __ldg(p + i);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                xr[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                xr[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
        }
    }
}

template <int NC>
__device__ __forceinline__ void load_h(const float *hrow, int col, float *hr) {
    const float4 *p = reinterpret_cast<const float4 *>(hrow + col);
#pragma unroll
    for (int i = 0; i < NC / 4; ++i) {
        const float4 f = p[i];
        hr[4 * i] = f.x; hr[4 * i + 1] = f.y; hr[4 * i + 2] = f.z; hr[4 * i + 3] = f.w;
    }
}

// Hides a register's value from the optimiser so that code decoding is not hoisted out of the
// token loop (keeping every decoded float of R rows live would exhaust the register file).
__device__ __forceinline__ uint4 opaque(uint4 v) {
    asm volatile("" : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w));
    return v;
}

// Dot of one 16-byte chunk of codes with NC = 4*CPW activations.
template <int FMT>
__device__ __forceinline__ float dot_chunk(const uint4 &q, const float *xr) {
    constexpr int CPW = Codes<FMT>::CPW;
    const uint32_t w[4] = {q.x ^ Codes<FMT>::FLIP, q.y ^ Codes<FMT>::FLIP,
                           q.z ^ Codes<FMT>::FLIP, q.w ^ Codes<FMT>::FLIP};
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int wi = 0; wi < 4; ++wi)
#pragma unroll
        for (int k = 0; k < CPW; k += 2) {
            a0 = fmaf(code_at<FMT>(w[wi], k), xr[wi * CPW + k], a0);
            a1 = fmaf(code_at<FMT>(w[wi], k + 1), xr[wi * CPW + k + 1], a1);
        }
    return a0 + a1;
}

// Sum a value over the L lanes of a row slot.  Lanes of a slot are contiguous; when L > 32 the
// per-warp partials go through shared memory (red[slot][L/32]) and the caller reads the total
// from lane c == 0 after the second barrier.  Returns the total in the c == 0 lane.
__device__ __forceinline__ float warp_sum(float v, int L) {
    const int span = L < 32 ? L : 32;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        if (o < span) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

struct ExpertRef {
    const uint8_t *rec;
    int begin, count;   // slot positions [begin, begin+count)
    bool shared;
    bool ok;
};

__device__ __forceinline__ ExpertRef expert_ref(const FfnParams &p, int we, int U) {
    ExpertRef r;
    if (we < U) {
        const int e = p.unique[we];
        r.shared = false;
        if (e < 0 || e >= p.E) {
            r.ok = false; r.rec = nullptr; r.begin = 0; r.count = 0;
            return r;
        }
        r.rec = p.experts + static_cast<size_t>(e) * p.stride;
        int b = p.offsets[e], en = p.offsets[e + 1];
        const int n = p.T * p.K;
        r.ok = !(b < 0 || en < b || en > n);
        if (!r.ok) { b = 0; en = 0; }
        r.begin = b;
        r.count = en - b;
    } else {
        r.rec = p.shared; r.begin = 0; r.count = p.T; r.shared = true; r.ok = true;
    }
    return r;
}

// Token, combine weight and h row of the q-th slot of an expert; false for a bad slot.
__device__ __forceinline__ bool slot_info(const FfnParams &p, const ExpertRef &x, int q,
                                          int &tok, float &wt, int &hrow) {
    if (x.shared) {
        tok = q; wt = 1.0f; hrow = p.T * p.K + q;
        return true;
    }
    const int pos = x.begin + q;
    const int s = p.perm[pos];
    if (s < 0 || s >= p.T * p.K) return false;
    tok = s / p.K; wt = p.topk_w[s]; hrow = pos;
    return true;
}

__device__ __forceinline__ int read_u(const FfnParams &p) {
    int U = *p.n_unique;
    return U < 0 ? 0 : (U > p.E ? p.E : U);
}

// ---------------------------------------------------------------- gate / up ---------------
template <int FMT, int ACT, int R>
__global__ void __launch_bounds__(GU_THREADS) gateup_kernel(FfnParams p, int L, int P) {
    constexpr int NC = 4 * Codes<FMT>::CPW;  // columns per 16-byte chunk
    extern __shared__ float red[];           // [P][R][2][L/32] partials when L > 32
    const int tid = threadIdx.x;
    const int c = tid % L, slot = tid / L;
    const bool active = slot < P;
    const int nwarp_row = L > 32 ? L / 32 : 1;
    const int U = read_u(p);
    const int nwe = U + p.S;
    const int rpp = P * R;
    const int ppe = (p.I + rpp - 1) / rpp;
    const long total = static_cast<long>(nwe) * ppe;
    // passes dealt round-robin over the grid: a pass costs in proportion to its expert's token
    // count, and the shared expert (all T tokens) would otherwise load a few CTAs only
    for (long pi = blockIdx.x; pi < total; pi += gridDim.x) {
        const int we = static_cast<int>(pi / ppe);
        const int i0 = static_cast<int>(pi % ppe) * rpp;
        const ExpertRef ex = expert_ref(p, we, U);
        if (!ex.ok) {
            if (tid == 0) atomicOr(p.err, we < U && (p.unique[we] < 0 || p.unique[we] >= p.E)
                                              ? COLI_DEVERR_EXPERT_ID : COLI_DEVERR_GROUPING);
            continue;
        }
        if (ex.count > p.gemv_nmax) continue;  // the grouped GEMM's expert
        const uint8_t *wg = ex.rec;
        const uint8_t *wu = ex.rec + p.off_wu;
        const float *sg = reinterpret_cast<const float *>(ex.rec + p.off_sg);
        const float *su = reinterpret_cast<const float *>(ex.rec + p.off_su);
        uint4 qg[R], qu[R];
        // group-scaled container: the scale of this lane's chunk (its group of 64 columns)
        float lg[R], lu[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int i = i0 + slot * R + r;
            lg[r] = lu[r] = 1.0f;
            if (active && i < p.I) {
                qg[r] = ld_stream(wg + static_cast<size_t>(i) * p.rb_h + c * 16);
                qu[r] = ld_stream(wu + static_cast<size_t>(i) * p.rb_h + c * 16);
                if (p.group) {
                    const size_t gi = static_cast<size_t>(i) * p.nsh + (c * NC) / p.group;
                    lg[r] = __ldg(sg + gi);
                    lu[r] = __ldg(su + gi);
                }
            } else {
                qg[r] = make_uint4(0, 0, 0, 0);
                qu[r] = make_uint4(0, 0, 0, 0);
            }
        }
        for (int q = 0; q < ex.count; ++q) {
            int tok, hrow;
            float wt;
            const bool good = slot_info(p, ex, q, tok, wt, hrow);
            if (!good) {
                if (tid == 0) atomicOr(p.err, COLI_DEVERR_GROUPING);
                continue;  // uniform across the CTA
            }
            float xr[NC];
            if (active) load_x<ACT, NC>(p.x, p.H, tok, c * NC, xr);
            float ag[R], au[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                ag[r] = active ? lg[r] * dot_chunk<FMT>(opaque(qg[r]), xr) : 0.f;
                au[r] = active ? lu[r] * dot_chunk<FMT>(opaque(qu[r]), xr) : 0.f;
                ag[r] = warp_sum(ag[r], L);
                au[r] = warp_sum(au[r], L);
            }
            if (nwarp_row > 1) {
                if (active && (c & 31) == 0) {
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        red[((slot * R + r) * 2 + 0) * nwarp_row + (c >> 5)] = ag[r];
                        red[((slot * R + r) * 2 + 1) * nwarp_row + (c >> 5)] = au[r];
                    }
                }
                __syncthreads();
                if (active && c == 0) {
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        float sgv = 0.f, suv = 0.f;
                        for (int k = 0; k < nwarp_row; ++k) {
                            sgv += red[((slot * R + r) * 2 + 0) * nwarp_row + k];
                            suv += red[((slot * R + r) * 2 + 1) * nwarp_row + k];
                        }
                        ag[r] = sgv; au[r] = suv;
                    }
                }
                __syncthreads();
            }
            if (active && c == 0) {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int i = i0 + slot * R + r;
                    if (i < p.I) {
                        const float g = (p.group ? 1.0f : sg[i]) * ag[r];
                        const float u = (p.group ? 1.0f : su[i]) * au[r];
                        p.h[static_cast<size_t>(hrow) * p.I + i] = (g / (1.0f + expf(-g))) * u;
                    }
                }
            }
        }
    }
}

// ---------------------------------------------------------------- down + combine -----------
template <int FMT, int R>
__global__ void __launch_bounds__(DN_THREADS) down_kernel(FfnParams p, int L, int P) {
    constexpr int NC = 4 * Codes<FMT>::CPW;
    extern __shared__ float dsm[];
    const int rpp = P * R;
    const int nwarp_row = L > 32 ? L / 32 : 1;
    const int TA = p.gemv_atomic ? 0 : p.T;             // tokens with accumulators here
    float *acc = dsm;                                   // [TA][rpp]
    float *red = dsm + static_cast<size_t>(TA) * rpp;   // [P][R][L/32]
    const int tid = threadIdx.x;
    const int c = tid % L, slot = tid / L;
    const bool active = slot < P;
    const int U = read_u(p);
    const int nwe = U + p.S;
    const int passes = (p.H + rpp - 1) / rpp;
    const int beg = static_cast<int>(static_cast<long>(passes) * blockIdx.x / gridDim.x);
    const int end = static_cast<int>(static_cast<long>(passes) * (blockIdx.x + 1) / gridDim.x);

    for (int pass = beg; pass < end; ++pass) {
        const int j0 = pass * rpp;
        for (int i = tid; i < TA * rpp; i += blockDim.x) acc[i] = 0.f;
        __syncthreads();
        for (int we = 0; we < nwe; ++we) {
            const ExpertRef ex = expert_ref(p, we, U);
            if (!ex.ok || ex.count > p.gemv_nmax) continue;  // flagged by the gate/up kernel; or the GEMM's
            const uint8_t *wd = ex.rec + p.off_wd;
            const float *sd = reinterpret_cast<const float *>(ex.rec + p.off_sd);
            uint4 qd[R];
            float ld[R];  // group-scaled container: the scale of this lane's chunk
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int j = j0 + slot * R + r;
                qd[r] = (active && j < p.H) ? ld_stream(wd + static_cast<size_t>(j) * p.rb_i + c * 16)
                                            : make_uint4(0, 0, 0, 0);
                ld[r] = (p.group && active && j < p.H) ? __ldg(sd + static_cast<size_t>(j) * p.nsi + (c * NC) / p.group)
                                                       : 1.0f;
            }
            for (int q = 0; q < ex.count; ++q) {
                int tok, hrow;
                float wt;
                if (!slot_info(p, ex, q, tok, wt, hrow)) continue;
                float hr[NC];
                if (active) load_h<NC>(p.h + static_cast<size_t>(hrow) * p.I, c * NC, hr);
                float a[R];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    a[r] = active ? ld[r] * dot_chunk<FMT>(opaque(qd[r]), hr) : 0.f;
                    a[r] = warp_sum(a[r], L);
                }
                if (nwarp_row > 1) {
                    if (active && (c & 31) == 0) {
#pragma unroll
                        for (int r = 0; r < R; ++r) red[(slot * R + r) * nwarp_row + (c >> 5)] = a[r];
                    }
                    __syncthreads();
                    if (active && c == 0) {
#pragma unroll
                        for (int r = 0; r < R; ++r) {
                            float s = 0.f;
                            for (int k = 0; k < nwarp_row; ++k) s += red[(slot * R + r) * nwarp_row + k];
                            a[r] = s;
                        }
                    }
                    __syncthreads();
                }
                if (active && c == 0) {
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const int j = j0 + slot * R + r;
                        if (j >= p.H) continue;
                        const float v = wt * ((p.group ? 1.0f : sd[j]) * a[r]);
                        if (p.gemv_atomic) atomicAdd(p.out + static_cast<size_t>(tok) * p.H + j, v);
                        else acc[tok * rpp + slot * R + r] += v;
                    }
                }
            }
            __syncthreads();
        }
        for (int i = tid; i < TA * rpp; i += blockDim.x) {
            const int t = i / rpp, rr = i % rpp, j = j0 + rr;
            if (j < p.H) p.out[static_cast<size_t>(t) * p.H + j] = acc[i];
        }
        __syncthreads();
    }
}

template <int FMT, int ACT>
cudaError_t launch_fmt(const FfnParams &p, cudaStream_t st, bool gateup, bool down) {
    constexpr int R_GU = 4, R_DN = 4;
    const int sms = device_sm_count();
    // gate/up
    if (gateup) {
        const int L = static_cast<int>(p.rb_h / 16);
        const int P = GU_THREADS / L > 0 ? GU_THREADS / L : 1;
        const int threads = ((L * P + 31) / 32) * 32;
        const size_t smem = L > 32 ? static_cast<size_t>(P) * R_GU * 2 * (L / 32) * sizeof(float) : 0;
        const int grid = sms * 2;
        gateup_kernel<FMT, ACT, R_GU><<<grid, threads, smem, st>>>(p, L, P);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // down + combine
    if (down) {
        const int L = static_cast<int>(p.rb_i / 16);
        const int P = DN_THREADS / L > 0 ? DN_THREADS / L : 1;
        const int threads = ((L * P + 31) / 32) * 32;
        const int rpp = P * R_DN;
        const size_t smem = (static_cast<size_t>(p.gemv_atomic ? 0 : p.T) * rpp +
                             (L > 32 ? static_cast<size_t>(P) * R_DN * (L / 32) : 0)) * sizeof(float);
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(down_kernel<FMT, R_DN>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem));
            if (e != cudaSuccess) return e;
        }
        const int passes = (p.H + rpp - 1) / rpp;
        const int grid = passes < sms * 4 ? passes : sms * 4;
        down_kernel<FMT, R_DN><<<grid, threads, smem, st>>>(p, L, P);
    }
    return cudaGetLastError();
}

}  // namespace

bool gemv_shape_ok(int row_bytes) {
    if (row_bytes <= 0 || row_bytes % 16) return false;
    const int L = row_bytes / 16;
    if (L > 384) return false;
    if (L < 32) return 32 % L == 0;
    return L % 32 == 0;
}

int gemv_max_tokens(const coli_moe_config &) {
    // The down kernel keeps T x (P*R) float accumulators in shared memory and walks every slot
    // of every expert per row block; beyond a few hundred tokens the grouped tensor-core path
    // is the one that fits.
    return 256;
}

static cudaError_t launch_parts(const FfnParams &p, cudaStream_t st, bool gateup, bool down) {
    if (p.act == COLI_ACT_F32) {
        if (p.fmt == 4) return launch_fmt<4, COLI_ACT_F32>(p, st, gateup, down);
        if (p.fmt == 8) return launch_fmt<8, COLI_ACT_F32>(p, st, gateup, down);
        if (p.fmt == 2) return launch_fmt<2, COLI_ACT_F32>(p, st, gateup, down);
    } else {
        if (p.fmt == 4) return launch_fmt<4, COLI_ACT_BF16>(p, st, gateup, down);
        if (p.fmt == 8) return launch_fmt<8, COLI_ACT_BF16>(p, st, gateup, down);
        if (p.fmt == 2) return launch_fmt<2, COLI_ACT_BF16>(p, st, gateup, down);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_ffn_gemv(const FfnParams &p, cudaStream_t st) { return launch_parts(p, st, true, true); }
cudaError_t launch_ffn_gemv_gateup(const FfnParams &p, cudaStream_t st) { return launch_parts(p, st, true, false); }
cudaError_t launch_ffn_gemv_down(const FfnParams &p, cudaStream_t st) { return launch_parts(p, st, false, true); }

}  // namespace coli
