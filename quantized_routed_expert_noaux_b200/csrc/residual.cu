// residual.cu -- the residual update that chains MoE layers on the device.
//
// JustVugg/colibri README, "Never wait for the disk twice": the GPU-resident pipeline keeps the
// residual stream on the device across layers.  The next layer's input is the residual stream
// plus this layer's output, x_next = x + out: the sum is one float32 addition (round to nearest
// even) and, for bf16 activations, the result is rounded to bf16 (round to nearest even).
//
// HBM-bound elementwise pass: each thread takes 8 bf16 (or 4 float32) elements per step with
// 16-byte loads and stores, grid-stride over the tensor with a grid of up to 8 CTAs per SM (the
// element count is a multiple of 64: the hidden size is).  Every element is read and written by
// the same thread, so x_next may be x itself.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "residual.h"

namespace coli {

namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// float32 -> bf16 bits, round to nearest even; NaN stays a (quiet) NaN.
__device__ __forceinline__ uint32_t f32_to_bf16_rne(float v) {
    const uint32_t u = __float_as_uint(v);
    if ((u & 0x7fffffffu) > 0x7f800000u) return ((u >> 16) | 0x40u) & 0xffffu;
    return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
}

__global__ void __launch_bounds__(256) residual_bf16_kernel(const uint16_t *x, const float *out,
                                                            size_t n, uint16_t *x_next) {
    const size_t n8 = n / 8;
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const uint4 xv = __ldcs(reinterpret_cast<const uint4 *>(x) + i);
        const float4 o0 = __ldcs(reinterpret_cast<const float4 *>(out) + 2 * i);
        const float4 o1 = __ldcs(reinterpret_cast<const float4 *>(out) + 2 * i + 1);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
        uint32_t r[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lo = __fadd_rn(bf16_bits_to_f32(xw[k] & 0xffffu), ov[2 * k]);
            const float hi = __fadd_rn(bf16_bits_to_f32(xw[k] >> 16), ov[2 * k + 1]);
            r[k] = f32_to_bf16_rne(lo) | (f32_to_bf16_rne(hi) << 16);
        }
        reinterpret_cast<uint4 *>(x_next)[i] = make_uint4(r[0], r[1], r[2], r[3]);
    }
}

__global__ void __launch_bounds__(256) residual_f32_kernel(const float *x, const float *out,
                                                           size_t n, float *x_next) {
    const size_t n4 = n / 4;
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 a = __ldcs(reinterpret_cast<const float4 *>(x) + i);
        const float4 o = __ldcs(reinterpret_cast<const float4 *>(out) + i);
        reinterpret_cast<float4 *>(x_next)[i] =
            make_float4(__fadd_rn(a.x, o.x), __fadd_rn(a.y, o.y), __fadd_rn(a.z, o.z), __fadd_rn(a.w, o.w));
    }
}

}  // namespace

cudaError_t launch_residual(const coli_moe_config &c, const void *x, const float *out, int T, void *x_next,
                            cudaStream_t st) {
    const size_t n = static_cast<size_t>(T) * c.hidden;
    const int per = c.act == COLI_ACT_BF16 ? 8 : 4;
    const size_t units = n / per;
    const int sms = device_sm_count();
    size_t blocks = (units + 255) / 256;
    const size_t cap = static_cast<size_t>(sms > 0 ? sms : 148) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (c.act == COLI_ACT_BF16)
        residual_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            static_cast<const uint16_t *>(x), out, n, static_cast<uint16_t *>(x_next));
    else
        residual_f32_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            static_cast<const float *>(x), out, n, static_cast<float *>(x_next));
    return cudaGetLastError();
}

}  // namespace coli
