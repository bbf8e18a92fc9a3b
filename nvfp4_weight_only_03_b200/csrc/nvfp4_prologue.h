// Input prologues of the GEMV calls: the transforms of x that the decode step runs just before
// a projection ("Blueprint - circuit executor" page for qwen3.8-27b-nvfp4 on GB10, table "Kernels
// the plan launches": residual_add_rms_norm / rms_norm before the attention and FFN projections,
// sigmoid_gate_mul before the attention output projection).  The prologue grid ahead of the
// 1..8-row GEMV (nvfp4_gemv.cu) and the x pass of the tensor-core tier (nvfp4_gemv_tc.cu) both
// use these helpers, so the two form x' with the same operations.
//
//   NVFP4_PROLOGUE_ADD_RMSNORM:  h = bf16(x + r);  x' = bf16((h * inv) * gamma),
//                                inv = 1 / sqrt(sum_k h^2 / K + eps)
//   NVFP4_PROLOGUE_SIGMOID_GATE: x' = bf16(x / (1 + e^-gate))
//   NVFP4_PROLOGUE_GATED_RMSNORM: x fp32; x' = bf16(((x * inv_g) * gamma[k mod G]) * silu(z)),
//                                inv_g = 1 / sqrt(sum_{group} x^2 / G + eps), silu(t) = t / (1 + e^-t)
//
// in fp32.  x + r of two bf16 values rounded once to bf16 equals the exactly rounded sum (fp32
// carries more than twice bf16's precision plus two bits).  Each caller sums a row's squares in
// an order fixed by K alone, so x' of a row does not depend on M.
#ifndef NVFP4_PROLOGUE_H
#define NVFP4_PROLOGUE_H

#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4.h"

namespace nvfp4_pro {

struct Prologue {
    int kind;              // NVFP4_PROLOGUE_*
    float eps;             // ADD_RMSNORM
    const uint16_t* in;    // residual (ADD_RMSNORM) or gate (SIGMOID_GATE): bf16 [M][ld_in]
    int64_t ld_in;
    const uint16_t* gamma; // ADD_RMSNORM: bf16 [K]
    uint16_t* hout;        // ADD_RMSNORM: h = bf16(x + r), bf16 [M][ldh], or null
    int64_t ldh;
    int group;             // GATED_RMSNORM: channels per group
};

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t bf2_rn(float lo, float hi) {
    uint32_t u;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(hi), "f"(lo));
    return u;
}

// h = bf16(x + r) for 8 bf16 values
__device__ __forceinline__ uint4 add_8(uint4 x, uint4 r) {
    return make_uint4(bf2_rn(bf_lo(x.x) + bf_lo(r.x), bf_hi(x.x) + bf_hi(r.x)),
                      bf2_rn(bf_lo(x.y) + bf_lo(r.y), bf_hi(x.y) + bf_hi(r.y)),
                      bf2_rn(bf_lo(x.z) + bf_lo(r.z), bf_hi(x.z) + bf_hi(r.z)),
                      bf2_rn(bf_lo(x.w) + bf_lo(r.w), bf_hi(x.w) + bf_hi(r.w)));
}

// ss + h_0^2 + ... + h_7^2, one fused multiply-add per element in element order
__device__ __forceinline__ float sum_squares_8(uint4 h, float ss) {
    const uint32_t w[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        ss = fmaf(bf_lo(w[i]), bf_lo(w[i]), ss);
        ss = fmaf(bf_hi(w[i]), bf_hi(w[i]), ss);
    }
    return ss;
}

// inv = 1 / sqrt(ss / K + eps)
__device__ __forceinline__ float rms_inverse(float ss, int64_t k, float eps) {
    return 1.0f / sqrtf(ss / (float)k + eps);
}

// x' = bf16((h * inv) * gamma) for 8 values of h
__device__ __forceinline__ uint4 scale_8(uint4 h, uint4 g, float inv) {
    return make_uint4(bf2_rn(bf_lo(h.x) * inv * bf_lo(g.x), bf_hi(h.x) * inv * bf_hi(g.x)),
                      bf2_rn(bf_lo(h.y) * inv * bf_lo(g.y), bf_hi(h.y) * inv * bf_hi(g.y)),
                      bf2_rn(bf_lo(h.z) * inv * bf_lo(g.z), bf_hi(h.z) * inv * bf_hi(g.z)),
                      bf2_rn(bf_lo(h.w) * inv * bf_lo(g.w), bf_hi(h.w) * inv * bf_hi(g.w)));
}

// x' = bf16((h * inv) * gamma), h = bf16(x + r)
__device__ __forceinline__ uint4 norm_8(uint4 x, uint4 r, uint4 g, float inv) {
    return scale_8(add_8(x, r), g, inv);
}

__device__ __forceinline__ float gated(float a, float t) { return a / (1.0f + expf(-t)); }

// x' = bf16(x * sigmoid(gate))
__device__ __forceinline__ uint4 gate_8(uint4 x, uint4 t) {
    return make_uint4(bf2_rn(gated(bf_lo(x.x), bf_lo(t.x)), gated(bf_hi(x.x), bf_hi(t.x))),
                      bf2_rn(gated(bf_lo(x.y), bf_lo(t.y)), gated(bf_hi(x.y), bf_hi(t.y))),
                      bf2_rn(gated(bf_lo(x.z), bf_lo(t.z)), gated(bf_hi(x.z), bf_hi(t.z))),
                      bf2_rn(gated(bf_lo(x.w), bf_lo(t.w)), gated(bf_hi(x.w), bf_hi(t.w))));
}

// x' = bf16(((x * inv) * gamma) * silu(z)) for 4 fp32 values of x, 4 bf16 of z and gamma
__device__ __forceinline__ uint2 gated_4(float4 x, uint2 z, uint2 g, float inv) {
    const float z0 = bf_lo(z.x), z1 = bf_hi(z.x), z2 = bf_lo(z.y), z3 = bf_hi(z.y);
    return make_uint2(bf2_rn(x.x * inv * bf_lo(g.x) * gated(z0, z0),
                             x.y * inv * bf_hi(g.x) * gated(z1, z1)),
                      bf2_rn(x.z * inv * bf_lo(g.y) * gated(z2, z2),
                             x.w * inv * bf_hi(g.y) * gated(z3, z3)));
}

// The transformed 8 values at (row m, k .. k+7) given x's raw values there.
__device__ __forceinline__ uint4 apply_8(const Prologue& p, uint4 x, int m, int64_t k, float inv) {
    const uint4 a = *reinterpret_cast<const uint4*>(p.in + m * p.ld_in + k);
    if (p.kind == NVFP4_PROLOGUE_ADD_RMSNORM)
        return norm_8(x, a, *reinterpret_cast<const uint4*>(p.gamma + k), inv);
    return gate_8(x, a);
}

}  // namespace nvfp4_pro

#endif
