// scan_math.cuh -- the scalar pieces of the selective-scan step, in fp32.
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
#pragma once

#include <cuda_runtime.h>

#include "poly_coeffs.cuh"

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;  // log2(e): exp(x) = 2^(x log2 e)

// 2^x on the special-function unit (MUFU.EX2); subnormal results flush to zero.
__device__ __forceinline__ float ex2_mufu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Step size Delta = softplus(x) with x = delta + bias ([Eng] §3.2: the bias sits inside
// softplus; [Card] 选择性机制: softplus keeps the step positive), evaluated as
//   softplus(x) = max(x, 0) + log1p(e),  e = e^{-|x|} in (0, 1],
// with log1p(e) = e * P(e) from a degree-8 polynomial fitted on [0, 1] (gen_poly.py;
// relative error 2.3e-7 in fp32).  One special-function op (the exponential); for
// x < -87 e flushes to zero and the result is 0 (the true value is below 1e-38).
__device__ __forceinline__ float softplus_f32(float x) {
    constexpr float c[] = SSM_LOG1P_POLY;
    const float e = ex2_mufu(-fabsf(x) * kLog2e);
    float p = c[8];
#pragma unroll
    for (int i = 7; i >= 0; --i) p = fmaf(p, e, c[i]);
    return fmaf(e, p, fmaxf(x, 0.f));
}

__device__ __forceinline__ float step_size(float raw, float bias, bool softplus) {
    const float x = raw + bias;
    return softplus ? softplus_f32(x) : x;
}

// Zero-order-hold input weight ([Eng] §2.2): Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B
// = Delta B phi(Delta A), phi(x) = (e^x - 1) / x, for a diagonal A (phi -> 1 as A -> 0).
// With y = Delta A log2(e) and a = 2^y already at hand, the weight times u is
//   |y| >= kZohSmall:  (a - 1) * (u B / A)              (no cancellation: |a - 1| > 0.06)
//   |y| <  kZohSmall:  (Delta u B) * phi, phi = 1 + x/2 + x^2/6 + x^3/24  (x = y ln 2;
//                      truncation error x^4/120 < 1.3e-7 relative at |x| = 1/16)
// Both are formed and one is selected, so A = 0 (u B / A infinite) never reaches the result.
constexpr float kZohSmall = 0.0901684400f;  // log2(e) / 16: |Delta A| < 1/16
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kZohP1 = kLn2 / 2.f, kZohP2 = kLn2 * kLn2 / 6.f, kZohP3 = kLn2 * kLn2 * kLn2 / 24.f;

__device__ __forceinline__ float zoh_beta(float y, float a, float wB, float uB_over_A) {
    const float phi = fmaf(fmaf(fmaf(kZohP3, y, kZohP2), y, kZohP1), y, 1.f);
    return fabsf(y) < kZohSmall ? wB * phi : (a - 1.f) * uB_over_A;
}

// The same for a pair of chains (f32x2 arithmetic).
__device__ __forceinline__ float2 zoh_beta2(float2 y, float2 a, float2 wB, float2 uB_over_A) {
    const float2 phi = __ffma2_rn(__ffma2_rn(__ffma2_rn(make_float2(kZohP3, kZohP3), y, make_float2(kZohP2, kZohP2)), y,
                                             make_float2(kZohP1, kZohP1)),
                                  y, make_float2(1.f, 1.f));
    const float2 small = __fmul2_rn(wB, phi);
    const float2 big = __fmul2_rn(__fadd2_rn(a, make_float2(-1.f, -1.f)), uB_over_A);
    return make_float2(fabsf(y.x) < kZohSmall ? small.x : big.x, fabsf(y.y) < kZohSmall ? small.y : big.y);
}

// The zero-order-hold weight per unit B u itself, phi = expm1(Delta A) / A, for a pair of chains,
// from y = Delta A log2(e), a = 2^y, dt = Delta and invA = 1 / A:
//   |y| >= kZohSmall:  (a - 1) / A = fma(a, invA, -invA)     (one rounding)
//   |y| <  kZohSmall:  Delta (1 + x/2 + x^2/6 + x^3/24), x = y ln 2   (as zoh_beta2)
// (the weight of zoh_beta2 without its factor u B, which the caller applies once).
__device__ __forceinline__ float2 zoh_phi2(float2 y, float2 a, float2 dt, float2 invA) {
    const float2 poly = __ffma2_rn(__ffma2_rn(__ffma2_rn(make_float2(kZohP3, kZohP3), y, make_float2(kZohP2, kZohP2)),
                                              y, make_float2(kZohP1, kZohP1)),
                                   y, make_float2(1.f, 1.f));
    const float2 small = __fmul2_rn(dt, poly);
    const float2 big = __ffma2_rn(a, invA, make_float2(-invA.x, -invA.y));
    return make_float2(fabsf(y.x) < kZohSmall ? small.x : big.x, fabsf(y.y) < kZohSmall ? small.y : big.y);
}

// Derivative of the zero-order-hold weight per unit input, phi(Delta, A) = expm1(Delta A) / A,
// with respect to A, for a pair of chains (the backward of the ZOH scan):
//   dphi/dA = (Delta a - phi) / A                             for |y| >= kZohSmall,
//           = Delta^2 (1/2 + x/3 + x^2/8 + x^3/30)              for |y| <  kZohSmall (x = y ln 2),
// the second the Taylor series of the first (the k-th coefficient of (x e^x - e^x + 1) / x^2 is
// 1 / (k! (k + 2)); the first term left out, x^4 / 144, is 2.1e-7 of the sum at |x| = 1/16), which avoids the
// cancellation of Delta a - phi for small Delta A.  phi is the weight (zoh_phi2); the derivative
// with respect to Delta is a itself.
constexpr float kZohQ1 = kLn2 / 3.f, kZohQ2 = kLn2 * kLn2 / 8.f, kZohQ3 = kLn2 * kLn2 * kLn2 / 30.f;

__device__ __forceinline__ float2 zoh_dphi_dA2(float2 y, float2 a, float2 dt, float2 phi, float2 invA) {
    const float2 q = __ffma2_rn(__ffma2_rn(__ffma2_rn(make_float2(kZohQ3, kZohQ3), y, make_float2(kZohQ2, kZohQ2)), y,
                                           make_float2(kZohQ1, kZohQ1)),
                                y, make_float2(0.5f, 0.5f));
    const float2 small = __fmul2_rn(__fmul2_rn(dt, dt), q);
    const float2 big = __fmul2_rn(__ffma2_rn(dt, a, make_float2(-phi.x, -phi.y)), invA);
    return make_float2(fabsf(y.x) < kZohSmall ? small.x : big.x, fabsf(y.y) < kZohSmall ? small.y : big.y);
}

// silu(z) = z / (1 + e^-z), the SiLU gate of the Mamba block ([Hist] Mamba Block 数据流).
// For z -> -inf the denominator overflows to +inf and the result is 0.
__device__ __forceinline__ float silu_f32(float z) {
    return __fdividef(z, 1.f + ex2_mufu(-z * kLog2e));
}

// silu(z) = z * sigmoid(z) with sigmoid(z) = (1 + tanh(z/2)) / 2 on the special-function
// unit (tanh.approx, relative error <= 2^-11): one special-function op instead of two.
// Used only where the gated output is rounded to bf16 (relative step 2^-8), so the
// approximation stays below the output's own rounding.
__device__ __forceinline__ float silu_tanh_f32(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    return z * fmaf(0.5f, t, 0.5f);
}

// The gate used for an output element type: accurate for fp32 outputs, the one-op
// tanh form for bf16 outputs.
template <typename IO>
__device__ __forceinline__ float gate_silu(float z) {
    if constexpr (sizeof(IO) == 2) return silu_tanh_f32(z);
    else return silu_f32(z);
}

}  // namespace ssm
