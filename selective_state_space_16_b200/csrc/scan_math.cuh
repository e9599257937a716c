// scan_math.cuh -- the scalar pieces of the selective-scan step, in fp32.
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
#pragma once

#include <cuda_runtime.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;  // log2(e): exp(x) = 2^(x log2 e)

// 2^x on the special-function unit (MUFU.EX2); subnormal results flush to zero.
__device__ __forceinline__ float ex2_mufu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Step size Delta = softplus(x) with x = delta + bias ([Eng] §3.2: the bias sits inside
// softplus; [Card] 选择性机制: softplus keeps the step positive).  Above x = 20 the
// correction log1p(e^-x) < 2.1e-9 is below fp32 resolution of x, so x is returned.
__device__ __forceinline__ float softplus_f32(float x) {
    return x > 20.f ? x : log1pf(ex2_mufu(x * kLog2e));
}

__device__ __forceinline__ float step_size(float raw, float bias, bool softplus) {
    const float x = raw + bias;
    return softplus ? softplus_f32(x) : x;
}

// silu(z) = z / (1 + e^-z), the SiLU gate of the Mamba block ([Hist] Mamba Block 数据流).
// For z -> -inf the denominator overflows to +inf and the result is 0.
__device__ __forceinline__ float silu_f32(float z) {
    return __fdividef(z, 1.f + ex2_mufu(-z * kLog2e));
}

}  // namespace ssm
