// scan_fwd_wide.cuh -- forward scan and decode for wider states: d_state N in {32, 64, 128, 256}
// ([Eng] §7.1: a larger d_state trades on-chip residency for capacity; [Card] 状态空间原理).
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
//
// The step is the one of the d_state = 16 kernels (simplified or zero-order-hold weight,
// [Card] 离散化变换 / [Eng] §2.2).  With N exponentials per element these shapes are bound by
// the special-function unit (N/16 times the work of N = 16 per element).  G = N/4 lanes per
// channel (N/8 for N = 256), each lane holding 4 (8) chains of the channel in registers for
// the whole sequence in f32x2 pairs, 32/G channels per warp, 8 warps per block, all on one
// batch row.  The block stages the packed fp32 B/C rows (2N floats per step) of 64 (32) steps
// at a time through a double-buffered cp.async ring in shared memory.  Steps go in batches of
// G: lane nl of a channel loads (one batch ahead) and evaluates the step size of step nl, the
// lanes walk the G steps with the step size and input broadcast by shuffles, and the G lanes'
// partial sums of C.h are reduce-scattered so that lane nl finishes (D skip, gate, rounding,
// store) step nl.
#pragma once

#include "common.cuh"
#include "scan_math.cuh"

namespace ssm {

struct WideParams {
    const void *u, *delta, *z;  // (batch, dim, L) IO
    const float* bc;            // packed [batch][L][2N] fp32: B[0..N-1], C[0..N-1] per step
    const float *A, *D, *bias, *h0;
    void* y;
    float* last_state;          // (batch, dim, N) or null
    int batch, dim;
    long long L;
    int softplus, zoh;
};

template <int N>
struct WideCfg {
    static constexpr int kNC = N <= 128 ? 4 : 8;  // chains per lane
    static constexpr int kG = N / kNC;             // lanes per channel: 8, 16, 32, 32
    static constexpr int kCPW = 32 / kG;           // channels per warp: 4, 2, 1, 1
    static constexpr int kT = kG;                  // steps per batch (one step per lane of a channel)
    // warps per block (one batch row per block); N = 256 stages 128 KB per block, so its
    // blocks are twice as large to keep 16 warps per SM
    static constexpr int kWarps = N == 256 ? 16 : 8;
    static constexpr int kCPB = kWarps * kCPW;     // channels per block
    static constexpr int kST = N <= 64 ? 64 : 32;  // steps per staged stage of B/C rows
    static constexpr int kStageFloats = kST * 2 * N;
    static constexpr int kSmem = 2 * kStageFloats * 4;  // double-buffered stages
};

// Blocks per SM in the launch bound: measured on B200 (batch 4, d_inner 2048, L 2048), 3 blocks
// (80 registers) take N = 128 from 1.081 to 0.948 ms but spill at N = 32, 64 (0.31 -> 0.33 ms,
// 0.535 -> 0.547 ms); N = 256 holds 128 KB of B/C stages (one block).
template <int N>
constexpr int wide_min_blocks() { return N == 256 ? 1 : N == 128 ? 3 : 2; }

template <typename IO, int N>
__global__ void __launch_bounds__(WideCfg<N>::kWarps * 32, wide_min_blocks<N>()) scan_fwd_wide_kernel(const WideParams p) {
    using Cfg = WideCfg<N>;
    constexpr int NC = Cfg::kNC, G = Cfg::kG, CPW = Cfg::kCPW, T = Cfg::kT, ST = Cfg::kST;
    static_assert(N == 32 || N == 64 || N == 128 || N == 256, "N in {32, 64, 128, 256}");
    static_assert(ST % T == 0, "whole batches per stage");
    extern __shared__ float4 wide_smem[];
    float* ring = reinterpret_cast<float*>(wide_smem);  // [2][ST][2N]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cg = lane / G, nl = lane % G, gbase = lane & ~(G - 1);
    const int b = blockIdx.y;
    const int d = blockIdx.x * Cfg::kCPB + warp * CPW + cg;
    const bool valid = d < p.dim;
    const int dd = valid ? d : 0;
    const long long L = p.L;
    const long long ch = static_cast<long long>(b) * p.dim + dd;
    const IO* u = static_cast<const IO*>(p.u) + ch * L;
    const IO* dl = static_cast<const IO*>(p.delta) + ch * L;
    const IO* z = p.z ? static_cast<const IO*>(p.z) + ch * L : nullptr;
    IO* y = static_cast<IO*>(p.y) + ch * L;
    const float* bcrow = p.bc + static_cast<long long>(b) * L * (2 * N);

    float2 A2[NC / 2], invA[NC / 2], h[NC / 2];
#pragma unroll
    for (int j = 0; j < NC / 2; ++j) {
        const float a0 = p.A[static_cast<long long>(dd) * N + nl * NC + 2 * j];
        const float a1 = p.A[static_cast<long long>(dd) * N + nl * NC + 2 * j + 1];
        A2[j] = make_float2(a0 * kLog2e, a1 * kLog2e);
        invA[j] = make_float2(1.f / a0, 1.f / a1);
        h[j] = (p.h0 && valid) ? *reinterpret_cast<const float2*>(p.h0 + ch * N + nl * NC + 2 * j)
                               : make_float2(0.f, 0.f);
    }
    const float Dd = (valid && p.D) ? p.D[dd] : 0.f;
    const float bias = (valid && p.bias) ? p.bias[dd] : 0.f;
    const bool softplus = p.softplus != 0, zoh = p.zoh != 0;

    // B/C rows of stage k into ring slot k & 1 (zero past L), one cp.async group per stage.
    const long long nstages = (L + ST - 1) / ST;
    auto issue = [&](long long k) {
        if (k < nstages) {
            float* dst = ring + (k & 1) * Cfg::kStageFloats;
            for (int c = threadIdx.x; c < Cfg::kStageFloats / 4; c += blockDim.x) {
                const int i = c / (2 * N / 4), part = c % (2 * N / 4);
                const long long t = k * ST + i;
                const bool in = t < L;
                cp_async_16(dst + i * 2 * N + part * 4, in ? bcrow + t * 2 * N + part * 4 : bcrow, in ? 16u : 0u);
            }
        }
        cp_async_commit();
    };
    // Inputs of the lane's own step of a batch (0 past L), loaded one batch ahead.
    auto load_own = [&](long long t, float& ul, float& xl, float& zl) {
        const bool in = valid && t < L;
        ul = in ? IoTraits<IO>::to_f32(u[t]) : 0.f;
        xl = in ? IoTraits<IO>::to_f32(dl[t]) : 0.f;
        zl = (in && z) ? IoTraits<IO>::to_f32(z[t]) : 0.f;
    };

    issue(0);
    float un, xn, zn;
    load_own(nl, un, xn, zn);
    for (long long k = 0; k < nstages; ++k) {
        issue(k + 1);
        cp_async_wait<1>();
        __syncthreads();  // stage k visible to every warp
        const float* stage = ring + (k & 1) * Cfg::kStageFloats + nl * NC;
#pragma unroll 1
        for (int bt = 0; bt < ST; bt += T) {
            const long long t0 = k * ST + bt;
            const long long t = t0 + nl;
            const float ul = un, zl = zn;
            const float dtl = (valid && t < L) ? step_size(xn, bias, softplus) : 0.f;  // 0 past L
            load_own(t + T, un, xn, zn);  // next batch (the next stage's first for the last batch)
            float yp[T];
#pragma unroll
            for (int i = 0; i < T; ++i) {
                const float dti = __shfl_sync(0xffffffffu, dtl, gbase | i);
                const float ui = __shfl_sync(0xffffffffu, ul, gbase | i);
                const float* row = stage + (bt + i) * 2 * N;
                float2 Bv[NC / 2], Cv[NC / 2];
#pragma unroll
                for (int j = 0; j < NC / 2; j += 2) {
                    const float4 bq = *reinterpret_cast<const float4*>(row + 2 * j);
                    const float4 cq = *reinterpret_cast<const float4*>(row + N + 2 * j);
                    Bv[j] = make_float2(bq.x, bq.y);
                    Bv[j + 1] = make_float2(bq.z, bq.w);
                    Cv[j] = make_float2(cq.x, cq.y);
                    Cv[j + 1] = make_float2(cq.z, cq.w);
                }
                const float2 dd2 = make_float2(dti, dti), ww = make_float2(dti * ui, dti * ui);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < NC / 2; ++j) {
                    const float2 arg = __fmul2_rn(dd2, A2[j]);
                    const float2 a = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                    float2 beta = __fmul2_rn(ww, Bv[j]);
                    if (zoh)
                        beta = zoh_beta2(arg, a, beta, __fmul2_rn(__fmul2_rn(make_float2(ui, ui), Bv[j]), invA[j]));
                    h[j] = __ffma2_rn(a, h[j], beta);
                    acc = __ffma2_rn(Cv[j], h[j], acc);
                }
                yp[i] = acc.x + acc.y;
            }
            // Reduce-scatter the T partial sums over the G lanes of the channel (upper lane
            // bit first): lane nl ends with the full sum of step t0 + nl in yp[0].
#pragma unroll
            for (int m = G / 2; m >= 1; m >>= 1) {
                const bool upper = (nl & m) != 0;
#pragma unroll
                for (int i = 0; i < m; ++i) {
                    const float send = upper ? yp[i] : yp[i + m];
                    const float keep = upper ? yp[i + m] : yp[i];
                    yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            if (valid && t < L) {
                float v = fmaf(Dd, ul, yp[0]);
                if (z) v *= silu_f32(zl);
                y[t] = IoTraits<IO>::from_f32(v);
            }
        }
        __syncthreads();  // every warp is done with slot k & 1 before it is refilled
    }
    cp_async_wait<0>();
    if (p.last_state && valid)
#pragma unroll
        for (int j = 0; j < NC / 2; ++j) *reinterpret_cast<float2*>(p.last_state + ch * N + nl * NC + 2 * j) = h[j];
}

// B, C (batch, N, L) -> fp32 rows [batch][L][2N] (B then C): 32 x 32 tiles through shared
// memory.  grid = (ceil(L/32), batch, 2N/32), block 32 x 8.
template <typename IO>
__global__ void __launch_bounds__(256) pack_bc_wide_kernel(const IO* __restrict__ B, const IO* __restrict__ C,
                                                           float* __restrict__ bc, long long L, int N) {
    __shared__ float tile[32][33];
    const int b = blockIdx.y;
    const long long t0 = static_cast<long long>(blockIdx.x) * 32;
    const int j0 = blockIdx.z * 32;  // component index in [0, 2N)
    for (int r = threadIdx.y; r < 32; r += 8) {
        const int j = j0 + r;
        const IO* src = j < N ? B : C;
        const int n = j < N ? j : j - N;
        const long long t = t0 + threadIdx.x;
        tile[r][threadIdx.x] = t < L ? IoTraits<IO>::to_f32(src[(static_cast<long long>(b) * N + n) * L + t]) : 0.f;
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += 8) {
        const long long t = t0 + r;
        if (t < L) bc[(static_cast<long long>(b) * L + t) * (2 * N) + j0 + threadIdx.x] = tile[threadIdx.x][r];
    }
}

// One-token decode for d_state N: TPC = min(N/4, 32) threads per channel, each owning NC =
// N / TPC consecutive state values (fp32, in place); C.h combined by xor shuffles.
template <typename IO, int N>
__global__ void __launch_bounds__(256) state_update_wide_kernel(const float* A, const float* D, const float* bias,
                                                                float* state, const void* u, const void* delta,
                                                                const void* B, const void* C, const void* z, void* y,
                                                                int batch, int dim, int softplus, int zoh) {
    constexpr int TPC = N / 4 < 32 ? N / 4 : 32, NC = N / TPC;
    const long long gid = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
    const long long row = gid / TPC;
    const int q = static_cast<int>(gid % TPC);
    const bool valid = row < static_cast<long long>(batch) * dim;
    const long long rr = valid ? row : 0;
    const int b = static_cast<int>(rr / dim), d = static_cast<int>(rr % dim);
    float hs[NC], Bq[NC], Cq[NC], As[NC];
    float ut = 0.f, dt = 0.f, zt = 0.f;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        hs[j] = valid ? state[rr * N + q * NC + j] : 0.f;
        As[j] = valid ? A[static_cast<long long>(d) * N + q * NC + j] : 0.f;
        Bq[j] = valid ? IoTraits<IO>::to_f32(static_cast<const IO*>(B)[static_cast<long long>(b) * N + q * NC + j]) : 0.f;
        Cq[j] = valid ? IoTraits<IO>::to_f32(static_cast<const IO*>(C)[static_cast<long long>(b) * N + q * NC + j]) : 0.f;
    }
    if (valid) {
        ut = IoTraits<IO>::to_f32(static_cast<const IO*>(u)[rr]);
        dt = step_size(IoTraits<IO>::to_f32(static_cast<const IO*>(delta)[rr]), bias ? bias[d] : 0.f, softplus != 0);
        if (z) zt = IoTraits<IO>::to_f32(static_cast<const IO*>(z)[rr]);
    }
    const float w = dt * ut;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        const float yj = dt * As[j] * kLog2e;
        const float a = ex2_mufu(yj);
        const float beta = zoh ? zoh_beta(yj, a, w * Bq[j], ut * Bq[j] / As[j]) : w * Bq[j];
        hs[j] = fmaf(a, hs[j], beta);
        acc = fmaf(Cq[j], hs[j], acc);
    }
#pragma unroll
    for (int m = 1; m < TPC; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m, 32);
    if (valid) {
#pragma unroll
        for (int j = 0; j < NC; ++j) state[rr * N + q * NC + j] = hs[j];
        if (q == 0) {
            float v = fmaf(D ? D[d] : 0.f, ut, acc);
            if (z) v *= silu_f32(zt);
            static_cast<IO*>(y)[rr] = IoTraits<IO>::from_f32(v);
        }
    }
}

}  // namespace ssm
