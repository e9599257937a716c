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
// the special-function unit (N/16 times the work of N = 16 per element) -- and, were every
// lane to load its own B/C values, equally by the shared-memory data path: a lane's chains need
// 2 floats of B/C per exponential, one 4-byte wavefront slot per float, so N/16 wavefronts per
// element against the unit's N/16 clocks.  Each lane therefore holds the same NC chains of TWO
// channels (CPL = 2; N = 32 keeps one), so that one load of B/C feeds both: G = N/NC lanes per
// channel group (WideCfg), the chains in f32x2 pairs in registers for the whole sequence, all
// warps of a block on one batch row.  The block stages the packed fp32 B/C rows (2N floats
// per step) of 16 to 64 steps at a time through a double-buffered cp.async ring in shared
// memory.  Steps go in batches of 8: lane nl loads (one batch ahead) and
// evaluates the step size of step nl mod 8 of its channels (the G/8 copies redundantly), the
// lanes walk the 8 steps with step size and input broadcast by shuffles, and the partial sums
// of C.h are reduce-scattered over 8 lanes and added over the G/8 copies, so that each (step,
// channel) is finished (D skip, gate, rounding, store) by one lane.
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
    // chains per lane and channel, channels per lane (one load of B/C feeds them all), warps
    // per block, steps per staged stage of B/C rows: the best of the configurations measured
    // on B200 (batch 4, d_inner 2048, L 2048, bf16) -- N = 32 keeps one channel per lane
    // (its 8192 channels would leave too few warps), N = 256 stages 16 steps so that two
    // blocks fit.
    static constexpr int kNC = N == 32 ? 4 : N == 64 ? 4 : 8;
    static constexpr int kCPL = N == 32 ? 1 : 2;
    static constexpr int kWarps = N == 32 ? 4 : 8;
    static constexpr int kST = N == 32 ? 64 : N == 64 ? 64 : N == 128 ? 32 : 16;
    static constexpr int kG = N / kNC;             // lanes per channel group: 8, 16, 16, 32
    static constexpr int kGPW = 32 / kG;           // lane groups per warp
    static constexpr int kCPW = kGPW * kCPL;       // channels per warp: 4, 4, 4, 2
    static constexpr int kT = 8;                   // steps per batch
    static constexpr int kCPB = kWarps * kCPW;     // channels per block
    static constexpr int kStageFloats = kST * 2 * N;
    static constexpr int kSmem = 2 * kStageFloats * 4;  // double-buffered stages
};

// Blocks per SM in the launch bound (128 registers per thread at 16 warps per SM).
template <int N>
constexpr int wide_min_blocks() { return N == 32 ? 4 : 2; }

template <typename IO, int N, bool ZOH>
__global__ void __launch_bounds__(WideCfg<N>::kWarps * 32, wide_min_blocks<N>()) scan_fwd_wide_kernel(const WideParams p) {
    using Cfg = WideCfg<N>;
    constexpr int NC = Cfg::kNC, CPL = Cfg::kCPL, G = Cfg::kG, T = Cfg::kT, ST = Cfg::kST;
    static_assert(N == 32 || N == 64 || N == 128 || N == 256, "N in {32, 64, 128, 256}");
    static_assert(ST % T == 0 && G % T == 0 && NC % 4 == 0, "whole batches per stage, 16-byte B/C loads");
    extern __shared__ float4 wide_smem[];
    float* ring = reinterpret_cast<float*>(wide_smem);  // [2][ST][2N]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gi = lane / G, nl = lane % G, gbase = lane & ~(G - 1);
    const int own = nl & (T - 1);  // the lane's step of each batch (all G / T copies hold it)
    const int b = blockIdx.y;
    const long long L = p.L;
    const float* bcrow = p.bc + static_cast<long long>(b) * L * (2 * N);

    int d[CPL];
    bool valid[CPL];
    long long ch[CPL];
    float2 A2[CPL][NC / 2], invA[CPL][ZOH ? NC / 2 : 1], h[CPL][NC / 2];
    float Dd[CPL], bias[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        d[c] = blockIdx.x * Cfg::kCPB + warp * Cfg::kCPW + gi * CPL + c;
        valid[c] = d[c] < p.dim;
        const int dd = valid[c] ? d[c] : 0;
        ch[c] = static_cast<long long>(b) * p.dim + dd;
#pragma unroll
        for (int j = 0; j < NC / 2; ++j) {
            const float a0 = p.A[static_cast<long long>(dd) * N + nl * NC + 2 * j];
            const float a1 = p.A[static_cast<long long>(dd) * N + nl * NC + 2 * j + 1];
            A2[c][j] = make_float2(a0 * kLog2e, a1 * kLog2e);
            if constexpr (ZOH) invA[c][j] = make_float2(1.f / a0, 1.f / a1);
            h[c][j] = (p.h0 && valid[c]) ? *reinterpret_cast<const float2*>(p.h0 + ch[c] * N + nl * NC + 2 * j)
                                         : make_float2(0.f, 0.f);
        }
        Dd[c] = (valid[c] && p.D) ? p.D[dd] : 0.f;
        bias[c] = (valid[c] && p.bias) ? p.bias[dd] : 0.f;
    }
    const bool softplus = p.softplus != 0;
    const IO* zbase = static_cast<const IO*>(p.z);

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
    // Inputs of the lane's own step of a batch for its channels (0 past L), loaded one batch ahead.
    auto load_own = [&](long long t, float (&ul)[CPL], float (&xl)[CPL], float (&zl)[CPL]) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const bool in = valid[c] && t < L;
            ul[c] = in ? IoTraits<IO>::to_f32(static_cast<const IO*>(p.u)[ch[c] * L + t]) : 0.f;
            xl[c] = in ? IoTraits<IO>::to_f32(static_cast<const IO*>(p.delta)[ch[c] * L + t]) : 0.f;
            zl[c] = (in && zbase) ? IoTraits<IO>::to_f32(zbase[ch[c] * L + t]) : 0.f;
        }
    };

    issue(0);
    float un[CPL], xn[CPL], zn[CPL];
    load_own(own, un, xn, zn);
    for (long long k = 0; k < nstages; ++k) {
        issue(k + 1);
        cp_async_wait<1>();
        __syncthreads();  // stage k visible to every warp
        const float* stage = ring + (k & 1) * Cfg::kStageFloats + nl * NC;
#pragma unroll 1
        for (int bt = 0; bt < ST; bt += T) {
            const long long t = k * ST + bt + own;
            float ul[CPL], zl[CPL], dtl[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                ul[c] = un[c];
                zl[c] = zn[c];
                dtl[c] = (valid[c] && t < L) ? step_size(xn[c], bias[c], softplus) : 0.f;  // 0 past L
            }
            load_own(t + T, un, xn, zn);  // next batch (the next stage's first for the last batch)
            float yp[CPL][T];
#pragma unroll
            for (int i = 0; i < T; ++i) {
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
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    const float dti = __shfl_sync(0xffffffffu, dtl[c], gbase | i);
                    const float ui = __shfl_sync(0xffffffffu, ul[c], gbase | i);
                    const float2 dd2 = make_float2(dti, dti), ww = make_float2(dti * ui, dti * ui);
                    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < NC / 2; ++j) {
                        const float2 arg = __fmul2_rn(dd2, A2[c][j]);
                        const float2 a = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                        float2 beta;
                        if constexpr (ZOH)  // phi (u B), phi the hold weight per unit input
                            beta = __fmul2_rn(zoh_phi2(arg, a, dd2, invA[c][j]), __fmul2_rn(make_float2(ui, ui), Bv[j]));
                        else
                            beta = __fmul2_rn(ww, Bv[j]);
                        h[c][j] = __ffma2_rn(a, h[c][j], beta);
                        acc = __ffma2_rn(Cv[j], h[c][j], acc);
                    }
                    yp[c][i] = acc.x + acc.y;
                }
            }
            // Reduce-scatter the T partial sums of each channel over lane bits 2, 1, 0 (upper
            // bit first): lane nl ends with its 8-lane subgroup's sum of step `own` in yp[c][0];
            // then the G / 8 subgroups are added by xor shuffles over the higher lane bits.
#pragma unroll
            for (int m = T / 2; m >= 1; m >>= 1) {
                const bool upper = (nl & m) != 0;
#pragma unroll
                for (int c = 0; c < CPL; ++c)
#pragma unroll
                    for (int i = 0; i < m; ++i) {
                        const float send = upper ? yp[c][i] : yp[c][i + m];
                        const float keep = upper ? yp[c][i + m] : yp[c][i];
                        yp[c][i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                    }
            }
#pragma unroll
            for (int m = T; m < G; m <<= 1)
#pragma unroll
                for (int c = 0; c < CPL; ++c) yp[c][0] += __shfl_xor_sync(0xffffffffu, yp[c][0], m);
            // Epilogue ([Eng] §2.2 D skip; [Hist] SiLU gate): copy q = nl / 8 of step `own`
            // finishes channel q (G >= 16; copies past the channels idle), or the only copy
            // finishes both (G = 8).  (The channel is picked by selects, not by an index.)
            auto finish = [&](float yv, float uv, float zv, float Dv, long long cv) {
                float v = fmaf(Dv, uv, yv);
                if (zbase) v *= silu_f32(zv);
                static_cast<IO*>(p.y)[cv * L + t] = IoTraits<IO>::from_f32(v);
            };
            if constexpr (G / T >= CPL) {
                const int q = nl / T;
                float yv = 0.f, uv = 0.f, zv = 0.f, Dv = 0.f;
                long long cv = 0;
                bool ok = false;
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    if (c == q) {
                        yv = yp[c][0];
                        uv = ul[c];
                        zv = zl[c];
                        Dv = Dd[c];
                        cv = ch[c];
                        ok = valid[c];
                    }
                if (ok && t < L) finish(yv, uv, zv, Dv, cv);
            } else {
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    if (valid[c] && t < L) finish(yp[c][0], ul[c], zl[c], Dd[c], ch[c]);
            }
        }
        __syncthreads();  // every warp is done with slot k & 1 before it is refilled
    }
    cp_async_wait<0>();
    if (p.last_state)
#pragma unroll
        for (int c = 0; c < CPL; ++c)
            if (valid[c])
#pragma unroll
                for (int j = 0; j < NC / 2; ++j)
                    *reinterpret_cast<float2*>(p.last_state + ch[c] * N + nl * NC + 2 * j) = h[c][j];
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
