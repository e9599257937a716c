// scan_bwd.cuh -- backward of the selective scan (gradients of every input), by
// recomputation: the forward is run again instead of storing its states ([Tech] 四.1:
// keep little in the forward pass and rebuild in the backward pass; [S4M] 3.3: the
// state stays on chip, forward and backward in one persistent pass).
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [S4M]  "State Space Models 深度实战：从 S4 到 Mamba 的架构演进与 CUDA 优化"
//   [Tech] "Transformer架构遭遇颠覆性突破：Mamba模型如何用状态空间重新定义序列建模效率？"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
//
// The forward step (per channel b, d and chain n; simplified discretisation, [Card] 离散化变换):
//   Delta_t = softplus(delta_t + bias)      a_t = exp(Delta_t A_n)
//   h_t = a_t h_{t-1} + Delta_t B_t u_t      v_t = sum_n C_t h_t + D u_t      y_t = v_t silu(z_t)
// and, for L = sum dy y + sum dlast h_{L-1}, with g the gradient reaching h_t:
//   dv_t = dy_t silu(z_t)                    dz_t = dy_t v_t silu'(z_t)
//   g += dv_t C_t                            dC_t += dv_t h_t           (summed over channels)
//   dDelta_t = sum_n g (A_n a_t h_{t-1} + B_t u_t)
//   dB_t += g Delta_t u_t                    (summed over channels)
//   du_t = sum_n g Delta_t B_t + D dv_t      dA_n += g Delta_t a_t h_{t-1}
//   g <- a_t g  (the gradient reaching h_{t-1}); after step 0 it is d initial_state
//   ddelta_t = dDelta_t sigmoid(delta_t + bias)   (softplus' ; 1 without softplus)
//
// Work split.  A CTA of 8 warps takes 64 consecutive channels of one batch row; a warp
// takes 8 channels, 4 lanes per channel, each lane 4 of the 16 chains (as the forward
// kernels).  Each warp first runs the forward over the whole sequence and stores the
// state at the start of every 16-step segment (checkpoints, in the workspace).  Then it
// walks the segments from the last to the first: it re-runs the segment from its
// checkpoint, keeping h_{t-1} of the 16 steps in shared memory, forms v_t, dz_t and
// dv_t, and runs the gradient recurrence backwards through the segment.
//   - Sums over the 16 chains (du, dDelta, v) are reduce-scattered over the 4 lanes of a
//     channel, so that lane nl finishes steps 4nl .. 4nl+3 of the segment.
//   - Sums over channels (dB, dC) are reduce-scattered over the 8 channels of a warp,
//     added over the CTA's 8 warps in a fixed order, and written per CTA to the
//     workspace; a second kernel adds the CTAs of a batch row (fixed order: the result
//     does not depend on scheduling).
//   - dA, dD and ddelta_bias are summed over time in registers, written per batch row and
//     added over batch rows by the second kernel.
#pragma once

#include "common.cuh"
#include "scan_math.cuh"

namespace ssm {

constexpr int kBwdSeg = 16;      // steps per segment (checkpoint interval)
constexpr int kBwdWarps = 8;     // warps per CTA
constexpr int kBwdChannels = kBwdWarps * 8;

struct BwdParams {
    const void *u, *delta, *z, *dy;  // (batch, dim, L) IO
    const float* bc;                 // packed B/C rows, fp32 [batch][L][32]
    const float *A, *D, *bias, *h0, *dlast;
    void *du, *ddelta, *dz;          // (batch, dim, L) IO outputs (dz only with z)
    float* dh0;                      // (batch, dim, 16) or null
    float* ckpt;                     // workspace: [batch][nseg][dim][16]
    float* dbc_part;                 // workspace: [batch][ncta][L][32]  (dB n, then dC n)
    float* dA_part;                  // workspace: [batch][dim][16]
    float* dD_part;                  // workspace: [batch][dim]
    float* dbias_part;               // workspace: [batch][dim]
    int batch, dim;
    long long L;
    int nseg, ncta;
    int softplus;
};

__device__ __forceinline__ float sigmoid_f32(float x) { return __fdividef(1.f, 1.f + ex2_mufu(-x * kLog2e)); }

template <typename IO>
__device__ __forceinline__ float load_io(const void* base, long long i) {
    return IoTraits<IO>::to_f32(static_cast<const IO*>(base)[i]);
}

template <typename IO>
__global__ void __launch_bounds__(kBwdWarps * 32, 2) scan_bwd_kernel(const BwdParams p) {
    constexpr int T = kBwdSeg, NC = 4, G = 4, PER = T / G;
    extern __shared__ float4 bwd_smem[];
    // h_{t-1} of the segment's steps: [warp][step][lane] (16 bytes per lane and step)
    float4* hstage = bwd_smem;
    // per-warp dB/dC partials of the segment's steps: [warp][step][32 columns]
    float* cstage = reinterpret_cast<float*>(bwd_smem + kBwdWarps * T * 32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cg = lane >> 2, nl = lane & 3, gbase = lane & ~3;
    const int b = blockIdx.y;
    const int d = blockIdx.x * kBwdChannels + warp * 8 + cg;
    const bool valid = d < p.dim;
    const int dd = valid ? d : 0;
    const long long L = p.L;
    const long long row = (static_cast<long long>(b) * p.dim + dd) * L;
    const float* bcb = p.bc + static_cast<long long>(b) * L * 32 + nl * NC;
    const bool softplus = p.softplus != 0;

    float An[NC], A2[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        An[j] = valid ? p.A[dd * 16 + nl * NC + j] : 0.f;
        A2[j] = An[j] * kLog2e;
    }
    const float Dd = (valid && p.D) ? p.D[dd] : 0.f;
    const float bias = (valid && p.bias) ? p.bias[dd] : 0.f;
    const long long srow = (static_cast<long long>(b) * p.dim + dd) * 16 + nl * NC;  // state row of this lane

    // Step sizes, inputs of the lane's own steps 4nl .. 4nl+3 of segment s (0 past L).
    auto own_inputs = [&](long long t0, float (&dt)[PER], float (&uo)[PER], float (&xo)[PER]) {
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const long long t = t0 + nl * PER + r;
            const bool in = valid && t < L;
            const float raw = in ? load_io<IO>(p.delta, row + t) : 0.f;
            xo[r] = raw + bias;
            dt[r] = in ? step_size(raw, bias, softplus) : 0.f;
            uo[r] = in ? load_io<IO>(p.u, row + t) : 0.f;
        }
    };

    // ------------------------------------------------------------ forward sweep, checkpoints
    float h[NC];
    {
        const float4 h0 = (valid && p.h0) ? *reinterpret_cast<const float4*>(p.h0 + srow) : make_float4(0, 0, 0, 0);
        h[0] = h0.x; h[1] = h0.y; h[2] = h0.z; h[3] = h0.w;
    }
    for (int s = 0; s < p.nseg; ++s) {
        const long long t0 = static_cast<long long>(s) * T;
        if (valid)
            *reinterpret_cast<float4*>(p.ckpt + ((static_cast<long long>(b) * p.nseg + s) * p.dim + dd) * 16 +
                                       nl * NC) = make_float4(h[0], h[1], h[2], h[3]);
        float dt[PER], uo[PER], xo[PER];
        own_inputs(t0, dt, uo, xo);
#pragma unroll
        for (int i = 0; i < T; ++i) {
            const float dti = __shfl_sync(0xffffffffu, dt[i % PER], gbase | (i / PER));
            const float ui = __shfl_sync(0xffffffffu, uo[i % PER], gbase | (i / PER));
            const long long t = t0 + i;
            const float4 Bq = t < L ? *reinterpret_cast<const float4*>(bcb + t * 32) : make_float4(0, 0, 0, 0);
            const float Bv[NC] = {Bq.x, Bq.y, Bq.z, Bq.w};
            const float w = dti * ui;
#pragma unroll
            for (int j = 0; j < NC; ++j) h[j] = fmaf(ex2_mufu(dti * A2[j]), h[j], w * Bv[j]);
        }
    }

    // ------------------------------------------------------------ reverse sweep
    float g[NC];
    {
        const float4 gl = (valid && p.dlast) ? *reinterpret_cast<const float4*>(p.dlast + srow) : make_float4(0, 0, 0, 0);
        g[0] = gl.x; g[1] = gl.y; g[2] = gl.z; g[3] = gl.w;
    }
    float dA_acc[NC] = {0.f, 0.f, 0.f, 0.f};
    float dD_acc = 0.f, dbias_acc = 0.f;
    float4* hst = hstage + warp * T * 32;
    float* cst = cstage + warp * T * 32;
    const int col = (cg >> 2) * 16 + nl * NC + (cg & 3);  // dB/dC column this lane ends with

    for (int s = p.nseg - 1; s >= 0; --s) {
        const long long t0 = static_cast<long long>(s) * T;
        float dt[PER], uo[PER], xo[PER];
        own_inputs(t0, dt, uo, xo);

        // Re-run the segment from its checkpoint: h_{t-1} of each step to shared memory,
        // the lane's part of sum_n C_t h_t per step.
        float hs[NC];
        {
            const float4 c = valid ? *reinterpret_cast<const float4*>(
                                         p.ckpt + ((static_cast<long long>(b) * p.nseg + s) * p.dim + dd) * 16 + nl * NC)
                                   : make_float4(0, 0, 0, 0);
            hs[0] = c.x; hs[1] = c.y; hs[2] = c.z; hs[3] = c.w;
        }
        float vp[T];
#pragma unroll
        for (int i = 0; i < T; ++i) {
            const float dti = __shfl_sync(0xffffffffu, dt[i % PER], gbase | (i / PER));
            const float ui = __shfl_sync(0xffffffffu, uo[i % PER], gbase | (i / PER));
            const long long t = t0 + i;
            float4 Bq = make_float4(0, 0, 0, 0), Cq = make_float4(0, 0, 0, 0);
            if (t < L) {
                Bq = *reinterpret_cast<const float4*>(bcb + t * 32);
                Cq = *reinterpret_cast<const float4*>(bcb + t * 32 + 16);
            }
            hst[i * 32 + lane] = make_float4(hs[0], hs[1], hs[2], hs[3]);
            const float Bv[NC] = {Bq.x, Bq.y, Bq.z, Bq.w}, Cv[NC] = {Cq.x, Cq.y, Cq.z, Cq.w};
            const float w = dti * ui;
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < NC; ++j) {
                hs[j] = fmaf(ex2_mufu(dti * A2[j]), hs[j], w * Bv[j]);
                acc = fmaf(Cv[j], hs[j], acc);
            }
            vp[i] = acc;
        }
        // Reduce-scatter over the 4 lanes: lane nl gets sum_n C h of its steps 4nl.. 4nl+3.
#pragma unroll
        for (int m = 2, half = T / 2; m >= 1; m >>= 1, half >>= 1) {
            const bool upper = (nl & m) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = upper ? vp[i] : vp[i + half];
                const float keep = upper ? vp[i + half] : vp[i];
                vp[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        // vp[r] now belongs to step 4*nl' + r, nl' = the lane's position after the
        // scatter: lower half -> first half of the steps.  With the upper bit taken first
        // (m = 2: steps 8..15 to lanes 2,3), then m = 1, lane nl holds steps nl*4 + r.
        float dv[PER], dzv[PER];
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const long long t = t0 + nl * PER + r;
            const bool in = valid && t < L;
            const float v = fmaf(Dd, uo[r], vp[r]);
            const float dyv = in ? load_io<IO>(p.dy, row + t) : 0.f;
            if (p.z) {
                const float zt = in ? load_io<IO>(p.z, row + t) : 0.f;
                const float sg = sigmoid_f32(zt);
                dv[r] = dyv * zt * sg;
                dzv[r] = dyv * v * sg * fmaf(zt, 1.f - sg, 1.f);
            } else {
                dv[r] = dyv;
                dzv[r] = 0.f;
            }
            dD_acc = fmaf(dv[r], uo[r], dD_acc);
        }
        __syncwarp();

        // Gradient recurrence backwards through the segment.
        float hn[NC] = {hs[0], hs[1], hs[2], hs[3]};  // h_t of the step being processed
        float ddt[T], dup[T];
#pragma unroll
        for (int i = T - 1; i >= 0; --i) {
            const float dti = __shfl_sync(0xffffffffu, dt[i % PER], gbase | (i / PER));
            const float ui = __shfl_sync(0xffffffffu, uo[i % PER], gbase | (i / PER));
            const float dvi = __shfl_sync(0xffffffffu, dv[i % PER], gbase | (i / PER));
            const long long t = t0 + i;
            float4 Bq = make_float4(0, 0, 0, 0), Cq = make_float4(0, 0, 0, 0);
            if (t < L) {
                Bq = *reinterpret_cast<const float4*>(bcb + t * 32);
                Cq = *reinterpret_cast<const float4*>(bcb + t * 32 + 16);
            }
            const float Bv[NC] = {Bq.x, Bq.y, Bq.z, Bq.w}, Cv[NC] = {Cq.x, Cq.y, Cq.z, Cq.w};
            const float4 hq = hst[i * 32 + lane];
            const float hp[NC] = {hq.x, hq.y, hq.z, hq.w};
            const float w = dti * ui;
            float vals[2 * NC];  // dB (this channel's part) then dC
            float sdt = 0.f, sdu = 0.f;
#pragma unroll
            for (int j = 0; j < NC; ++j) {
                const float a = ex2_mufu(dti * A2[j]);
                g[j] = fmaf(dvi, Cv[j], g[j]);
                vals[NC + j] = dvi * hn[j];
                const float ah = a * hp[j];
                dA_acc[j] = fmaf(g[j] * dti, ah, dA_acc[j]);
                sdt = fmaf(g[j], fmaf(An[j], ah, Bv[j] * ui), sdt);
                sdu = fmaf(g[j], Bv[j], sdu);
                vals[j] = g[j] * w;
                g[j] *= a;
                hn[j] = hp[j];
            }
            ddt[i] = sdt;
            dup[i] = sdu * dti;
            // dB/dC: reduce-scatter the 8 values over the warp's 8 channels (lane bits 4, 3, 2).
#pragma unroll
            for (int m = 16, half = NC; m >= 4; m >>= 1, half >>= 1) {
                const bool upper = (lane & m) != 0;
#pragma unroll
                for (int k = 0; k < half; ++k) {
                    const float send = upper ? vals[k] : vals[k + half];
                    const float keep = upper ? vals[k + half] : vals[k];
                    vals[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            cst[i * 32 + col] = vals[0];
        }
        // Reduce-scatter dDelta and du over the 4 lanes of the channel (as vp above).
#pragma unroll
        for (int m = 2, half = T / 2; m >= 1; m >>= 1, half >>= 1) {
            const bool upper = (nl & m) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float s1 = upper ? ddt[i] : ddt[i + half];
                const float k1 = upper ? ddt[i + half] : ddt[i];
                const float s2 = upper ? dup[i] : dup[i + half];
                const float k2 = upper ? dup[i + half] : dup[i];
                ddt[i] = k1 + __shfl_xor_sync(0xffffffffu, s1, m);
                dup[i] = k2 + __shfl_xor_sync(0xffffffffu, s2, m);
            }
        }
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const long long t = t0 + nl * PER + r;
            if (valid && t < L) {
                const float dx = softplus ? ddt[r] * sigmoid_f32(xo[r]) : ddt[r];
                dbias_acc += dx;
                static_cast<IO*>(p.ddelta)[row + t] = IoTraits<IO>::from_f32(dx);
                static_cast<IO*>(p.du)[row + t] = IoTraits<IO>::from_f32(fmaf(Dd, dv[r], dup[r]));
                if (p.z) static_cast<IO*>(p.dz)[row + t] = IoTraits<IO>::from_f32(dzv[r]);
            }
        }

        // CTA sum of the warps' dB/dC partials (fixed order), one row per step.
        __syncthreads();
        for (int k = threadIdx.x; k < T * 32; k += blockDim.x) {
            const int i = k >> 5, c = k & 31;
            const long long t = t0 + i;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kBwdWarps; ++w) sum += cstage[(w * T + i) * 32 + c];
            if (t < L)
                p.dbc_part[((static_cast<long long>(b) * p.ncta + blockIdx.x) * L + t) * 32 + c] = sum;
        }
        __syncthreads();
    }

    // Per-channel results: d initial_state, and the time sums of dA, dD, ddelta_bias.
    if (valid) {
        if (p.dh0) *reinterpret_cast<float4*>(p.dh0 + srow) = make_float4(g[0], g[1], g[2], g[3]);
        *reinterpret_cast<float4*>(p.dA_part + srow) = make_float4(dA_acc[0], dA_acc[1], dA_acc[2], dA_acc[3]);
    }
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
        dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, m);
        dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, m);
    }
    if (valid && nl == 0) {
        p.dD_part[static_cast<long long>(b) * p.dim + dd] = dD_acc;
        p.dbias_part[static_cast<long long>(b) * p.dim + dd] = dbias_acc;
    }
}

// ---------------------------------------------------------------------------------------
// Second kernel: the sums over the CTAs of a batch row (dB, dC, transposed to (b, N, L))
// and over batch rows (dA, dD, ddelta_bias), in a fixed order.
// grid.x = ceil(L / 32) time tiles, grid.y = batch; 256 threads.  Block (0, 0) extra work
// is avoided: dA/dD/dbias are done by a separate small launch of the same kernel with
// grid.y = 0 semantics handled by `param_pass`.
// ---------------------------------------------------------------------------------------
struct BwdFinalParams {
    const float* dbc_part;
    const float *dA_part, *dD_part, *dbias_part;
    float *dB, *dC, *dA, *dD, *dbias;
    int batch, dim, ncta;
    long long L;
};

__global__ void __launch_bounds__(256) scan_bwd_reduce_bc_kernel(const BwdFinalParams p) {
    __shared__ float tile[32][33];
    const int b = blockIdx.y;
    const long long t0 = static_cast<long long>(blockIdx.x) * 32;
    // threads: (t local, column) with column fastest for coalesced partial reads
    for (int k = threadIdx.x; k < 32 * 32; k += blockDim.x) {
        const int tl = k >> 5, c = k & 31;
        const long long t = t0 + tl;
        float s = 0.f;
        if (t < p.L)
            for (int j = 0; j < p.ncta; ++j) s += p.dbc_part[((static_cast<long long>(b) * p.ncta + j) * p.L + t) * 32 + c];
        tile[c][tl] = s;
    }
    __syncthreads();
    // write rows of 32 steps: dB[b][n][t0..] (c < 16) and dC[b][n][t0..] (c >= 16)
    for (int k = threadIdx.x; k < 32 * 32; k += blockDim.x) {
        const int c = k >> 5, tl = k & 31;
        const long long t = t0 + tl;
        if (t < p.L) {
            float* dst = c < 16 ? p.dB : p.dC;
            dst[(static_cast<long long>(b) * 16 + (c & 15)) * p.L + t] = tile[c][tl];
        }
    }
}

__global__ void __launch_bounds__(256) scan_bwd_reduce_params_kernel(const BwdFinalParams p) {
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < static_cast<long long>(p.dim) * 16) {
        float s = 0.f;
        for (int b = 0; b < p.batch; ++b) s += p.dA_part[static_cast<long long>(b) * p.dim * 16 + i];
        p.dA[i] = s;
    }
    if (i < p.dim) {
        float sd = 0.f, sb = 0.f;
        for (int b = 0; b < p.batch; ++b) {
            sd += p.dD_part[static_cast<long long>(b) * p.dim + i];
            sb += p.dbias_part[static_cast<long long>(b) * p.dim + i];
        }
        if (p.dD) p.dD[i] = sd;
        if (p.dbias) p.dbias[i] = sb;
    }
}

}  // namespace ssm
