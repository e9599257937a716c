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
// When the forward stored these checkpoints itself (ssm_fwd_options_t.checkpoints) the
// forward sweep below is skipped and the walk reads them instead.
//
// Work split.  A CTA of 3 warps takes 24 consecutive channels of one batch row; a warp
// takes 8 channels, 4 lanes per channel, each lane 4 of the 16 chains (as the forward
// kernels), with the chain arithmetic in f32x2 pairs.  Each warp first runs the forward
// over the whole sequence and stores the state at the start of every 8-step segment
// (checkpoints, in the workspace).  Then it walks the segments from the last to the
// first: it re-runs the segment from its checkpoint, keeping h_{t-1} of the 8 steps in
// shared memory, forms v_t, dz_t and dv_t, and runs the gradient recurrence backwards
// through the segment (recomputing exp(Delta A): the shared-memory data path, not the
// exponential unit, bounds this kernel).
//   - Sums over the 16 chains (du, dDelta, v) are reduce-scattered over the 4 lanes of a
//     channel, so that lane nl finishes steps 2nl, 2nl+1 of the segment.
//   - Sums over channels (dB, dC) are reduce-scattered over the 8 channels of a warp,
//     added over the CTA's warps in a fixed order, and written per CTA to the
//     workspace; a second kernel adds the CTAs of a batch row (fixed order: the result
//     does not depend on scheduling).
//   - dA, dD and ddelta_bias are summed over time in registers, written per batch row and
//     added over batch rows by the second kernel.
//
// Zero-order hold (ZOH, [Eng] §2.2): the input weight Delta B becomes phi B with
// phi = expm1(Delta A) / A, so that dB_t += g phi u_t, du_t = sum_n g phi B_t + D dv_t,
// dDelta_t = sum_n g (A a_t h_{t-1} + a_t B_t u_t) (dphi/dDelta = a_t) and
// dA_n += g (Delta_t a_t h_{t-1} + dphi/dA B_t u_t) (zoh_dphi_dA2).
//
// Conv prologue (CONV, [Hist] Mamba Block 数据流: x -> conv1d -> SiLU -> S6): the kernel reads x
// and forms u = silu(p), p_t = cb + sum_k w_k x_{t-3+k} (taps right-aligned, rounded to the I/O
// type as the forward rounds it) from a 5-step window of x per lane.  The conv's backward is
// folded into the reverse walk: dp_t = du_t silu'(p_t), and dx_t = sum_k w_k dp_{t+3-k} needs
// dp of steps t .. t+3 -- the lane's own two steps, the next lanes' and, across the segment
// boundary, the first steps of the later segment, which the walk has already finished and
// carries in registers.  dw_k and the conv bias are summed like dD; after step 0 the carried
// dp gives the gradient of the conv's carried-in inputs.  du itself never reaches HBM.
#pragma once

#include "common.cuh"
#include "scan_math.cuh"
#include "scan_fwd_seq.cuh"  // f2

namespace ssm {

constexpr int kBwdSeg = 8;       // steps per segment (checkpoint interval)
constexpr int kBwdWarps = 3;     // warps per CTA: 6 CTAs (18 warps) per SM at 96 registers, so a
                                 // shape's CTAs spread evenly (the headline's 856 give every SM 5
                                 // or 6; 4-warp CTAs gave 48 SMs 5 and 100 SMs 4, idling those)
constexpr int kBwdChannels = kBwdWarps * 8;
constexpr int kBwdRing = 4;      // segments of B/C rows in flight (cp.async ring)
// dynamic shared memory of scan_bwd_kernel: h stage, dB/dC stage, B/C ring (sized for
// fp32 rows; bf16 rows use half of it)
constexpr int kBwdSmem = kBwdWarps * kBwdSeg * 32 * (16 + 4) + kBwdRing * kBwdSeg * 32 * 4;

struct BwdParams {
    const void *u, *delta, *z, *dy;  // (batch, dim, L) IO
    const void* bc;                  // packed B/C rows: fp32 [batch][L][32] (B then C), or for
                                     // bf16 inputs bf16 state pairs (pack_bc_pairs_kernel)
    const float *A, *D, *bias, *h0, *dlast;
    void *du, *ddelta, *dz;          // (batch, dim, L) IO outputs (dz only with z)
    float* dh0;                      // (batch, dim, 16) or null
    float* ckpt;                     // workspace, or the forward's: [batch][nseg][dim][16]
    int ckpt_given;                  // the checkpoints came from the forward: no forward sweep
    float* dbc_part;                 // workspace: [batch][ncta][L][32]  (dB n, then dC n)
    float* dA_part;                  // workspace: [batch][dim][16]
    float* dD_part;                  // workspace: [batch][dim]
    float* dbias_part;               // workspace: [batch][dim]
    // conv prologue (CONV kernels): u holds x
    const float *conv_w, *conv_b;    // (dim, conv_k) oldest tap first; (dim) or null
    const float* conv_in;            // (batch, dim, conv_k - 1): inputs before t = 0, or null (zero)
    const float* dconv_out;          // (batch, dim, conv_k - 1): gradient reaching the carried-out inputs, or null
    float* dconv_in;                 // (batch, dim, conv_k - 1) output, or null
    float* dcw_part;                 // workspace: [batch][dim][4] (taps right-aligned)
    float* dcb_part;                 // workspace: [batch][dim]
    int conv_k;
    int batch, dim;
    long long L;
    int nseg, ncta;
    int softplus;
    WorkspaceHeader* hdr;            // status word (debug range checks)
};

// Two bf16 values packed in a 32-bit word (low half first) as fp32 (exact).
__device__ __forceinline__ float2 bf16_pair(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ float sigmoid_f32(float x) { return __fdividef(1.f, 1.f + ex2_mufu(-x * kLog2e)); }

template <typename IO>
__device__ __forceinline__ float load_io(const void* base, long long i) {
    return IoTraits<IO>::to_f32(static_cast<const IO*>(base)[i]);
}

template <typename IO, bool ZOH, bool CONV>
__global__ void __launch_bounds__(kBwdWarps * 32, 6) scan_bwd_kernel(const BwdParams p) {
    constexpr int T = kBwdSeg, G = 4, PER = T / G, R = kBwdRing;
    extern __shared__ float4 bwd_smem[];
    // h_{t-1} of the segment's steps: [warp][step][lane] (16 bytes each)
    float4* hstage = bwd_smem;
    // per-warp dB/dC partials of the segment's steps: [warp][step][32 columns]
    float* cstage = reinterpret_cast<float*>(bwd_smem + kBwdWarps * T * 32);
    // ring of R segments of packed B/C rows (shared by the CTA: one batch row): [slot][step][RB bytes]
    constexpr int RB = sizeof(IO) == 2 ? 64 : 128;  // bytes of one step's row
    constexpr int CPR = RB / 16;                    // 16-byte chunks per row
    uint8_t* bcring = reinterpret_cast<uint8_t*>(cstage + kBwdWarps * T * 32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cg = lane >> 2, nl = lane & 3, gbase = lane & ~3;
    const int b = blockIdx.y;
    const int d = blockIdx.x * kBwdChannels + warp * 8 + cg;
    const bool valid = d < p.dim;
    const int dd = valid ? d : 0;
    const int L = static_cast<int>(p.L);  // the host launches this kernel for L < 2^31 - 16 only
    const long long row = (static_cast<long long>(b) * p.dim + dd) * p.L;
    const IO* x_row = static_cast<const IO*>(p.delta) + row;
    const IO* u_row = static_cast<const IO*>(p.u) + row;
    const IO* dy_row = static_cast<const IO*>(p.dy) + row;
    const IO* z_row = p.z ? static_cast<const IO*>(p.z) + row : nullptr;
    IO* du_row = static_cast<IO*>(p.du) + row;
    IO* ddelta_row = static_cast<IO*>(p.ddelta) + row;
    IO* dz_row = p.dz ? static_cast<IO*>(p.dz) + row : nullptr;
    const uint8_t* bcrow = static_cast<const uint8_t*>(p.bc) + static_cast<long long>(b) * p.L * RB;
    float* ckrow = p.ckpt + (static_cast<long long>(b) * p.nseg * p.dim + dd) * 16 + nl * 4;  // segment stride dim*16
    const long long ckstride = static_cast<long long>(p.dim) * 16;
    int srcl[4];  // lanes of this channel, by step owner
#pragma unroll
    for (int k = 0; k < 4; ++k) srcl[k] = gbase | k;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.z != nullptr;

    float2 An[2], A2[2], invA[2];  // A of the lane's 4 chains as pairs; A2 = A log2(e); 1 / A (ZOH)
    {
        const float4 a = valid ? *reinterpret_cast<const float4*>(p.A + dd * 16 + nl * 4) : make_float4(0, 0, 0, 0);
        An[0] = f2(a.x, a.y);
        An[1] = f2(a.z, a.w);
        A2[0] = f2(a.x * kLog2e, a.y * kLog2e);
        A2[1] = f2(a.z * kLog2e, a.w * kLog2e);
        if constexpr (ZOH) {
            invA[0] = f2(1.f / a.x, 1.f / a.y);
            invA[1] = f2(1.f / a.z, 1.f / a.w);
        }
    }
    const float Dd = (valid && p.D) ? p.D[dd] : 0.f;
    const float bias = (valid && p.bias) ? p.bias[dd] : 0.f;
    const long long srow = (static_cast<long long>(b) * p.dim + dd) * 16 + nl * 4;  // state row of this lane
    auto ld4 = [](const float* q) { const float4 v = *reinterpret_cast<const float4*>(q); return v; };
    auto lo = [](float4 v) { return f2(v.x, v.y); };
    auto hi = [](float4 v) { return f2(v.z, v.w); };
    auto decay = [&](float dti, int j) {
        const float2 arg = __fmul2_rn(f2(dti, dti), A2[j]);
        return f2(ex2_mufu(arg.x), ex2_mufu(arg.y));
    };
    // input weight times u of chain pair j (per unit B): Delta u, or phi u with the ZOH weight
    // phi formed from a = decay(Delta, j)
    auto weight_u = [&](float dti, float ui, int j, float2 a) {
        if constexpr (ZOH)
            return __fmul2_rn(zoh_phi2(__fmul2_rn(f2(dti, dti), A2[j]), a, f2(dti, dti), invA[j]), f2(ui, ui));
        else return f2(dti * ui, dti * ui);
    };
    // conv taps (right-aligned: tap k of a width-K conv at 4 - K + k) and bias
    float cw[4] = {0.f, 0.f, 0.f, 0.f}, cb = 0.f;
    const int K = CONV ? p.conv_k : 1;
    const long long crow = (static_cast<long long>(b) * p.dim + dd) * (K - 1);  // conv state row
    if constexpr (CONV) {
        if (valid) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k = j - (4 - K);
                cw[j] = k >= 0 ? p.conv_w[static_cast<long long>(dd) * K + k] : 0.f;
            }
            cb = p.conv_b ? p.conv_b[dd] : 0.f;
        }
    }
    auto ckpt_at = [&](int s) { return ckrow + s * ckstride; };
    // B and C of the lane's 4 chains at one step, from the lane's place in a ring row
    // (byte 16 nl: fp32 B there and C 64 bytes on; bf16 pairs (B, C, B, C) there).
    auto load_bc = [&](const uint8_t* r, float2 (&Bv)[2], float2 (&Cv)[2]) {
        if constexpr (sizeof(IO) == 2) {
            const uint4 w = *reinterpret_cast<const uint4*>(r);
            Bv[0] = bf16_pair(w.x); Cv[0] = bf16_pair(w.y); Bv[1] = bf16_pair(w.z); Cv[1] = bf16_pair(w.w);
        } else {
            const float4 Bq = ld4(reinterpret_cast<const float*>(r)), Cq = ld4(reinterpret_cast<const float*>(r + 64));
            Bv[0] = lo(Bq); Bv[1] = hi(Bq); Cv[0] = lo(Cq); Cv[1] = hi(Cq);
        }
    };
    auto load_b = [&](const uint8_t* r, float2 (&Bv)[2]) {
        if constexpr (sizeof(IO) == 2) {
            const uint4 w = *reinterpret_cast<const uint4*>(r);
            Bv[0] = bf16_pair(w.x); Bv[1] = bf16_pair(w.z);
        } else {
            const float4 Bq = ld4(reinterpret_cast<const float*>(r));
            Bv[0] = lo(Bq); Bv[1] = hi(Bq);
        }
    };

    // B/C rows of segment `seg` into ring slot `slot` (threads 0..63, 16 bytes each; zero
    // past L); every thread commits a group, so that group counts agree across threads.
    auto issue_bc = [&](int seg, int slot) {
        if (threadIdx.x < T * CPR && seg >= 0 && seg < p.nseg) {
            const int i = threadIdx.x / CPR, part = threadIdx.x % CPR;
            const int t = seg * T + i;
            const bool in = t < L;
            cp_async_16(bcring + (slot * T + i) * RB + part * 16, in ? bcrow + static_cast<long long>(t) * RB + part * 16 : bcrow,
                        in ? 16u : 0u);
        }
        cp_async_commit();
    };

    // Raw inputs of the lane's own steps 2nl, 2nl+1 of segment seg: delta, u, dy, z.  With the
    // conv, xw holds the conv inputs of steps 2nl-3 .. 2nl+1 (x, the carried-in state before
    // t = 0) and conv_u() forms p and u from them once the loads have landed.
    constexpr int W = CONV ? PER + 3 : 1;
    struct Raw {
        float x[PER], u[PER], dy[PER], z[PER], xw[W], pre[CONV ? PER : 1];
    };
    auto load_raw = [&](int seg, bool with_grad, Raw& r) {
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int t = seg * T + nl * PER + k;
            const bool in = valid && seg >= 0 && t < L;
            r.x[k] = in ? IoTraits<IO>::to_f32(x_row[t]) : 0.f;
            if constexpr (!CONV) r.u[k] = in ? IoTraits<IO>::to_f32(u_row[t]) : 0.f;
            r.dy[k] = (in && with_grad) ? IoTraits<IO>::to_f32(dy_row[t]) : 0.f;
            r.z[k] = (in && with_grad && has_z) ? IoTraits<IO>::to_f32(z_row[t]) : 0.f;
        }
        if constexpr (CONV) {
#pragma unroll
            for (int i = 0; i < W; ++i) {
                const int t = seg * T + nl * PER - 3 + i;
                float v = 0.f;
                if (valid && seg >= 0 && t < L) {
                    if (t >= 0) v = IoTraits<IO>::to_f32(u_row[t]);
                    else if (p.conv_in && t >= -(K - 1)) v = p.conv_in[crow + (K - 1) + t];
                }
                r.xw[i] = v;
            }
        }
    };
    auto conv_u = [&](int seg, Raw& r) {
        if constexpr (CONV) {
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                float pre = cb;
#pragma unroll
                for (int j = 0; j < 4; ++j) pre = fmaf(cw[j], r.xw[k + j], pre);
                const int t = seg * T + nl * PER + k;
                r.pre[k] = pre;
                r.u[k] = (valid && t < L) ? IoTraits<IO>::to_f32(IoTraits<IO>::from_f32(silu_f32(pre))) : 0.f;
            }
        }
    };
    auto step_sizes = [&](int seg, const Raw& r, float (&dt)[PER]) {
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int t = seg * T + nl * PER + k;
            dt[k] = (valid && t < L) ? step_size(r.x[k], bias, softplus) : 0.f;
        }
    };

    // ------------------------------------------------------------ forward sweep, checkpoints
    // (skipped when the forward scan stored them: the checkpoints of ssm_fwd_options_t)
    Raw nxt;
    if (!p.ckpt_given) {
        float2 h[2];
        {
            const float4 h0 = (valid && p.h0) ? ld4(p.h0 + srow) : make_float4(0, 0, 0, 0);
            h[0] = lo(h0);
            h[1] = hi(h0);
        }
        for (int r = 0; r < R - 1; ++r) issue_bc(r, r);
        load_raw(0, false, nxt);
        for (int s = 0; s < p.nseg; ++s) {
            Raw cur = nxt;
            conv_u(s, cur);
            load_raw(s + 1, false, nxt);  // next segment's inputs, in flight during this one
            __syncthreads();              // every warp is done with the slot refilled below
            issue_bc(s + R - 1, (s + R - 1) % R);
            cp_async_wait<R - 1>();
            __syncthreads();              // segment s's B/C rows are visible to every warp
            if (valid && dcheck(p.hdr, s < p.nseg, kSiteBwdCkpt, s))
                *reinterpret_cast<float4*>(ckpt_at(s)) = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
            float dt[PER];
            step_sizes(s, cur, dt);
            const uint8_t* bcs = bcring + (s % R) * T * RB + nl * 16;
#pragma unroll
            for (int i = 0; i < T; ++i) {
                const float dti = __shfl_sync(0xffffffffu, dt[i % PER], srcl[i / PER]);
                const float ui = __shfl_sync(0xffffffffu, cur.u[i % PER], srcl[i / PER]);
                float2 Bv[2];
                load_b(bcs + i * RB, Bv);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float2 a = decay(dti, j);
                    h[j] = __ffma2_rn(a, h[j], __fmul2_rn(weight_u(dti, ui, j, a), Bv[j]));
                }
            }
        }
        cp_async_wait<0>();
        __syncthreads();
    }

    // ------------------------------------------------------------ reverse sweep
    float2 g[2], dA_acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
    {
        const float4 gl = (valid && p.dlast) ? ld4(p.dlast + srow) : make_float4(0, 0, 0, 0);
        g[0] = lo(gl);
        g[1] = hi(gl);
    }
    float dD_acc = 0.f, dbias_acc = 0.f;
    float4* hst = hstage + warp * T * 32;
    float* cst = cstage + warp * T * 32;
    const int col = (cg >> 2) * 16 + nl * 4 + (cg & 3);  // dB/dC column this lane ends with

    // k-th segment of the walk is s = nseg - 1 - k, in ring slot k % R.
    for (int r = 0; r < R - 1; ++r) issue_bc(p.nseg - 1 - r, r);
    load_raw(p.nseg - 1, true, nxt);
    float4 ck_nxt = valid ? ld4(ckpt_at(p.nseg - 1)) : make_float4(0, 0, 0, 0);
    float dpc[PER] = {0.f, 0.f};                       // conv: dp of the lane's steps in the later segment
    float dcw[4] = {0.f, 0.f, 0.f, 0.f}, dcb = 0.f;    // conv: weight and bias gradients (time sums)
    for (int k = 0; k < p.nseg; ++k) {
        const int s = p.nseg - 1 - k;
        const int t0 = s * T;
        Raw cur = nxt;
        conv_u(s, cur);
        const float4 ck = ck_nxt;
        load_raw(s - 1, true, nxt);
        if (valid && s > 0) ck_nxt = ld4(ckpt_at(s - 1));
        __syncthreads();
        issue_bc(s - (R - 1), (k + R - 1) % R);
        cp_async_wait<R - 1>();
        __syncthreads();
        const uint8_t* bcs = bcring + (k % R) * T * RB + nl * 16;
        float dt[PER];
        step_sizes(s, cur, dt);

        // Re-run the segment from its checkpoint: h_{t-1} and exp(Delta A) of each step to
        // shared memory, the lane's part of sum_n C_t h_t per step.
        float2 hs[2] = {lo(ck), hi(ck)};
        float vp[T];
#pragma unroll
        for (int i = 0; i < T; ++i) {
            const float dti = __shfl_sync(0xffffffffu, dt[i % PER], srcl[i / PER]);
            const float ui = __shfl_sync(0xffffffffu, cur.u[i % PER], srcl[i / PER]);
            float2 Bv[2], Cv[2];
            load_bc(bcs + i * RB, Bv, Cv);
            const float2 a0 = decay(dti, 0), a1 = decay(dti, 1);
            hst[i * 32 + lane] = make_float4(hs[0].x, hs[0].y, hs[1].x, hs[1].y);
            hs[0] = __ffma2_rn(a0, hs[0], __fmul2_rn(weight_u(dti, ui, 0, a0), Bv[0]));
            hs[1] = __ffma2_rn(a1, hs[1], __fmul2_rn(weight_u(dti, ui, 1, a1), Bv[1]));
            const float2 acc = __ffma2_rn(Cv[1], hs[1], __fmul2_rn(Cv[0], hs[0]));
            vp[i] = acc.x + acc.y;
        }
        // Reduce-scatter over the 4 lanes (upper lane bit first): lane nl ends with the
        // sums of its own steps 2nl, 2nl+1.
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
        float dv[PER], dzv[PER];
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const float v = fmaf(Dd, cur.u[r], vp[r]);
            if (has_z) {
                const float zt = cur.z[r];
                const float sg = sigmoid_f32(zt);
                dv[r] = cur.dy[r] * zt * sg;
                dzv[r] = cur.dy[r] * v * sg * fmaf(zt, 1.f - sg, 1.f);
            } else {
                dv[r] = cur.dy[r];
                dzv[r] = 0.f;
            }
            dD_acc = fmaf(dv[r], cur.u[r], dD_acc);
        }
        __syncwarp();

        // Gradient recurrence backwards through the segment.
        float2 hn[2] = {hs[0], hs[1]};  // h_t of the step being processed
        float ddt[T], dup[T];
#pragma unroll
        for (int i = T - 1; i >= 0; --i) {
            const float dti = __shfl_sync(0xffffffffu, dt[i % PER], srcl[i / PER]);
            const float ui = __shfl_sync(0xffffffffu, cur.u[i % PER], srcl[i / PER]);
            const float dvi = __shfl_sync(0xffffffffu, dv[i % PER], srcl[i / PER]);
            float2 Bv[2], Cv[2];
            load_bc(bcs + i * RB, Bv, Cv);
            const float4 hq = hst[i * 32 + lane];
            // exp(Delta A) again (the exponential unit has room; the shared-memory path does not)
            const float2 hp[2] = {lo(hq), hi(hq)}, av[2] = {decay(dti, 0), decay(dti, 1)};
            const float2 dv2 = f2(dvi, dvi), dt2 = f2(dti, dti), u2 = f2(ui, ui);
            const float2 w2 = f2(dti * ui, dti * ui);
            float2 sdt = f2(0.f, 0.f), sdu = f2(0.f, 0.f), dB[2], dC[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                g[j] = __ffma2_rn(dv2, Cv[j], g[j]);
                dC[j] = __fmul2_rn(dv2, hn[j]);
                const float2 ah = __fmul2_rn(av[j], hp[j]);
                if constexpr (ZOH) {
                    const float2 y = __fmul2_rn(dt2, A2[j]);
                    const float2 phi = zoh_phi2(y, av[j], dt2, invA[j]);
                    const float2 bu = __fmul2_rn(Bv[j], u2);
                    const float2 dphi = zoh_dphi_dA2(y, av[j], dt2, phi, invA[j]);
                    dA_acc[j] = __ffma2_rn(g[j], __ffma2_rn(dt2, ah, __fmul2_rn(dphi, bu)), dA_acc[j]);
                    sdt = __ffma2_rn(g[j], __ffma2_rn(An[j], ah, __fmul2_rn(av[j], bu)), sdt);
                    sdu = __ffma2_rn(g[j], __fmul2_rn(phi, Bv[j]), sdu);
                    dB[j] = __fmul2_rn(g[j], __fmul2_rn(phi, u2));
                } else {
                    dA_acc[j] = __ffma2_rn(__fmul2_rn(g[j], dt2), ah, dA_acc[j]);
                    sdt = __ffma2_rn(g[j], __ffma2_rn(An[j], ah, __fmul2_rn(Bv[j], u2)), sdt);
                    sdu = __ffma2_rn(g[j], Bv[j], sdu);
                    dB[j] = __fmul2_rn(g[j], w2);
                }
                g[j] = __fmul2_rn(g[j], av[j]);
                hn[j] = hp[j];
            }
            ddt[i] = sdt.x + sdt.y;
            dup[i] = ZOH ? sdu.x + sdu.y : (sdu.x + sdu.y) * dti;
            // dB/dC: reduce-scatter the 8 values over the warp's 8 channels (lane bits 4, 3, 2).
            float vals[8] = {dB[0].x, dB[0].y, dB[1].x, dB[1].y, dC[0].x, dC[0].y, dC[1].x, dC[1].y};
#pragma unroll
            for (int m = 16, half = 4; m >= 4; m >>= 1, half >>= 1) {
                const bool upper = (lane & m) != 0;
#pragma unroll
                for (int q = 0; q < half; ++q) {
                    const float send = upper ? vals[q] : vals[q + half];
                    const float keep = upper ? vals[q + half] : vals[q];
                    vals[q] = keep + __shfl_xor_sync(0xffffffffu, send, m);
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
        // Conv: dp = du silu'(p) of the lane's steps, then dx_t = sum_j cw_j dp_{t+3-j} from the
        // window dp_t .. dp_{t+4}: own steps, the next lane's, the first of the lane after
        // (lanes past the segment's end: their steps of the later segment, carried in dpc).
        float dxv[PER] = {0.f, 0.f};
        if constexpr (CONV) {
            float dp[PER];
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                const int t = t0 + nl * PER + r;
                const float pre = cur.pre[r];
                const float sg = sigmoid_f32(pre);
                dp[r] = (valid && t < L) ? fmaf(Dd, dv[r], dup[r]) * sg * fmaf(pre, 1.f - sg, 1.f) : 0.f;
                dcb += dp[r];
#pragma unroll
                for (int j = 0; j < 4; ++j) dcw[j] = fmaf(dp[r], cur.xw[r + j], dcw[j]);
            }
            const int l1 = gbase | ((nl + 1) & 3), l2 = gbase | ((nl + 2) & 3);
            const float a0 = __shfl_sync(0xffffffffu, dp[0], l1), a1 = __shfl_sync(0xffffffffu, dp[1], l1);
            const float b0 = __shfl_sync(0xffffffffu, dp[0], l2);
            const float c0 = __shfl_sync(0xffffffffu, dpc[0], l1), c1 = __shfl_sync(0xffffffffu, dpc[1], l1);
            const float e0 = __shfl_sync(0xffffffffu, dpc[0], l2);
            const float win[PER + 3] = {dp[0], dp[1], nl + 1 < 4 ? a0 : c0, nl + 1 < 4 ? a1 : c1, nl + 2 < 4 ? b0 : e0};
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) acc = fmaf(cw[j], win[r + 3 - j], acc);
                dxv[r] = acc;
            }
            dpc[0] = dp[0];
            dpc[1] = dp[1];
        }
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int t = t0 + nl * PER + r;
            if (valid && t < L &&
                dcheck(p.hdr, row + t < static_cast<long long>(p.batch) * p.dim * L, kSiteBwdOut, t)) {
                const float dx = softplus ? ddt[r] * sigmoid_f32(cur.x[r] + bias) : ddt[r];
                dbias_acc += dx;
                ddelta_row[t] = IoTraits<IO>::from_f32(dx);
                if constexpr (CONV) {
                    float v = dxv[r];
                    if (p.dconv_out && t >= L - (K - 1)) v += p.dconv_out[crow + t - (L - (K - 1))];
                    du_row[t] = IoTraits<IO>::from_f32(v);  // du holds dx with the conv
                } else {
                    du_row[t] = IoTraits<IO>::from_f32(fmaf(Dd, dv[r], dup[r]));
                }
                if (has_z) dz_row[t] = IoTraits<IO>::from_f32(dzv[r]);
            }
        }

        // CTA sum of the warps' dB/dC partials (fixed order), one row per step.
        __syncthreads();
        for (int q = threadIdx.x; q < T * 32; q += blockDim.x) {
            const int i = q >> 5, c = q & 31;
            const int t = t0 + i;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kBwdWarps; ++w) sum += cstage[(w * T + i) * 32 + c];
            if (t < L && dcheck(p.hdr, blockIdx.x < static_cast<unsigned>(p.ncta) && b < p.batch, kSiteBwdPart, t))
                p.dbc_part[((static_cast<long long>(b) * p.ncta + blockIdx.x) * p.L + t) * 32 + c] = sum;
        }
    }
    cp_async_wait<0>();

    // Per-channel results: d initial_state, and the time sums of dA, dD, ddelta_bias.
    if (valid) {
        if (p.dh0) *reinterpret_cast<float4*>(p.dh0 + srow) = make_float4(g[0].x, g[0].y, g[1].x, g[1].y);
        *reinterpret_cast<float4*>(p.dA_part + srow) = make_float4(dA_acc[0].x, dA_acc[0].y, dA_acc[1].x, dA_acc[1].y);
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
    if constexpr (CONV) {
        // Conv carried-in inputs x_s, s = -3 .. -1: d x_s = sum_j cw_j dp_{s+3-j} over dp_0 .. dp_2
        // (lane nl 0 holds steps 0, 1 and lane 1 step 2 of segment 0 in dpc).
        const float q0 = __shfl_sync(0xffffffffu, dpc[0], gbase), q1 = __shfl_sync(0xffffffffu, dpc[1], gbase);
        const float q2 = __shfl_sync(0xffffffffu, dpc[0], gbase | 1);
#pragma unroll
        for (int m = 1; m <= 2; m <<= 1) {
            dcb += __shfl_xor_sync(0xffffffffu, dcb, m);
#pragma unroll
            for (int j = 0; j < 4; ++j) dcw[j] += __shfl_xor_sync(0xffffffffu, dcw[j], m);
        }
        if (valid && nl == 0) {
            const long long prow = static_cast<long long>(b) * p.dim + dd;
            *reinterpret_cast<float4*>(p.dcw_part + prow * 4) = make_float4(dcw[0], dcw[1], dcw[2], dcw[3]);
            p.dcb_part[prow] = dcb;
            if (p.dconv_in) {
                const float dxs[3] = {cw[0] * q0, fmaf(cw[0], q1, cw[1] * q0), fmaf(cw[0], q2, fmaf(cw[1], q1, cw[2] * q0))};
#pragma unroll
                for (int i = 0; i < 3; ++i) {   // input index s = i - 3
                    const int j = i - (4 - K);  // its place in the carried-in state
                    if (j >= 0) {
                        float v = dxs[i];
                        if (p.dconv_out && i - 3 >= L - (K - 1)) v += p.dconv_out[crow + i - 3 - (L - (K - 1))];
                        p.dconv_in[crow + j] = v;
                    }
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Second pass: the sums over the CTAs of a batch row (dB, dC, transposed to (b, N, L);
// grid (ceil(L / 8), batch)) and over batch rows (dA, dD, ddelta_bias; one thread per
// output), each in a fixed order.
// ---------------------------------------------------------------------------------------
struct BwdFinalParams {
    const float* dbc_part;
    const float *dA_part, *dD_part, *dbias_part;
    float *dB, *dC, *dA, *dD, *dbias;
    const float *dcw_part, *dcb_part;  // conv prologue (conv_k > 0)
    float *dconv_w, *dconv_b;
    int conv_k;
    int batch, dim, ncta;
    long long L;
};

// One output per thread: thread (i, c) of block (x, b) sums the CTAs' rows of step 8x + i,
// column c, in CTA order (independent loads, unrolled, so many are in flight), and writes
// dB[b][c][t] (c < 16) or dC[b][c - 16][t].  grid (ceil(L / 8), batch), 256 threads.
__global__ void __launch_bounds__(256) scan_bwd_reduce_bc_kernel(const BwdFinalParams p) {
    const int b = blockIdx.y;
    const int i = threadIdx.x >> 5, c = threadIdx.x & 31;
    const long long t = static_cast<long long>(blockIdx.x) * 8 + i;
    if (t >= p.L) return;
    const float* src = p.dbc_part + (static_cast<long long>(b) * p.ncta * p.L + t) * 32 + c;
    const long long stride = p.L * 32;  // floats between the rows of consecutive CTAs
    float s = 0.f;
#pragma unroll 8
    for (int j = 0; j < p.ncta; ++j) s += src[j * stride];
    float* dst = c < 16 ? p.dB : p.dC;
    dst[(static_cast<long long>(b) * 16 + (c & 15)) * p.L + t] = s;
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
        if (p.conv_k > 0) {
            float w[4] = {0.f, 0.f, 0.f, 0.f}, cb = 0.f;
            for (int b = 0; b < p.batch; ++b) {
                const long long r = static_cast<long long>(b) * p.dim + i;
                for (int k = 0; k < 4; ++k) w[k] += p.dcw_part[r * 4 + k];
                cb += p.dcb_part[r];
            }
            for (int k = 0; k < p.conv_k; ++k) p.dconv_w[i * p.conv_k + k] = w[4 - p.conv_k + k];
            if (p.dconv_b) p.dconv_b[i] = cb;
        }
    }
}

}  // namespace ssm
