// scan_fwd_seq.cuh -- forward selective scan, "sequential" kernel family.
//
// Each CTA owns R channels of one batch row and walks the whole sequence; the state
// of every (channel, n) chain stays in registers from t = 0 to t = L-1 and only the
// final state is written to HBM ([Eng] §4.2: the state lives on chip and only h_N is
// written back; [S4M] 3.3: state accumulated on chip, written once at the end).
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [S4M]  "State Space Models 深度实战：从 S4 到 Mamba 的架构演进与 CUDA 优化"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
//
// Work split.  G lanes share one channel; lane `nl` of the group holds the NC = 16/G
// chains n = nl*NC .. nl*NC+NC-1 in registers.  Per step each lane computes
//   a = 2^(Delta * A[d,n] * log2 e),  h = a*h + (Delta*u)*B[n],  y_partial += C[n]*h
// and the G partial sums of y_t = sum_n C_t[n] h_t[n] are combined by a shuffle
// reduce-scatter over each 16-byte group of steps, so that every lane finishes the
// epilogue (D skip, silu gate, rounding) of GS/G steps and no work is duplicated.
//
// Staging.  A producer warp streams each stage (TC steps = one 128-byte row per
// channel) of u, delta, z for the CTA's R channels plus the stage's B/C (already
// transposed to fp32 [t][32] in the workspace) into shared memory with TMA, two
// stages deep, signalled through mbarriers.  u/delta/z/y tiles use the 128-byte
// swizzle, so the per-lane 16-byte reads of one column hit distinct banks.
// Outputs go through a per-warp shared-memory tile and a TMA store.
#pragma once

#include "common.cuh"
#include "scan_math.cuh"

namespace ssm {

struct SeqParams {
    const float* A;        // (dim, 16)
    const float* D;        // (dim) or null
    const float* bias;     // (dim) or null
    float* last_state;     // (batch, dim, 16) or null
    WorkspaceHeader* hdr;  // status word
    int batch, dim;
    long long L;
    int tiles_per_batch;
    int softplus;
    int has_z;
    uint32_t wait_limit;
};

__host__ __device__ constexpr int round_up_i(int v, int m) { return (v + m - 1) / m * m; }

template <typename IO, int G, int NW>
struct SeqCfg {
    static constexpr int kNC = 16 / G;                       // chains per lane
    static constexpr int kCW = 32 / G;                       // channels per warp
    static constexpr int kR = NW * kCW;                      // channels per CTA
    static constexpr int kGS = 16 / IoTraits<IO>::kBytes;    // steps per 16-byte group
    static constexpr int kTC = 128 / IoTraits<IO>::kBytes;   // steps per stage
    static constexpr int kNG = kTC / kGS;                    // groups per stage (8)
    static constexpr int kStages = 2;
    static constexpr int kTileLoad = kR * 128;               // bytes one u/delta/z box carries
    static constexpr int kTile = round_up_i(kTileLoad, 1024);
    static constexpr int kBC = kTC * 128;                    // fp32 [TC][32] B/C rows
    static constexpr int kStage = 3 * kTile + round_up_i(kBC, 1024);
    static constexpr int kOutWarp = round_up_i(kCW * 128, 1024);
    static constexpr int kSmem = kStages * kStage + 2 * NW * kOutWarp + 1024;  // +1024: alignment slack
    static constexpr int kThreads = (NW + 1) * 32;           // NW consumer warps + 1 producer warp
    static_assert(G >= 2 && G <= kGS && (16 % G) == 0, "G lanes must split a 16-byte group");
    static_assert(kNC % 2 == 0, "chains are processed in fp32 pairs");
};

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }

// Load N consecutive IO elements (N * sizeof(IO) bytes, naturally aligned) as fp32.
template <typename IO, int N>
__device__ __forceinline__ void load_run(const uint8_t* src, float (&out)[N]) {
    if constexpr (sizeof(IO) == 2 && N == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(src);
        out[0] = __uint_as_float(w.x << 16); out[1] = __uint_as_float(w.x & 0xffff0000u);
        out[2] = __uint_as_float(w.y << 16); out[3] = __uint_as_float(w.y & 0xffff0000u);
    } else if constexpr (sizeof(IO) == 2 && N == 2) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
        out[0] = __uint_as_float(w << 16); out[1] = __uint_as_float(w & 0xffff0000u);
    } else if constexpr (sizeof(IO) == 4 && N == 2) {
        const float2 w = *reinterpret_cast<const float2*>(src);
        out[0] = w.x; out[1] = w.y;
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i)
            out[i] = IoTraits<IO>::to_f32(reinterpret_cast<const IO*>(src)[i]);
    }
}

template <typename IO, int G, int NW>
__global__ void __launch_bounds__((NW + 1) * 32)
scan_fwd_seq_kernel(const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_dl,
                    const __grid_constant__ CUtensorMap map_z, const __grid_constant__ CUtensorMap map_bc,
                    const __grid_constant__ CUtensorMap map_y, const SeqParams p) {
    using Cfg = SeqCfg<IO, G, NW>;
    constexpr int NC = Cfg::kNC, CW = Cfg::kCW, R = Cfg::kR, GS = Cfg::kGS, TC = Cfg::kTC, NG = Cfg::kNG;
    constexpr int S = Cfg::kStages;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[S], empty_bar[S];
    __shared__ int abort_flag;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / p.tiles_per_batch;
    const int d0 = (blockIdx.x % p.tiles_per_batch) * R;
    const int nstages = static_cast<int>((p.L + TC - 1) / TC);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NW);
        }
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();

    // ---------------------------------------------------------------- producer warp
    if (warp == NW) {
        if (lane != 0) return;
        tma_prefetch_map(&map_u);
        tma_prefetch_map(&map_dl);
        tma_prefetch_map(&map_bc);
        if (p.has_z) tma_prefetch_map(&map_z);
        const uint32_t bytes = (p.has_z ? 3u : 2u) * Cfg::kTileLoad + Cfg::kBC;
        for (int k = 0; k < nstages; ++k) {
            const int s = k % S;
            if (k >= S) {
                if (!mbar_wait_bounded(&empty_bar[s], ((k / S) - 1) & 1, p.wait_limit)) {
                    report_status(p.hdr, kDevTimeout, 1, blockIdx.x, k, p.wait_limit);
                    abort_flag = 1;
                    return;
                }
            }
            uint8_t* st = smem + s * Cfg::kStage;
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&full_bar[s], bytes);
            const int t0 = k * TC;
            tma_load_3d(st, &map_u, &full_bar[s], t0, d0, b);
            tma_load_3d(st + Cfg::kTile, &map_dl, &full_bar[s], t0, d0, b);
            if (p.has_z) tma_load_3d(st + 2 * Cfg::kTile, &map_z, &full_bar[s], t0, d0, b);
            tma_load_3d(st + 3 * Cfg::kTile, &map_bc, &full_bar[s], 0, t0, b);
        }
        return;
    }

    // ---------------------------------------------------------------- consumer warps
    const int chw = lane / G;           // channel within the warp
    const int nl = lane % G;            // which NC-chain slice of the channel this lane holds
    const int row = warp * CW + chw;    // channel row within the CTA tile
    const int d = d0 + row;
    const bool valid = d < p.dim;

    float A2[NC];
    float h[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        A2[j] = valid ? p.A[d * 16 + nl * NC + j] * kLog2e : 0.f;
        h[j] = 0.f;
    }
    const float Dd = (valid && p.D) ? p.D[d] : 0.f;
    const float bias = (valid && p.bias) ? p.bias[d] : 0.f;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.has_z != 0;

    for (int k = 0; k < nstages; ++k) {
        const int s = k % S;
        // The outcome of the bounded wait is made warp-uniform, so that a timeout can
        // never leave part of the warp inside the full-mask shuffles below.
        const bool ready = __all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[s], (k / S) & 1, p.wait_limit));
        if (!ready) {
            if (lane == 0) report_status(p.hdr, kDevTimeout, 2, blockIdx.x, k, p.wait_limit);
            break;
        }
        if (__any_sync(0xffffffffu, *(volatile int*)&abort_flag != 0)) break;
        const uint8_t* st = smem + s * Cfg::kStage;
        const uint8_t* tu = st;
        const uint8_t* tdl = st + Cfg::kTile;
        const uint8_t* tz = st + 2 * Cfg::kTile;
        const float* bc = reinterpret_cast<const float*>(st + 3 * Cfg::kTile);
        uint8_t* out = smem + S * Cfg::kStage + (warp * 2 + (k & 1)) * Cfg::kOutWarp;

        // The TMA store issued from this buffer two stages ago must have read it.
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();

        const long long t_stage = static_cast<long long>(k) * TC;
#pragma unroll 1
        for (int g = 0; g < NG; ++g) {
            const int chunk = row * 128 + (g ^ (row & 7)) * 16;
            float uf[GS];
            Group16<IO>::unpack(*reinterpret_cast<const uint4*>(tu + chunk), uf);

            // Step sizes: each of the G lanes evaluates softplus for the PER = GS/G steps
            // i = q*G + nl of the group, then the group exchanges them by shuffles, so every
            // lane has all GS step sizes and no softplus is evaluated twice.
            constexpr int PER = GS / G;
            float mine[PER];
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int i = q * G + nl;
                const float raw = IoTraits<IO>::to_f32(
                    *reinterpret_cast<const IO*>(tdl + chunk + i * IoTraits<IO>::kBytes));
                const long long t = t_stage + g * GS + i;
                mine[q] = (t < p.L) ? step_size(raw, bias, softplus) : 0.f;
            }
            float dt[GS];
#pragma unroll
            for (int i = 0; i < GS; ++i)
                dt[i] = __shfl_sync(0xffffffffu, mine[i / G], (lane & ~(G - 1)) | (i % G), 32);

            float yp[GS];
#pragma unroll
            for (int i = 0; i < GS; ++i) {
                const float* bcr = bc + (g * GS + i) * 32;
                const float w = dt[i] * uf[i];
                const float2 dd = f2(dt[i], dt[i]);
                const float2 ww = f2(w, w);
                float2 acc = f2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < NC; j += 2) {
                    // B and C of chains j, j+1 (8-byte aligned pairs; NC may be 2).
                    const float2 Bp = *reinterpret_cast<const float2*>(bcr + nl * NC + j);
                    const float2 Cp = *reinterpret_cast<const float2*>(bcr + 16 + nl * NC + j);
                    const float2 arg = __fmul2_rn(dd, f2(A2[j], A2[j + 1]));
                    const float2 a = f2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                    const float2 hn = __ffma2_rn(a, f2(h[j], h[j + 1]), __fmul2_rn(ww, Bp));
                    h[j] = hn.x;
                    h[j + 1] = hn.y;
                    acc = __ffma2_rn(Cp, hn, acc);
                }
                yp[i] = acc.x + acc.y;
            }

            // Reduce-scatter the G partial sums: after it, lane nl holds the full
            // y_t for steps nl*PER .. nl*PER+PER-1 of this group in yp[0..PER-1].
#pragma unroll
            for (int m = G / 2, half = GS / 2; m >= 1; m >>= 1, half >>= 1) {
                const bool upper = (nl & m) != 0;
#pragma unroll
                for (int i = 0; i < half; ++i) {
                    const float send = upper ? yp[i] : yp[i + half];
                    const float keep = upper ? yp[i + half] : yp[i];
                    yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, m, 32);
                }
            }

            // Epilogue: D skip and silu gate for this lane's PER steps, rounded to IO.
            float ue[PER], ze[PER];
            load_run<IO, PER>(tu + chunk + nl * PER * IoTraits<IO>::kBytes, ue);
            if (has_z) load_run<IO, PER>(tz + chunk + nl * PER * IoTraits<IO>::kBytes, ze);
            float yo[PER];
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                float v = fmaf(Dd, ue[q], yp[q]);
                if (has_z) v *= silu_f32(ze[q]);
                yo[q] = v;
            }
            uint8_t* orow = out + chw * 128 + ((g ^ (chw & 7)) * 16) + nl * PER * IoTraits<IO>::kBytes;
            if constexpr (sizeof(IO) == 2) {
                if constexpr (PER == 4) {
                    *reinterpret_cast<uint2*>(orow) = make_uint2(pack_bf16x2(yo[0], yo[1]), pack_bf16x2(yo[2], yo[3]));
                } else if constexpr (PER == 2) {
                    *reinterpret_cast<uint32_t*>(orow) = pack_bf16x2(yo[0], yo[1]);
                } else {
                    *reinterpret_cast<__nv_bfloat16*>(orow) = __float2bfloat16_rn(yo[0]);
                }
            } else {
                if constexpr (PER == 2) {
                    *reinterpret_cast<float2*>(orow) = make_float2(yo[0], yo[1]);
                } else {
                    *reinterpret_cast<float*>(orow) = yo[0];
                }
            }
        }

        // Release the input stage to the producer, then store this warp's output tile.
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && d0 + warp * CW < p.dim) {  // a box wholly past `dim` has nothing to store
            tma_store_3d(&map_y, out, static_cast<int>(t_stage), d0 + warp * CW, b);
            bulk_commit();
        }
    }
    if (lane == 0) bulk_wait_all<0>();

    if (valid && p.last_state) {
        float* dst = p.last_state + (static_cast<long long>(b) * p.dim + d) * 16 + nl * NC;
#pragma unroll
        for (int j = 0; j < NC; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(h[j], h[j + 1], h[j + 2], h[j + 3]);
    }
}

}  // namespace ssm
