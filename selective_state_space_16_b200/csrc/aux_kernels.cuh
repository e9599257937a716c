// aux_kernels.cuh -- the kernels around the main forward scans:
//   pack_bc_kernel      B, C (batch, 16, L) -> fp32 [batch][L][32] rows (B then C), so a
//                       step's 16 B and 16 C values are one 128-byte row for broadcast reads;
//   pack_bc_pairs_kernel bf16 B, C -> bf16 rows ordered by state pairs (the backward's
//                       shared-memory ring: half the bytes per step);
//   scan_fwd_direct     forward scan with direct global loads, for any seqlen / alignment;
//   state_update_kernel the one-token decode step, fp32 state read-modified-written in place.
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
#pragma once

#include "common.cuh"
#include "scan_math.cuh"

namespace ssm {

// ---------------------------------------------------------------------------------------
// B/C transpose into the workspace.  grid = (ceil(L/64), batch), 256 threads.
// ---------------------------------------------------------------------------------------
template <typename IO>
__global__ void __launch_bounds__(256) pack_bc_kernel(const IO* __restrict__ B, const IO* __restrict__ C,
                                                      float* __restrict__ bc, long long L, WorkspaceHeader* hdr) {
    pdl_launch_dependents();  // the scan may start its prologue; it waits for these rows before loading them
    __shared__ float tile[32][65];
    const int b = blockIdx.y;
    const long long t0 = static_cast<long long>(blockIdx.x) * 64;
    for (int idx = threadIdx.x; idx < 32 * 64; idx += 256) {
        const int r = idx >> 6, c = idx & 63;
        const long long t = t0 + c;
        const IO* src = (r < 16) ? B : C;
        tile[r][c] = (t < L) ? IoTraits<IO>::to_f32(src[(static_cast<long long>(b) * 16 + (r & 15)) * L + t]) : 0.f;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 32 * 64; idx += 256) {
        const int c = idx >> 5, r = idx & 31;
        const long long t = t0 + c;
        if (t < L && dcheck(hdr, (static_cast<long long>(b) * L + t) * 32 + r < static_cast<long long>(gridDim.y) * L * 32,
                            kSitePack, t))
            bc[(static_cast<long long>(b) * L + t) * 32 + r] = tile[r][c];
    }
}

// The same transpose for bf16 inputs, kept in bf16 (exact) and ordered by state pairs:
// [batch][L][16] 32-bit words, word 2j = (B_2j, B_2j+1), word 2j+1 = (C_2j, C_2j+1) (low
// half the even state), so the B and C values of a lane's chains at one step are one
// contiguous vector and a step's row is 64 bytes.  grid = (ceil(L/64), batch), 256 threads.
__global__ void __launch_bounds__(256) pack_bc_pairs_kernel(const uint16_t* __restrict__ B,
                                                            const uint16_t* __restrict__ C,
                                                            uint32_t* __restrict__ bc, long long L) {
    __shared__ uint16_t tile[32][66];
    const int b = blockIdx.y;
    const long long t0 = static_cast<long long>(blockIdx.x) * 64;
    for (int idx = threadIdx.x; idx < 32 * 64; idx += 256) {
        const int r = idx >> 6, c = idx & 63;
        const long long t = t0 + c;
        const uint16_t* src = (r < 16) ? B : C;
        tile[r][c] = (t < L) ? src[(static_cast<long long>(b) * 16 + (r & 15)) * L + t] : uint16_t(0);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 16 * 64; idx += 256) {
        const int c = idx >> 4, k = idx & 15;
        const long long t = t0 + c;
        const int r = (k & 1) * 16 + (k >> 1) * 2;  // first row of the word's pair
        if (t < L)
            bc[(static_cast<long long>(b) * L + t) * 16 + k] =
                static_cast<uint32_t>(tile[r][c]) | (static_cast<uint32_t>(tile[r + 1][c]) << 16);
    }
}

// ---------------------------------------------------------------------------------------
// Rows of `rows` x L elements (L * sizeof(IO) not a multiple of 16) copied into rows of Lp
// elements (Lp * sizeof(IO) a multiple of 16, zero past L), so that TMA can address them;
// up to three arrays at once (blockIdx.y selects the array).  One thread per 16-byte chunk
// of an output row: the chunk's 16 source bytes start at a 2-byte (bf16) or 4-byte (fp32)
// aligned address and are assembled from the two aligned 16-byte words that hold them
// (byte_perm funnel); at the end of a row or of the source array (where the second word
// could lie past it), element by element.  Measured on B200 at ~4 TB/s of read + write:
// 118 us for the three 84 MB arrays of batch 4, d_inner 5120, L 2047.
// ---------------------------------------------------------------------------------------
struct PadArrays {
    const void* src[3];
    void* dst[3];
};

template <typename IO>
__device__ __forceinline__ uint4 pad_chunk(const IO* __restrict__ src, long long r, long long t0, long long L,
                                           long long n_src, uint4 w0, uint4 w1, bool fast) {
    constexpr int E = 16 / sizeof(IO);
    if (fast) {
        const uint32_t sh = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(src + r * L + t0) & 15u);
        const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const uint32_t k = sh >> 2;  // whole words to skip (0 .. 3)
        uint32_t sw[5];              // words k .. k+4
#pragma unroll
        for (int m = 0; m < 5; ++m) sw[m] = k == 0 ? w[m] : k == 1 ? w[m + 1] : k == 2 ? w[m + 2] : w[m + 3];
        // with a 2-byte remainder each output word is the upper half of one word and the lower
        // half of the next
        const uint32_t sel = (sh & 3u) ? 0x5432u : 0x3210u;
        return make_uint4(__byte_perm(sw[0], sw[1], sel), __byte_perm(sw[1], sw[2], sel),
                          __byte_perm(sw[2], sw[3], sel), __byte_perm(sw[3], sw[4], sel));
    }
    // row end (or array end): element by element, zero past L
    __align__(16) IO v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = (t0 + e < L && r * L + t0 + e < n_src) ? src[r * L + t0 + e] : IoTraits<IO>::from_f32(0.f);
    return *reinterpret_cast<const uint4*>(v);
}

template <typename IO>
__global__ void __launch_bounds__(256) pad_rows_kernel(const PadArrays arrays, long long rows, long long L,
                                                       long long Lp) {
    constexpr int E = 16 / sizeof(IO);  // elements per 16-byte chunk
    const IO* __restrict__ src = static_cast<const IO*>(arrays.src[blockIdx.y]);
    uint4* __restrict__ dst = static_cast<uint4*>(arrays.dst[blockIdx.y]);
    const long long cpr = Lp / E;       // chunks per output row
    const long long total = rows * cpr;
    const long long n_src = rows * L;
    for (long long q = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; q < total;
         q += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long r = q / cpr;
        const long long t0 = (q - r * cpr) * E;
        const long long s0 = r * L + t0;  // first source element of the chunk
        uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
        const bool fast = t0 + E <= L && s0 + 2 * E <= n_src;
        if (fast) {
            const uint4* wp = reinterpret_cast<const uint4*>(reinterpret_cast<uintptr_t>(src + s0) & ~uintptr_t(15));
            w0 = __ldg(wp);
            w1 = __ldg(wp + 1);
        }
        dst[q] = pad_chunk<IO>(src, r, t0, L, n_src, w0, w1, fast);
    }
}

// ---------------------------------------------------------------------------------------
// Direct-load forward scan (fallback for seqlen whose rows are not 16-byte multiples).
// G lanes per channel, NC = 16/G chains per lane, 128 threads per block.
// Per step: h = exp(Delta A) h + Delta B u; y = C.h + D u; y *= silu(z)
// ([Card] 选择性机制 and Python 演示; [Hist] Mamba Block 数据流).
// ---------------------------------------------------------------------------------------
struct DirectParams {
    const void* u;
    const void* delta;
    const void* z;
    const float* bc;       // packed [batch][L][32]
    const float* A;
    const float* D;
    const float* bias;
    const float* h0;       // (batch, dim, 16) initial state or null (zero)
    void* y;
    float* last_state;
    int batch, dim;
    long long L;
    int softplus;
    int zoh;  // zero-order-hold input weight instead of Delta*B
    // causal conv1d + SiLU prologue (conv_k > 0): u = silu(conv(x)), x given in `u`
    const float* conv_w;   // (dim, conv_k), oldest tap first
    const float* conv_b;   // (dim) or null
    const float* conv_in;  // (batch, dim, conv_k - 1) or null
    float* conv_out;       // (batch, dim, conv_k - 1) or null
    void* u_out;           // (batch, dim, L) IO or null
    int conv_k;            // 0: no conv
    WorkspaceHeader* hdr;  // status word (debug range checks)
};

template <typename IO, int G>
__global__ void __launch_bounds__(128) scan_fwd_direct_kernel(const DirectParams p) {
    constexpr int NC = 16 / G;
    const int lane = threadIdx.x & 31;
    const int nl = lane % G;
    const long long ch = (static_cast<long long>(blockIdx.x) * 128 + threadIdx.x) / G;  // flat (b, d)
    const bool valid = ch < static_cast<long long>(p.batch) * p.dim;
    const int b = valid ? static_cast<int>(ch / p.dim) : 0;
    const int d = valid ? static_cast<int>(ch % p.dim) : 0;

    const IO* u = static_cast<const IO*>(p.u) + ch * p.L;
    const IO* dl = static_cast<const IO*>(p.delta) + ch * p.L;
    const IO* z = p.z ? static_cast<const IO*>(p.z) + ch * p.L : nullptr;
    IO* y = static_cast<IO*>(p.y) + ch * p.L;
    const float* bcb = p.bc + static_cast<long long>(b) * p.L * 32;

    float A2[NC], invA[NC], h[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        const float a = valid ? p.A[d * 16 + nl * NC + j] : 0.f;
        A2[j] = a * kLog2e;
        invA[j] = 1.f / a;
        h[j] = (valid && p.h0) ? p.h0[ch * 16 + nl * NC + j] : 0.f;
    }
    const float Dd = (valid && p.D) ? p.D[d] : 0.f;
    const float bias = (valid && p.bias) ? p.bias[d] : 0.f;
    // conv prologue: taps right-aligned in cw, the last three inputs in xh (oldest first)
    const int K = p.conv_k;
    float cw[4] = {0.f, 0.f, 0.f, 0.f}, xh[3] = {0.f, 0.f, 0.f};
    const float cb = (K > 0 && valid && p.conv_b) ? p.conv_b[d] : 0.f;
    if (K > 0 && valid) {
        for (int k = 0; k < K; ++k) cw[4 - K + k] = p.conv_w[d * K + k];
        if (p.conv_in)
            for (int k = 0; k < K - 1; ++k) xh[3 - (K - 1) + k] = p.conv_in[ch * (K - 1) + k];
    }

    for (long long t = 0; t < p.L; ++t) {
        float ut = 0.f, dt = 0.f;
        if (valid) {
            ut = IoTraits<IO>::to_f32(u[t]);
            dt = step_size(IoTraits<IO>::to_f32(dl[t]), bias, p.softplus != 0);
            if (K > 0) {  // u = silu(conv(x)) rounded to the I/O type, as a separate conv kernel would store it
                const float xt = ut;
                const float pre = fmaf(cw[3], xt, fmaf(cw[2], xh[2], fmaf(cw[1], xh[1], fmaf(cw[0], xh[0], cb))));
                xh[0] = xh[1];
                xh[1] = xh[2];
                xh[2] = xt;
                ut = IoTraits<IO>::to_f32(IoTraits<IO>::from_f32(silu_f32(pre)));
                if (p.u_out && nl == 0) static_cast<IO*>(p.u_out)[ch * p.L + t] = IoTraits<IO>::from_f32(ut);
            }
        }
        const float w = dt * ut;
        const float* row = dcheck(p.hdr, (static_cast<long long>(b) * p.L + t) * 32 + 32 <= static_cast<long long>(p.batch) * p.L * 32,
                                  kSiteDirect, t)
                               ? bcb + t * 32
                               : p.bc;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            const float y = dt * A2[j];
            const float a = ex2_mufu(y);
            const float Bn = row[nl * NC + j];
            const float beta = p.zoh ? zoh_beta(y, a, w * Bn, ut * Bn * invA[j]) : w * Bn;
            h[j] = fmaf(a, h[j], beta);
            acc = fmaf(row[16 + nl * NC + j], h[j], acc);
        }
#pragma unroll
        for (int m = G / 2; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m, 32);
        if (valid && nl == 0 && dcheck(p.hdr, ch * p.L + t < static_cast<long long>(p.batch) * p.dim * p.L, kSiteDirect, t)) {
            float v = fmaf(Dd, ut, acc);
            if (z) v *= silu_f32(IoTraits<IO>::to_f32(z[t]));
            y[t] = IoTraits<IO>::from_f32(v);
        }
    }
    if (valid && p.last_state &&
        dcheck(p.hdr, ch * 16 + nl * NC + NC <= static_cast<long long>(p.batch) * p.dim * 16, kSiteDirect, ch)) {
        float* dst = p.last_state + ch * 16 + nl * NC;
#pragma unroll
        for (int j = 0; j < NC; ++j) dst[j] = h[j];
    }
    if (K > 1 && valid && p.conv_out && nl == 0)
        for (int k = 0; k < K - 1; ++k) p.conv_out[ch * (K - 1) + k] = xh[3 - (K - 1) + k];
}

// ---------------------------------------------------------------------------------------
// One-token decode ([Card] 线性扫描算法: one fixed-size state update per token;
// [Eng] §6.3: the states of a batch laid out on contiguous threads).
// TPC = 16 / NS threads per (b, d) channel, each owning NS consecutive fp32 state values
// (NS / 4 16-byte vectors), so a warp reads and writes contiguous state.  grid.y is the
// batch row (B and C are the same for the whole CTA), grid.x covers dim.
// ---------------------------------------------------------------------------------------
struct DecodeParams {
    float* state;
    const void* u;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    const float* bias;
    void* y;
    int batch, dim;
    int softplus;
    int zoh;     // zero-order-hold input weight instead of Delta*B
    int bc_vec;  // B and C 16-byte aligned: vector loads
    // causal conv1d + SiLU (conv_k > 0): u = silu(conv([conv_state, x])), x given in `u`;
    // conv_state (batch, dim, conv_k - 1) fp32, oldest first, shifted in place
    const float* conv_w;
    const float* conv_b;
    float* conv_state;
    int conv_k;
};

// NS consecutive IO values at src (index in elements) as fp32; `vec`: src is 2*NS- (bf16)
// or 4*NS-byte aligned (NS = 4, 8 or 16), else element loads.
template <typename IO, int NS>
__device__ __forceinline__ void decode_load(const IO* src, bool vec, float (&out)[NS]) {
    if (vec) {
        if constexpr (sizeof(IO) == 2) {
            uint32_t w[NS / 2];
            if constexpr (NS == 4) {
                const uint2 v = *reinterpret_cast<const uint2*>(src);
                w[0] = v.x; w[1] = v.y;
            } else {
#pragma unroll
                for (int k = 0; k < NS / 8; ++k) {
                    const uint4 v = reinterpret_cast<const uint4*>(src)[k];
                    w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
                }
            }
#pragma unroll
            for (int k = 0; k < NS / 2; ++k) {
                out[2 * k] = __uint_as_float(w[k] << 16);
                out[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
            }
        } else {
#pragma unroll
            for (int k = 0; k < NS / 4; ++k) {
                const float4 v = reinterpret_cast<const float4*>(src)[k];
                out[4 * k] = v.x; out[4 * k + 1] = v.y; out[4 * k + 2] = v.z; out[4 * k + 3] = v.w;
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < NS; ++k) out[k] = IoTraits<IO>::to_f32(src[k]);
    }
}

// ZOH and CONV are template flags so that the plain step carries none of their registers.
// 64-thread CTAs, at most 40 registers for the plain step (24 CTAs = 48 warps per SM):
// measured on B200 (b256 d5120, 1000 chained steps) 33.6 us per step, against 34.4 with
// 128-thread CTAs and 35.0 with 256 at the same bound, 37.5 with 256 threads and 42
// registers (40 warps) and 41.0 with 32 registers (spills).
constexpr int kDecodeThreads = 64;
template <typename IO, bool ZOH, bool CONV, int NS>
__global__ void __launch_bounds__(kDecodeThreads, (ZOH || CONV) ? 16 : 24) state_update_kernel(const DecodeParams p) {
    constexpr int TPC = 16 / NS;
    const int b = blockIdx.y;
    const int tl = blockIdx.x * kDecodeThreads + threadIdx.x;
    const int d = tl / TPC, q = tl % TPC;
    const bool valid = d < p.dim;
    const int dd = valid ? d : p.dim - 1;
    const long long rr = static_cast<long long>(b) * p.dim + dd;  // flat (b, d)

    // every load first (state from HBM, the rest mostly from L2), then the arithmetic
    float hs[NS], as[NS], Bq[NS], Cq[NS];
#pragma unroll
    for (int k = 0; k < NS / 4; ++k) {
        const float4 h4 = reinterpret_cast<const float4*>(p.state + rr * 16 + q * NS)[k];
        const float4 a4 = reinterpret_cast<const float4*>(p.A + dd * 16 + q * NS)[k];
        hs[4 * k] = h4.x; hs[4 * k + 1] = h4.y; hs[4 * k + 2] = h4.z; hs[4 * k + 3] = h4.w;
        as[4 * k] = a4.x; as[4 * k + 1] = a4.y; as[4 * k + 2] = a4.z; as[4 * k + 3] = a4.w;
    }
    const bool vec = p.bc_vec != 0;
    decode_load<IO, NS>(static_cast<const IO*>(p.B) + b * 16 + q * NS, vec, Bq);
    decode_load<IO, NS>(static_cast<const IO*>(p.C) + b * 16 + q * NS, vec, Cq);
    float ut = IoTraits<IO>::to_f32(static_cast<const IO*>(p.u)[rr]);
    const float raw = IoTraits<IO>::to_f32(static_cast<const IO*>(p.delta)[rr]);
    const float zt = p.z ? IoTraits<IO>::to_f32(static_cast<const IO*>(p.z)[rr]) : 0.f;
    const float bias = p.bias ? p.bias[dd] : 0.f;
    const float Dd = p.D ? p.D[dd] : 0.f;
    float xt = 0.f;
    if constexpr (CONV) {  // u = silu(conv([conv_state, x])), rounded to the I/O type
        const int K = p.conv_k;
        xt = ut;
        float pre = p.conv_b ? p.conv_b[dd] : 0.f;
        for (int k = 0; k < K - 1; ++k) pre = fmaf(p.conv_w[dd * K + k], p.conv_state[rr * (K - 1) + k], pre);
        pre = fmaf(p.conv_w[dd * K + K - 1], xt, pre);
        ut = IoTraits<IO>::to_f32(IoTraits<IO>::from_f32(silu_f32(pre)));
    }
    const float dt = step_size(raw, bias, p.softplus != 0);
    const float w = dt * ut;
    const float dl = dt * kLog2e;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < NS; ++j) {
        const float y = dl * as[j];
        const float a = ex2_mufu(y);
        float beta = w * Bq[j];
        if constexpr (ZOH) beta = zoh_beta(y, a, beta, ut * Bq[j] / as[j]);
        hs[j] = fmaf(a, hs[j], beta);
        acc = fmaf(Cq[j], hs[j], acc);
    }
#pragma unroll
    for (int m = 1; m < TPC; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m, 32);
    if constexpr (CONV) {
        if (p.conv_k > 1) {
            __syncwarp();  // every thread of the channel has read conv_state
            if (valid && q == 0) {
                const int K = p.conv_k;
                for (int k = 0; k < K - 2; ++k) p.conv_state[rr * (K - 1) + k] = p.conv_state[rr * (K - 1) + k + 1];
                p.conv_state[rr * (K - 1) + K - 2] = xt;
            }
        }
    }
    if (valid) {
#pragma unroll
        for (int k = 0; k < NS / 4; ++k)
            reinterpret_cast<float4*>(p.state + rr * 16 + q * NS)[k] =
                make_float4(hs[4 * k], hs[4 * k + 1], hs[4 * k + 2], hs[4 * k + 3]);
        if (q == 0) {
            float v = fmaf(Dd, ut, acc);
            if (p.z) v *= silu_f32(zt);
            static_cast<IO*>(p.y)[rr] = IoTraits<IO>::from_f32(v);
        }
    }
}

}  // namespace ssm
