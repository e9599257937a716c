// scan_fwd_seq.cuh -- forward selective scan, "sequential" kernel family.
//
// Every (channel, n) chain is walked from t = 0 to t = L-1 by one lane, with the state
// in registers the whole time; only the final state is written to HBM ([Eng] §4.2: the
// state lives on chip and only h_N is written back; [S4M] 3.3: state accumulated on
// chip, written once at the end).
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [S4M]  "State Space Models 深度实战：从 S4 到 Mamba 的架构演进与 CUDA 优化"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
//
// Work split.  Channels are grouped in tiles of 8 consecutive channels of one batch
// row; the tiles are spread evenly over one persistent CTA per SM (each CTA takes a
// contiguous range, so every SM carries the same number of channel-steps to within
// one warp's share).  G lanes share a channel: lane `nl` of the group holds the
// NC = 16/G chains n = nl*NC .. nl*NC+NC-1, for CPL channels of the same batch row
// (CPL = 2 lets one load of a step's B/C rows serve two channels; the shared-memory
// data path is the scarce resource of this kernel).  Per step each lane computes
//   a = 2^(Delta * A[d,n] * log2 e),  h = a*h + (Delta*u)*B[n],  y_partial += C[n]*h
// (simplified discretisation Abar = exp(Delta A), Bbar = Delta B: [Card] 离散化变换; with ZOH the
// zero-order-hold weight of [Eng] §2.2, see zoh_phi2),
// and the G partial sums of y_t = sum_n C_t[n] h_t[n] are combined by a shuffle
// reduce-scatter over each 16-byte group of GS steps, so that every lane finishes the
// epilogue (D skip, silu gate, rounding, store) of GS/G steps and nothing is evaluated
// twice.  The step sizes Delta = softplus(delta + bias) of group q+1 are computed
// (split over the G lanes) while group q is scanned, and exchanged by shuffles.
//
// Staging.  A producer warp streams stage k (TC steps: one 128-byte row per channel)
// of u, delta and z for all the CTA's tiles, plus the stage's B/C rows (transposed in
// the workspace to fp32 [t][32]; at most two batch rows per CTA) into shared memory
// with TMA, through a ring of S stages signalled by mbarriers.  The 8-row u/delta/z
// boxes use the 128-byte swizzle, so the per-lane 16-byte reads of one column hit
// distinct banks; B/C are read as broadcasts.  The kernel may be launched as a
// programmatic dependent of the B/C transpose before it: the producer waits for that
// grid only before its first B/C copy.  Rows whose byte length is not a multiple of 16
// cannot be staged by TMA: the GA kernels leave u / delta / z to the consumer warps, which
// copy their own rows' 16-byte-aligned windows and shift them into the same tile layout
// (gather_copy, gather_align); the producer then streams only the B/C rows.
//
// Checkpoints (CK kernels, for the backward: [Tech] 四.1, keep a little in the forward
// pass): after every group of steps that ends on a multiple of 8, each lane also stores
// its chains, i.e. the state at the start of the next 8-step segment.
#pragma once

#include "common.cuh"
#include "scan_math.cuh"

namespace ssm {

struct SeqParams {
    const float* A;        // (dim, 16)
    const float* D;        // (dim) or null
    const float* bias;     // (dim) or null
    const float* h0;       // (batch, dim, 16) initial state or null (zero)
    float* last_state;     // (batch, dim, 16) or null
    void* y;               // (batch, dim, L) IO
    WorkspaceHeader* hdr;  // status word
    int batch, dim;
    long long L;
    int tiles_per_batch;   // ceil(dim / 8), rounded up to the tiles one warp covers
    long long total_tiles; // batch * tiles_per_batch
    int max_tiles;         // tiles one CTA stages per round (sets the shared-memory layout)
    int softplus;
    int has_z;
    uint32_t wait_limit;
    // causal conv1d + SiLU prologue (CONV kernels): the staged "u" tiles hold x
    const void* x;             // (batch, dim, L) IO: the conv input
    const float* conv_w;       // (dim, conv_k) fp32, oldest tap first
    const float* conv_b;       // (dim) or null
    const float* conv_in;      // (batch, dim, conv_k - 1) fp32 inputs before t = 0, or null (zero)
    float* conv_out;           // (batch, dim, conv_k - 1) fp32: the last conv_k - 1 inputs, or null
    void* u_out;               // (batch, dim, L) IO: the conv output, or null
    int conv_k;                // 1 .. 4
    // y rows are 16-byte aligned (L * sizeof(IO) a multiple of 16): vector stores; else
    // element stores
    int y_vec;
    // u / delta / z themselves, for the GA kernels (rows whose byte length is not a multiple of
    // 16, which TMA cannot address: see gather_copy); their tensor maps are then unused
    const void* u_rows;
    const void* dl_rows;
    const void* z_rows;
    // checkpoints for the backward, or null: (batch, nseg, dim, 16) fp32, the state at the
    // start of every 8-step segment (h before step 8s), nseg = ceil(L / 8)
    float* ckpt;
    int nseg;
};

__host__ __device__ constexpr int round_up_i(int v, int m) { return (v + m - 1) / m * m; }

template <typename IO, int G, int CPL>
struct SeqCfg {
    static constexpr int kNC = 16 / G;                       // chains per lane and channel
    static constexpr int kCW = 32 / G;                       // channel groups per warp
    static constexpr int kCPW = kCW * CPL;                   // channels per warp
    static constexpr int kTPW = kCPW >= 8 ? kCPW / 8 : 1;    // tiles per warp (a warp never spans batches)
    static constexpr int kGS = 16 / IoTraits<IO>::kBytes;    // steps per 16-byte group
    static constexpr int kPER = kGS / G;                     // epilogue steps per lane per group
    static constexpr int kTC = 128 / IoTraits<IO>::kBytes;   // steps per stage
    static constexpr int kNG = kTC / kGS;                    // groups per stage (8)
    static constexpr int kTileBytes = 1024;                  // 8 rows x 128 bytes (one swizzle atom)
    static constexpr int kBC = kTC * 128;                    // fp32 [TC][32] B/C rows of one batch row
    static constexpr int kMaxBatchRows = 2;                  // batch rows one CTA round may span
    // consumer warps per CTA (sets the register budget through the launch bound)
    static constexpr int kMaxWarps = CPL == 2 ? 12 : G == 2 ? 12 : G == 4 ? (sizeof(IO) == 2 ? 18 : 16) : 22;
    static_assert((G == 2 || G == 4 || G == 8) && G <= kGS, "G is 2, 4 or 8 and splits a 16-byte group");
    static_assert(CPL == 1 || CPL == 2, "one or two channels per lane");
    static_assert(kCPW % 8 == 0 || 8 % kCPW == 0, "warps tile the 8-channel tiles");

    __host__ __device__ static constexpr int warps_for(int tiles) { return (tiles * 8 + kCPW - 1) / kCPW; }
    __host__ __device__ static constexpr int stage_bytes(int max_tiles) {
        return 3 * max_tiles * kTileBytes + kMaxBatchRows * kBC;
    }
    __host__ __device__ static constexpr int smem_bytes(int max_tiles, int stages) {
        return stages * stage_bytes(max_tiles) + 1024;  // +1024: alignment slack
    }
    // GA kernels: one 8-byte word per u / delta / z row of a round after the ring (gather_row_info)
    __host__ __device__ static constexpr int gather_info_bytes(int max_tiles) { return max_tiles * 8 * 3 * 8; }
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

// Store N fp32 values as N consecutive IO elements at a naturally aligned address.
template <typename IO, int N>
__device__ __forceinline__ void store_run(IO* dst, const float (&v)[N]) {
    if constexpr (sizeof(IO) == 2 && N == 8) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                    pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    } else if constexpr (sizeof(IO) == 4 && N == 4) {
        *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (sizeof(IO) == 2 && N == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else if constexpr (sizeof(IO) == 2 && N == 2) {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(v[0], v[1]);
    } else if constexpr (sizeof(IO) == 4 && N == 2) {
        *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) dst[i] = IoTraits<IO>::from_f32(v[i]);
    }
}

// Gathered rows (GA kernels: rows of u / delta / z whose byte length is not a multiple of 16,
// which TMA cannot address).  Every consumer warp stages its own channels' rows itself, so
// the copies are spread over all warps (a single warp issuing them for the whole CTA fell
// behind the consumers):
//  * Row q of a round (tensor q / (nt * 8): u, delta, z; channel q % (nt * 8) of the round) is
//    described by one word set up at the start of the round, the address of its step 0
//    (0: no such row).  Its bytes sh = address & 15 before step 0 are the row's offset from the
//    16-byte grid; the window of stage k is the 128 bytes from (address & ~15) + k * 128.
//  * gather_copy copies a stage's windows with cp.async into the rows' 128-byte slots of the
//    tile area, unswizzled, three stages ahead.  Chunks holding no byte of the row's steps
//    0 .. L - 1 are zero-filled, not read (so nothing outside the caller's arrays, rounded to
//    16 bytes, is read).  One more stage is copied past the last (the chunks holding the last
//    step's bytes beyond the last window).
//  * gather_align, once stage k and k + 1 have landed, shifts the warp's rows of stage k into
//    place: lane (sub, c) takes window chunks c and c + 1 (chunk 8 is chunk 0 of the next
//    stage's window, not yet shifted), extracts bytes sh .. sh + 15 and writes them where the
//    128-byte-swizzled TMA box would have put chunk c (row r of a tile: ((c ^ r) << 4)).
//    Steps at or past L come out zero, as TMA fills them.
template <typename IO>
__device__ __forceinline__ uint64_t gather_row_info(const SeqParams& p, int q, int rows, int j0, int b_first) {
    const int tq = q >= rows ? (q >= 2 * rows ? 2 : 1) : 0;
    const int rr = q - tq * rows;
    const int jt = j0 + (rr >> 3);  // the round's tiles span at most two batch rows
    const int second = jt >= p.tiles_per_batch ? 1 : 0;
    const int b = b_first + second;
    const int d = (jt - second * p.tiles_per_batch) * 8 + (rr & 7);
    if (d >= p.dim || b >= p.batch) return 0;
    const uint8_t* base = static_cast<const uint8_t*>(tq == 0 ? p.u_rows : tq == 1 ? p.dl_rows : p.z_rows);
    return reinterpret_cast<uint64_t>(base + (static_cast<long long>(b) * p.dim + d) * p.L *
                                                 static_cast<long long>(IoTraits<IO>::kBytes));
}

// Shared-memory accesses of the gathering code by 32-bit shared-window address.
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t lds_u64(uint32_t a) {
    uint64_t v;
    asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ void cp_async_16_to(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Consumer warp `warp`: copy its rows' windows of stage k (0 <= k <= the number of stages) into
// the slot at shared address st (info: shared address of the row words; row_bytes = L *
// sizeof(IO)).  Pass r0 handles rows r0 .. r0 + 3 of the warp (tensor r0 / CPW), lane (sub, c)
// chunk c of row r0 + sub.
template <int CPW, int NT>
__device__ __forceinline__ void gather_copy(uint32_t st, uint32_t info, const SeqParams& p, int rows, int k,
                                            long long row_bytes, int warp, int lane) {
    const int sub = lane >> 3, c = lane & 7;
    const uint32_t tile_area = static_cast<uint32_t>(p.max_tiles) * 1024u;
    const int first = warp * CPW + sub;  // the lane's channel of the round in pass 0
    const uint32_t dst0 = st + first * 128 + c * 16;
    const uint32_t inf0 = info + first * 8;
    const long long rem = row_bytes - static_cast<long long>(k) * 128;  // row bytes from the window's t = 128k/size
    const long long kc = static_cast<long long>(k) * 128 + c * 16;
    const bool whole = rem >= 144;  // every chunk of every window holds step bytes (warp-uniform)
    const uint8_t* any = static_cast<const uint8_t*>(p.u_rows);  // (zero-fill: not read)
    // (every row a warp of a GA kernel covers is one of the round's: one channel per lane, and
    // the warps cover whole 8-channel tiles)
#pragma unroll
    for (int r0 = 0; r0 < CPW * NT; r0 += 4) {
        const int tq = r0 / CPW, rc = r0 % CPW;  // (CPW is a multiple of 4: a pass stays in one tensor)
        if (dcheck(p.hdr, first + rc < rows, kSiteSeqTma, first + rc)) {
            const uint64_t at = lds_u64(inf0 + (tq * rows + rc) * 8);
            const int sh = static_cast<int>(at & 15u);
            const bool need = at != 0 && (whole || c * 16 - sh < rem);  // the chunk holds a step byte
            const uint8_t* src = need ? reinterpret_cast<const uint8_t*>((at & ~uint64_t(15)) + kc) : any;
            cp_async_16_to(dst0 + tq * tile_area + rc * 128, src, need ? 16u : 0u);
        }
    }
}

// Consumer warp `warp`: shift its rows of the landed stage at shared address st into place (nx_st:
// the slot of the next stage, also landed; nbytes: bytes of the stage's steps in a row).  Lane
// c reads the 24 bytes from window byte 16c + (sh & 8) as three 8-byte words (those from byte
// 128 on are the next stage's window), keeps the words from (sh & 4) on and funnel-shifts by
// sh & 3.
template <int CPW, int NT>
__device__ __forceinline__ void gather_align(uint32_t st, uint32_t nx_st, uint32_t info, const SeqParams& p, int rows,
                                             int nbytes, int warp, int lane) {
    const int sub = lane >> 3, c = lane & 7;
    const int keep = nbytes - c * 16;  // bytes of this lane's chunk inside the row's steps
    const uint32_t tile_area = static_cast<uint32_t>(p.max_tiles) * 1024u;
    const int first = warp * CPW + sub;
    const uint32_t row0 = st + first * 128;
    const uint32_t inf0 = info + first * 8;
    const bool is7 = c == 7;
    const uint32_t nxd = nx_st - st - 128u;  // window byte 128 + j of a row -> byte j of its next window
    const uint32_t add2 = is7 ? nxd : 0u;
    const bool last = nbytes < 128;  // (warp-uniform) the row's last window: zero the steps past L
#pragma unroll
    for (int r0 = 0; r0 < CPW * NT; r0 += 4) {
        const int tq = r0 / CPW, rc = r0 % CPW;
        const bool mine = dcheck(p.hdr, first + rc < rows, kSiteSeqTma, first + rc);
        const uint32_t rowp = row0 + tq * tile_area + rc * 128;
        uint32_t sh = 0;
        uint2 w0 = make_uint2(0u, 0u), w1 = w0, w2 = w0;
        if (mine) {
            sh = lds_u32(inf0 + (tq * rows + rc) * 8) & 15u;  // (the row word's low half)
            const uint32_t la = rowp + c * 16 + (sh & 8u);
            const uint32_t add1 = (is7 && (sh & 8u)) ? nxd : 0u;
            w0 = lds_v2(la);
            w1 = lds_v2(la + 8 + add1);
            w2 = lds_v2(la + 16 + add2);
        }
        __syncwarp();  // every lane has read its words before any lane rewrites the row
        const uint32_t x[6] = {w0.x, w0.y, w1.x, w1.y, w2.x, w2.y};
        uint32_t u5[5], o[4];
#pragma unroll
        for (int i = 0; i < 5; ++i) u5[i] = (sh & 4u) ? x[i + 1] : x[i];
#pragma unroll
        for (int m = 0; m < 4; ++m) o[m] = __funnelshift_r(u5[m], u5[m + 1], (sh & 3u) * 8u);
        if (last) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int kb = keep - 4 * m;
                o[m] = kb >= 4 ? o[m] : kb <= 0 ? 0u : o[m] & ((1u << (8 * kb)) - 1u);
            }
        }
        if (mine) sts_v4(rowp + ((c ^ ((first + rc) & 7)) << 4), o[0], o[1], o[2], o[3]);
    }
    __syncwarp();
}

// Consumer warp of the sequential kernel (HZ: the z gate is present).
//
// Lane (cg, nl) holds the NC chains n = nl*NC .. of the channels cg + c*CW (c < CPL) of
// this warp's block of CPW channels; the CPL channels share the batch row, hence every
// B/C value the lane loads.  The walk goes stage by stage, and the eight 16-byte groups
// of a stage are unrolled (compile-time shared-memory offsets) with ping-pong step-size
// buffers: the step sizes of group g+1 (for the last group: group 0 of the next stage,
// after waiting for it) are computed while group g is scanned.
template <typename IO, int G, int CPL, int S, bool HZ, bool ZOH, bool CONV, bool CK, bool GA>
__device__ __forceinline__ void seq_consumer(uint8_t* smem, uint64_t* full_bar, uint64_t* empty_bar,
                                             const int* abort_flag, const SeqParams& p, long long r_begin, int nt,
                                             int b_first, int stage_bytes, int nstages, int L32) {
    using Cfg = SeqCfg<IO, G, CPL>;
    constexpr int NC = Cfg::kNC, CW = Cfg::kCW, CPW = Cfg::kCPW, GS = Cfg::kGS, TC = Cfg::kTC, NG = Cfg::kNG;
    constexpr int PER = Cfg::kPER, ES = IoTraits<IO>::kBytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cg = lane / G;
    const int nl = lane % G;
    const int gbase = lane & ~(G - 1);   // first lane of this channel group
    int cbase[CPL], d[CPL];
    bool valid[CPL];
    int b = 0;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int cl = warp * CPW + cg + c * CW;   // channel within the round's tiles
        const bool in_round = cl < nt * 8;
        const int j = in_round ? cl / 8 : 0;
        const int row = cl % 8;
        const long long tile = r_begin + j;
        if (c == 0) b = static_cast<int>(tile / p.tiles_per_batch);
        d[c] = static_cast<int>(tile % p.tiles_per_batch) * 8 + row;
        valid[c] = in_round && d[c] < p.dim;
        // Byte offset of the lane's 16-byte chunk of group g inside a u/delta/z tile block:
        // cbase ^ (g << 4) (the 128-byte swizzle XORs the chunk index with the row).
        cbase[c] = j * Cfg::kTileBytes + row * 128 + (row << 4);
        if (!dcheck(p.hdr, j < p.max_tiles && tile < p.total_tiles, kSiteSeqTile, j)) {
            valid[c] = false;
            cbase[c] = row * 128 + (row << 4);
        }
    }
    if (!dcheck(p.hdr, b >= b_first && b - b_first < Cfg::kMaxBatchRows, kSiteSeqTile, b - b_first)) b = b_first;
    const int dl_off = p.max_tiles * Cfg::kTileBytes;
    const int z_off = 2 * p.max_tiles * Cfg::kTileBytes;
    const int bc_off = 3 * p.max_tiles * Cfg::kTileBytes + (b - b_first) * Cfg::kBC + nl * NC * 4;

    float2 A2[CPL][NC / 2], h[CPL][NC / 2];
    float2 invA[CPL][ZOH ? NC / 2 : 1];  // 1 / A (zero-order hold only)
    float Dd[CPL], bias[CPL];
    IO* yrow[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const float* h0 = (valid[c] && p.h0) ? p.h0 + (static_cast<long long>(b) * p.dim + d[c]) * 16 + nl * NC
                                             : nullptr;
#pragma unroll
        for (int jj = 0; jj < NC / 2; ++jj) {
            const float a0 = valid[c] ? p.A[d[c] * 16 + nl * NC + 2 * jj] : 0.f;
            const float a1 = valid[c] ? p.A[d[c] * 16 + nl * NC + 2 * jj + 1] : 0.f;
            A2[c][jj] = f2(a0 * kLog2e, a1 * kLog2e);
            if constexpr (ZOH) invA[c][jj] = f2(1.f / a0, 1.f / a1);
            h[c][jj] = h0 ? *reinterpret_cast<const float2*>(h0 + 2 * jj) : f2(0.f, 0.f);
        }
        Dd[c] = (valid[c] && p.D) ? p.D[d[c]] : 0.f;
        bias[c] = (valid[c] && p.bias) ? p.bias[d[c]] : 0.f;
        yrow[c] = static_cast<IO*>(p.y) + (static_cast<long long>(b) * p.dim + (valid[c] ? d[c] : 0)) * p.L;
    }
    const bool softplus = p.softplus != 0;
    const uint32_t wait_limit = p.wait_limit;

    // Checkpoints for the backward: after the group that ends at step t_end (a multiple of 8
    // below L) the lane's chains hold h before step t_end, the start of segment t_end / 8.
    // (A compile-time variant: the store between the groups would otherwise cost the kernels
    // that write no checkpoints their cross-group scheduling.)
    auto checkpoint = [&](int t_end) {
        if (CK && (t_end & 7) == 0 && t_end < L32) {
#pragma unroll
            for (int c = 0; c < CPL; ++c)
                if (valid[c] && dcheck(p.hdr, (t_end >> 3) < p.nseg, kSiteSeqState, t_end)) {
                    float* dst = p.ckpt +
                                 ((static_cast<long long>(b) * p.nseg + (t_end >> 3)) * p.dim + d[c]) * 16 + nl * NC;
                    if constexpr (NC % 4 == 0) {  // 16-byte stores (nl * NC floats is a 16-byte offset)
#pragma unroll
                        for (int jj = 0; jj < NC / 2; jj += 2)
                            *reinterpret_cast<float4*>(dst + 2 * jj) =
                                make_float4(h[c][jj].x, h[c][jj].y, h[c][jj + 1].x, h[c][jj + 1].y);
                    } else {
#pragma unroll
                        for (int jj = 0; jj < NC / 2; ++jj) *reinterpret_cast<float2*>(dst + 2 * jj) = h[c][jj];
                    }
                }
        }
    };
    checkpoint(0);  // segment 0 starts from the initial state

    // Causal conv1d + SiLU of the staged x tile, in place ([Hist] Mamba Block 数据流: x -> 1D
    // conv -> SiLU -> S6).  Lane (cg, nl) converts steps nl*SPL .. of its channel cg; the three
    // inputs before its first step come from lane nl-1 by shuffle (lane 0: from the previous
    // stage, carried in registers).  u is rounded to the I/O type, as a separate conv kernel
    // writing u would round it; the scan below then reads u from the tile as usual.
    constexpr int SPL = TC / G;  // steps per lane
    static_assert(!CONV || (CPL == 1 && SPL % GS == 0 && SPL >= 3), "conv: one channel per lane");
    float cw[4] = {0.f, 0.f, 0.f, 0.f}, cb = 0.f, carry[3] = {0.f, 0.f, 0.f};
    if constexpr (CONV) {
        const int K = p.conv_k;
        if (valid[0]) {
            for (int k = 0; k < K; ++k) cw[4 - K + k] = p.conv_w[static_cast<long long>(d[0]) * K + k];
            cb = p.conv_b ? p.conv_b[d[0]] : 0.f;
            if (p.conv_in && nl == 0)
                for (int k = 0; k < K - 1; ++k)
                    carry[3 - (K - 1) + k] = p.conv_in[(static_cast<long long>(b) * p.dim + d[0]) * (K - 1) + k];
        }
    }
    auto conv_stage = [&](uint8_t* st, int tk) {
        if constexpr (CONV) {
            float xs[SPL];
#pragma unroll
            for (int m = 0; m < SPL / GS; ++m)
                Group16<IO>::unpack(*reinterpret_cast<const uint4*>(st + (cbase[0] ^ ((nl * (SPL / GS) + m) << 4))),
                                    *reinterpret_cast<float(*)[GS]>(xs + m * GS));
            // inputs before this lane's first step: the previous lane's last three (lane 0:
            // the carry); lane 0 keeps the last lane's last three for the next stage
            float prev[3];
            const int src = gbase | ((nl + G - 1) & (G - 1));
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const float got = __shfl_sync(0xffffffffu, xs[SPL - 3 + k], src, 32);
                prev[k] = nl == 0 ? carry[k] : got;
                if (nl == 0) carry[k] = got;
            }
            float uo[SPL];
#pragma unroll
            for (int i = 0; i < SPL; ++i) {
                float pre = cb;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int j = i - 3 + k;
                    pre = fmaf(cw[k], j >= 0 ? xs[j] : prev[3 + j], pre);
                }
                uo[i] = IoTraits<IO>::to_f32(IoTraits<IO>::from_f32(silu_f32(pre)));
            }
#pragma unroll
            for (int m = 0; m < SPL / GS; ++m) {
                float v[GS];
#pragma unroll
                for (int e = 0; e < GS; ++e) v[e] = uo[m * GS + e];
                uint8_t* dst = st + (cbase[0] ^ ((nl * (SPL / GS) + m) << 4));
                store_run<IO, GS>(reinterpret_cast<IO*>(dst), v);
            }
            if (p.u_out && valid[0]) {
                IO* urow = static_cast<IO*>(p.u_out) + (static_cast<long long>(b) * p.dim + d[0]) * p.L;
                const int t0 = tk + nl * SPL;
                if (p.y_vec && t0 + SPL <= L32) {  // (rows of u_out 16-byte aligned like those of y)
#pragma unroll
                    for (int m = 0; m < SPL / GS; ++m) {
                        float v[GS];
#pragma unroll
                        for (int e = 0; e < GS; ++e) v[e] = uo[m * GS + e];
                        store_run<IO, GS>(urow + t0 + m * GS, v);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < SPL; ++i)
                        if (t0 + i < L32) urow[t0 + i] = IoTraits<IO>::from_f32(uo[i]);
                }
            }
            __syncwarp();
        }
    };

    // Bounded, warp-uniform wait for ring slot s (a timeout can never leave part of the
    // warp inside the full-mask shuffles).
    auto wait_full = [&](int s, uint32_t parity, int k) -> bool {
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[s], parity, wait_limit));
        if (!ok && lane == 0) report_status(p.hdr, kDevTimeout, 2, blockIdx.x, k, wait_limit);
        return ok && !__any_sync(0xffffffffu, *(volatile const int*)abort_flag != 0);
    };

    // Step sizes of group g (first step tg) of the stage at st: lane nl evaluates softplus
    // for its PER steps i = r*G + nl of each of its channels.
    auto prologue = [&](const uint8_t* st, int g, int tg, float (&mine)[CPL][PER]) {
#pragma unroll
        for (int c = 0; c < CPL; ++c)
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                const int i = r * G + nl;
                const float raw = IoTraits<IO>::to_f32(
                    *reinterpret_cast<const IO*>(st + dl_off + (cbase[c] ^ (g << 4)) + i * ES));
                mine[c][r] = (tg + i < L32) ? step_size(raw, bias[c], softplus) : 0.f;  // 0 past L
            }
    };

    // Scan, reduce-scatter and epilogue of group g (first step tg) of the stage at st.
    auto scan_group = [&](const uint8_t* st, int g, int tg, const float (&mine)[CPL][PER]) {
        float uf[CPL][GS];
        int chunk[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            chunk[c] = cbase[c] ^ (g << 4);
            Group16<IO>::unpack(*reinterpret_cast<const uint4*>(st + chunk[c]), uf[c]);
        }
        const float* bc = reinterpret_cast<const float*>(st + bc_off) + g * GS * 32;
        float yp[CPL][GS];
#pragma unroll
        for (int i = 0; i < GS; ++i) {
            const float* bcr = bc + i * 32;
            float2 Bv[NC / 2], Cv[NC / 2];
#pragma unroll
            for (int jj = 0; jj < NC / 2; ++jj) {
                if constexpr (NC >= 4) {
                    const float4 Bq = *reinterpret_cast<const float4*>(bcr + (jj & ~1) * 2);
                    const float4 Cq = *reinterpret_cast<const float4*>(bcr + 16 + (jj & ~1) * 2);
                    Bv[jj] = (jj & 1) ? f2(Bq.z, Bq.w) : f2(Bq.x, Bq.y);
                    Cv[jj] = (jj & 1) ? f2(Cq.z, Cq.w) : f2(Cq.x, Cq.y);
                } else {
                    Bv[jj] = *reinterpret_cast<const float2*>(bcr + 2 * jj);
                    Cv[jj] = *reinterpret_cast<const float2*>(bcr + 16 + 2 * jj);
                }
            }
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const float dti = __shfl_sync(0xffffffffu, mine[c][i / G], gbase | (i % G), 32);
                const float wi = dti * uf[c][i];
                const float2 dd = f2(dti, dti);
                const float2 ww = f2(wi, wi);
                float2 acc = f2(0.f, 0.f);
#pragma unroll
                for (int jj = 0; jj < NC / 2; ++jj) {
                    const float2 arg = __fmul2_rn(dd, A2[c][jj]);
                    const float2 a = f2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                    float2 beta;
                    if constexpr (ZOH)  // phi (u B), phi the hold weight per unit input
                        beta = __fmul2_rn(zoh_phi2(arg, a, dd, invA[c][jj]),
                                          __fmul2_rn(f2(uf[c][i], uf[c][i]), Bv[jj]));
                    else
                        beta = __fmul2_rn(ww, Bv[jj]);
                    h[c][jj] = __ffma2_rn(a, h[c][jj], beta);
                    acc = __ffma2_rn(Cv[jj], h[c][jj], acc);
                }
                yp[c][i] = acc.x + acc.y;
            }
        }

        // Reduce-scatter the G partial sums of each channel: afterwards lane nl holds
        // the full y_t of steps nl*PER .. nl*PER+PER-1 in yp[c][0..PER-1].
#pragma unroll
        for (int m = G / 2, half = GS / 2; m >= 1; m >>= 1, half >>= 1) {
            const bool upper = (nl & m) != 0;
#pragma unroll
            for (int c = 0; c < CPL; ++c)
#pragma unroll
                for (int i = 0; i < half; ++i) {
                    const float send = upper ? yp[c][i] : yp[c][i + half];
                    const float keep = upper ? yp[c][i + half] : yp[c][i];
                    yp[c][i] = keep + __shfl_xor_sync(0xffffffffu, send, m, 32);
                }
        }

        // Epilogue: D skip and silu gate ([Eng] §2.2; [Hist] Mamba Block), round, store.
        const int t0 = tg + nl * PER;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int off = chunk[c] + nl * PER * ES;
            float ue[PER], ze[PER], yo[PER];
            load_run<IO, PER>(st + off, ue);
            if constexpr (HZ) load_run<IO, PER>(st + z_off + off, ze);
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                float v = fmaf(Dd[c], ue[r], yp[c][r]);
                if constexpr (HZ) v *= gate_silu<IO>(ze[r]);
                yo[r] = v;
            }
            // (steps at or past L store nothing)
            if (valid[c] &&
                dcheck(p.hdr, t0 >= L32 || (static_cast<long long>(b) * p.dim + d[c]) * p.L + t0 <
                                               static_cast<long long>(p.batch) * p.dim * p.L,
                       kSiteSeqY, t0)) {
                if (p.y_vec && t0 + PER <= L32) {
                    store_run<IO, PER>(yrow[c] + t0, yo);
                } else if (GA && t0 + PER <= L32) {  // (rows not 16-byte aligned: element stores)
#pragma unroll
                    for (int r = 0; r < PER; ++r) yrow[c][t0 + r] = IoTraits<IO>::from_f32(yo[r]);
                } else {
#pragma unroll
                    for (int r = 0; r < PER; ++r)
                        if (t0 + r < L32) yrow[c][t0 + r] = IoTraits<IO>::from_f32(yo[r]);
                }
            }
        }
    };

    float spA[CPL][PER], spB[CPL][PER];
    const uint8_t* st = smem;
    int slot = 0;
    uint32_t parity = 0;
    // GA: this warp's rows, copied three stages ahead (the copies of stage k land in a cp.async
    // group of their own), shifted into place when a stage and the next have landed
    const uint32_t smem_s = smem_u32(smem);
    const uint32_t ginfo = smem_s + S * stage_bytes;
    auto issue_stage = [&](int kk) {
        if constexpr (GA) {
            if (kk <= nstages) {  // (stage nstages: the chunks past the last window)
                gather_copy<CPW, HZ ? 3 : 2>(smem_s + (kk % S) * stage_bytes, ginfo, p, nt * 8, kk,
                                             p.L * static_cast<long long>(ES), warp, lane);
                cp_async_commit();
            }
        }
    };
    auto align_stage = [&](int kk) {
        if constexpr (GA) {
            cp_async_wait<0>();
            __syncwarp();
            gather_align<CPW, HZ ? 3 : 2>(smem_s + (kk % S) * stage_bytes, smem_s + ((kk + 1) % S) * stage_bytes,
                                          ginfo, p, nt * 8, min(TC, L32 - kk * TC) * ES, warp, lane);
        }
    };
    issue_stage(0);
    issue_stage(1);
    issue_stage(2);
    bool alive = wait_full(0, 0, 0);
    if (alive) {
        align_stage(0);
        conv_stage(smem, 0);
        prologue(st, 0, 0, spA);
    }
#pragma unroll 1
    for (int k = 0, tk = 0; alive && k < nstages; ++k, tk += TC) {
#pragma unroll
        for (int g = 0; g < NG; g += 2) {
            prologue(st, g + 1, tk + (g + 1) * GS, spB);
            scan_group(st, g, tk + g * GS, spA);
            if (g + 2 < NG) {
                prologue(st, g + 2, tk + (g + 2) * GS, spA);
            } else if (k + 1 < nstages) {
                const int sn = slot + 1 == S ? 0 : slot + 1;
                alive = wait_full(sn, slot + 1 == S ? parity ^ 1u : parity, k + 1);
                if (alive) {
                    align_stage(k + 1);
                    conv_stage(smem + sn * stage_bytes, tk + TC);
                    prologue(smem + sn * stage_bytes, 0, tk + TC, spA);
                }
            }
            checkpoint(tk + (g + 1) * GS);
            scan_group(st, g + 1, tk + (g + 1) * GS, spB);
            checkpoint(tk + (g + 2) * GS);
        }
        // The stage is consumed: release it to the producer.
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
        issue_stage(k + 3);  // (into the slot of stage k + 3 - S, which this warp is done with)
        if (++slot == S) {
            slot = 0;
            parity ^= 1u;
        }
        st = smem + slot * stage_bytes;
    }

    if constexpr (GA) cp_async_wait<0>();  // (after a timeout: no copy may land in the next round)
    if constexpr (CONV) {
        // the last conv_k - 1 inputs (from x, or from conv_in when the sequence is shorter)
        const int K = p.conv_k;
        if (p.conv_out && valid[0] && nl == 0) {
            const long long row = static_cast<long long>(b) * p.dim + d[0];
            for (int k = 0; k < K - 1; ++k) {
                const long long s2 = static_cast<long long>(L32) - (K - 1) + k;
                float v = 0.f;
                if (s2 >= 0) v = IoTraits<IO>::to_f32(static_cast<const IO*>(p.x)[row * p.L + s2]);
                else if (p.conv_in) v = p.conv_in[row * (K - 1) + (K - 1 + s2)];
                p.conv_out[row * (K - 1) + k] = v;
            }
        }
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c)
        if (valid[c] && p.last_state &&
            dcheck(p.hdr, (static_cast<long long>(b) * p.dim + d[c]) * 16 + nl * NC + NC <= static_cast<long long>(p.batch) * p.dim * 16,
                   kSiteSeqState, d[c])) {
            float* dst = p.last_state + (static_cast<long long>(b) * p.dim + d[c]) * 16 + nl * NC;
#pragma unroll
            for (int jj = 0; jj < NC / 2; ++jj) *reinterpret_cast<float2*>(dst + 2 * jj) = h[c][jj];
        }
}

template <typename IO, int G, int CPL, int S, bool ZOH = false, bool CONV = false, bool CK = false, bool GA = false>
__global__ void __launch_bounds__((SeqCfg<IO, G, CPL>::kMaxWarps + 1) * 32, 1)
scan_fwd_seq_kernel(const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_dl,
                    const __grid_constant__ CUtensorMap map_z, const __grid_constant__ CUtensorMap map_bc,
                    const SeqParams p) {
    using Cfg = SeqCfg<IO, G, CPL>;
    constexpr int TC = Cfg::kTC, TPW = Cfg::kTPW;
    static_assert(S >= 2 && S <= 8, "ring depth");
    static_assert(!GA || (S >= 3 && CPL == 1), "gathered rows: copies run three stages ahead of the scan");

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[S], empty_bar[S];
    __shared__ int abort_flag;
    // 1024-byte aligned base for the swizzled tiles (pointer arithmetic keeps the shared
    // address space visible to the compiler).
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int stage_bytes = Cfg::stage_bytes(p.max_tiles);
    uint64_t* ginfo = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);  // (GA)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int producer_warp = blockDim.x / 32 - 1;
    const int L32 = static_cast<int>(p.L);  // the host launches this kernel for L < 2^31 - 1024 only
    const int nstages = (L32 + TC - 1) / TC;

    // This CTA's tiles: [t_begin, t_end) of the flat (batch row, 8-channel tile) order,
    // cut at multiples of the tiles one warp covers (so no warp straddles two batch rows:
    // tiles_per_batch is a multiple of TPW, padded with empty tiles past `dim`).
    const long long units = p.total_tiles / TPW;
    const long long t_begin = units * blockIdx.x / gridDim.x * TPW;
    const long long t_end = units * (blockIdx.x + 1) / gridDim.x * TPW;

    // Rounds of at most max_tiles tiles (one round for the shapes the host launches;
    // more when the tiles do not fit in shared memory at once).
    for (long long r_begin = t_begin; r_begin < t_end; r_begin += p.max_tiles) {
        const int nt = static_cast<int>(min(static_cast<long long>(p.max_tiles), t_end - r_begin));
        const int b_first = static_cast<int>(r_begin / p.tiles_per_batch);
        const int nb = static_cast<int>((r_begin + nt - 1) / p.tiles_per_batch) - b_first + 1;  // 1 or 2
        const int nwarps = Cfg::warps_for(nt);

        if (threadIdx.x == 0) {
            for (int s = 0; s < S; ++s) {
                mbar_init(&full_bar[s], 1);
                mbar_init(&empty_bar[s], nwarps);
            }
            abort_flag = 0;
            mbar_fence_init();
        }
        if constexpr (GA) {
            const int rows = nt * 8;
            const int j0 = static_cast<int>(r_begin - static_cast<long long>(b_first) * p.tiles_per_batch);
            for (int q = threadIdx.x; q < rows * (p.has_z ? 3 : 2); q += blockDim.x)
                ginfo[q] = gather_row_info<IO>(p, q, rows, j0, b_first);
        }
        __syncthreads();

        if (warp == producer_warp) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                if (r_begin == t_begin) {
                    if constexpr (!GA) {
                        tma_prefetch_map(&map_u);
                        tma_prefetch_map(&map_dl);
                        if (p.has_z) tma_prefetch_map(&map_z);
                    }
                    tma_prefetch_map(&map_bc);
                }
                // (GA: the consumer warps copy u / delta / z themselves)
                const uint32_t bytes = (GA ? 0u : nt * (p.has_z ? 3u : 2u) * Cfg::kTileBytes) + nb * Cfg::kBC;
                for (int k = 0; k < nstages; ++k) {
                    const int s = k % S;
                    if (k >= S && !mbar_wait_sleep(&empty_bar[s], ((k / S) - 1) & 1, p.wait_limit)) {
                        report_status(p.hdr, kDevTimeout, 1, blockIdx.x, k, p.wait_limit);
                        atomicExch(&abort_flag, 1);
                        break;
                    }
                    uint8_t* st = smem + s * stage_bytes;
                    const int t0 = k * TC;
                    // the TMA x coordinate must be 16-byte aligned; every copy lands inside the slot
                    if (!dcheck(p.hdr, (t0 % TC) == 0 && nt <= p.max_tiles && nb <= Cfg::kMaxBatchRows &&
                                           b_first + nb <= p.batch,
                                kSiteSeqTma, t0)) {
                        atomicExch(&abort_flag, 1);
                        break;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(&full_bar[s], bytes);
                    for (int j = 0; j < (GA ? 0 : nt); ++j) {
                        const long long tile = r_begin + j;
                        const int b = static_cast<int>(tile / p.tiles_per_batch);
                        const int dd = static_cast<int>(tile % p.tiles_per_batch) * 8;
                        tma_load_3d(st + j * Cfg::kTileBytes, &map_u, &full_bar[s], t0, dd, b);
                        tma_load_3d(st + (p.max_tiles + j) * Cfg::kTileBytes, &map_dl, &full_bar[s], t0, dd, b);
                        if (p.has_z)
                            tma_load_3d(st + (2 * p.max_tiles + j) * Cfg::kTileBytes, &map_z, &full_bar[s], t0, dd, b);
                    }
                    // The B/C rows come from the kernel launched just before this one (which may
                    // still be running when this one starts): wait for it before the first copy.
                    if (k == 0 && r_begin == t_begin) pdl_wait_primary();
                    for (int bb = 0; bb < nb; ++bb)
                        tma_load_3d(st + 3 * p.max_tiles * Cfg::kTileBytes + bb * Cfg::kBC, &map_bc, &full_bar[s], 0,
                                    t0, b_first + bb);
                }
            }
        } else if (warp < nwarps) {
            if (p.has_z)
                seq_consumer<IO, G, CPL, S, true, ZOH, CONV, CK, GA>(smem, full_bar, empty_bar, &abort_flag, p, r_begin,
                                                                 nt, b_first, stage_bytes, nstages, L32);
            else
                seq_consumer<IO, G, CPL, S, false, ZOH, CONV, CK, GA>(smem, full_bar, empty_bar, &abort_flag, p, r_begin,
                                                                  nt, b_first, stage_bytes, nstages, L32);
        }
        // Every warp leaves the round before the barriers are re-initialised for the next.
        __syncthreads();
        if (threadIdx.x == 0)
            for (int s = 0; s < S; ++s) {
                mbar_inval(&full_bar[s]);
                mbar_inval(&empty_bar[s]);
            }
        __syncthreads();
    }
}

}  // namespace ssm
