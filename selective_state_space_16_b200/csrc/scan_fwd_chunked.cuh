// scan_fwd_chunked.cuh -- forward selective scan with the sequence split across CTAs.
//
// The sequence of every channel is cut into chunks of TC steps; a work unit is one
// 8-channel tile x one chunk, and persistent CTAs take units in chunk-major order
// from a ticket counter.  Inside a unit the chunk is split again into 8 slices of GS
// steps, one 16-byte group per lane (4 time-warps x 2 slices per warp).  The pieces
// are joined with the associative pair operator on (prod Abar, h):
//     (P1, H1) (x) (P2, H2) = (P2 * P1, P2 * H1 + H2)
// ([Eng] §4.1 parallel scan; [Card] 线性扫描算法: the recurrence regroups associatively),
// in three levels:
//   1. a register-resident sequential scan of each lane's slice from h = 0, keeping
//      the slice's Abar (and Delta u) of every step in registers (pass 1);
//   2. a warp-shuffle join of the two slices of a warp, then a shared-memory join of
//      the four time-warps of the unit;
//   3. a decoupled look-back across units of the same tile: each unit publishes its
//      aggregate (the chunk's summed step size, from which prod Abar = exp(A sum Delta),
//      and h with a zero carry-in) as soon as pass 1 is done, then walks back over its
//      predecessors' aggregates until it meets an inclusive state, and publishes its own
//      inclusive state ([S4M] 3.3: long sequences are chunked across SMs and scanned
//      in parallel inside each chunk; [Eng] §7.2 state continuation across chunks).
// With the carry-in known, every lane re-runs its slice from the stored values (pass 2)
// and produces the outputs: no exponential is evaluated twice.
//
// Pages (sections as printed):
//   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
//   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
//   [S4M]  "State Space Models 深度实战：从 S4 到 Mamba 的架构演进与 CUDA 优化"
//   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
//
// Flags and payloads live in the caller's workspace.  A flag holds (tag << 2) | state
// with state 1 = aggregate, 2 = inclusive and tag = epoch + 1 of this launch, so flags
// left by earlier launches never match; the last CTA of a launch advances the epoch and
// resets the ticket counter, which leaves the workspace ready for the next call.
// Every wait is bounded: a predecessor that never publishes makes the waiter record
// SSM_ERR_TIMEOUT in the workspace status word and carry on with a zero carry-in.
#pragma once

#include "common.cuh"
#include "scan_math.cuh"
#include "scan_fwd_seq.cuh"

namespace ssm {

struct ChunkParams {
    const float* A;        // (dim, 16)
    const float* D;        // (dim) or null
    const float* bias;     // (dim) or null
    float* last_state;     // (batch, dim, 16) or null
    void* y;               // (batch, dim, L) IO
    WorkspaceHeader* hdr;
    uint32_t* flags;       // [key] with key = (tile * 2 + column) * nchunks + chunk
    float* pay_agg;        // [key][4 channels][16]: h of the chunk with a zero carry-in
    float* pay_sdt;        // [key][4 channels]: sum of the chunk's step sizes
    float* pay_incl;       // [key][4 channels][16]: h at the end of the chunk
    const float* h0;       // (batch, dim, 16) state before step 0, or null (zero)
    int batch, dim;
    int L;
    int tiles_per_batch;   // ceil(dim / 8)
    int nchunks;           // ceil(L / TC)
    long long total_tiles; // batch * tiles_per_batch
    long long total_units; // total_tiles * nchunks
    int softplus;
    int has_z;
    uint32_t wait_limit;   // mbarrier tries
    uint32_t spin_limit;   // look-back polls
    int debug_skip_chunk;  // tests: units of this chunk never publish (-1: off)
};

template <typename IO>
struct ChunkCfg {
    static constexpr int kG = 4;                             // lanes per channel
    static constexpr int kNC = 4;                            // chains per lane
    static constexpr int kGS = 16 / IoTraits<IO>::kBytes;    // steps per slice (one 16-byte group)
    static constexpr int kPER = kGS / kG;                    // epilogue steps per lane
    static constexpr int kTC = 8 * kGS;                      // steps per chunk (one 128-byte row)
    static constexpr int kNWT = 4;                           // time-warps per unit (2 slices each)
    static constexpr int kNWC = 2;                           // channel columns (4 channels each)
    static constexpr int kWarps = kNWT * kNWC;               // consumer warps
    static constexpr int kThreads = (kWarps + 1) * 32;       // + producer warp
    static constexpr int kTile = 1024;                       // 8 rows x 128 bytes
    static constexpr int kBC = kTC * 128;                    // fp32 [TC][32] B/C rows
    static constexpr int kBuf = 3 * kTile + kBC;             // u, delta, z, B/C of one unit
    static constexpr int kBufs = 2;   // a deeper ring lengthens the look-back chains (measured)
    static constexpr int kAgg = kNWT * 8 * 16 * 8;           // (P, H) per time-warp, channel, chain
    static constexpr int kSpec = kBufs * 8 * 16 * 4;         // speculatively fetched carry-in per buffer
    static constexpr int kSmem = kBufs * kBuf + kAgg + 8 * 16 * 4 + kNWT * 8 * 4 + kSpec + 1024;
};

template <typename IO>
__global__ void __launch_bounds__(ChunkCfg<IO>::kThreads, 2)
scan_fwd_chunked_kernel(const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_dl,
                        const __grid_constant__ CUtensorMap map_z, const __grid_constant__ CUtensorMap map_bc,
                        const ChunkParams p) {
    using Cfg = ChunkCfg<IO>;
    constexpr int G = Cfg::kG, GS = Cfg::kGS, PER = Cfg::kPER, TC = Cfg::kTC, NWT = Cfg::kNWT;
    constexpr int ES = IoTraits<IO>::kBytes;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[Cfg::kBufs], empty_bar[Cfg::kBufs];
    __shared__ long long ticket_sm[Cfg::kBufs];
    __shared__ int spec_ok[Cfg::kBufs][Cfg::kNWC];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float2* agg = reinterpret_cast<float2*>(smem + Cfg::kBufs * Cfg::kBuf);          // [NWT][8][16]
    float* carry = reinterpret_cast<float*>(smem + Cfg::kBufs * Cfg::kBuf + Cfg::kAgg);  // [8][16]
    float* sdt_sm = carry + 8 * 16;                                                    // [NWT][8]
    float* spec = sdt_sm + NWT * 8;                                                    // [kBufs][8][16]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tag = (ld_acquire_gpu(&p.hdr->epoch) + 1u) & 0x3fffffffu;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::kBufs; ++s) {
            mbar_init(&full_bar[s], 2);  // TMA bytes + the producer's speculative carry-in
            mbar_init(&empty_bar[s], Cfg::kWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == Cfg::kWarps) {
        // -------------------------------------------------------------------- producer
        // Per unit: the next ticket (fetched one unit ahead), the TMA loads, and a
        // speculative read of the predecessor unit's inclusive state (in chunk-major order
        // it has usually been published long before), so that the consumers' look-back
        // rarely has to wait for global memory.
        if (lane == 0) {
            tma_prefetch_map(&map_u);
            tma_prefetch_map(&map_dl);
            tma_prefetch_map(&map_bc);
            if (p.has_z) tma_prefetch_map(&map_z);
        }
        const uint32_t bytes = (p.has_z ? 3u : 2u) * Cfg::kTile + Cfg::kBC;
        long long tk_next = 0;
        if (lane == 0) tk_next = static_cast<long long>(atomicAdd(&p.hdr->ticket, 1u));
        for (int it = 0;; ++it) {
            const int bi = it % Cfg::kBufs;
            bool ok = true;
            if (it >= Cfg::kBufs)
                ok = mbar_wait_bounded(&empty_bar[bi], ((it / Cfg::kBufs) - 1) & 1, p.wait_limit);
            ok = __all_sync(0xffffffffu, ok);
            const long long tk = __shfl_sync(0xffffffffu, tk_next, 0);
            if (!ok || tk >= p.total_units) {  // no more work (or a lost barrier): consumers leave
                if (lane == 0) {
                    if (!ok) report_status(p.hdr, kDevTimeout, 1, blockIdx.x, it, p.wait_limit);
                    ticket_sm[bi] = -1;
                    mbar_arrive(&full_bar[bi]);
                    mbar_arrive(&full_bar[bi]);
                }
                break;
            }
            const int k = static_cast<int>(tk / p.total_tiles);
            const long long tile = tk % p.total_tiles;
            if (lane == 0) {
                ticket_sm[bi] = tk;
                const int b = static_cast<int>(tile / p.tiles_per_batch);
                const int dd = static_cast<int>(tile % p.tiles_per_batch) * 8;
                uint8_t* st = smem + bi * Cfg::kBuf;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&full_bar[bi], bytes);
                tma_load_3d(st, &map_u, &full_bar[bi], k * TC, dd, b);
                tma_load_3d(st + Cfg::kTile, &map_dl, &full_bar[bi], k * TC, dd, b);
                if (p.has_z) tma_load_3d(st + 2 * Cfg::kTile, &map_z, &full_bar[bi], k * TC, dd, b);
                tma_load_3d(st + 3 * Cfg::kTile, &map_bc, &full_bar[bi], 0, k * TC, b);
                tk_next = static_cast<long long>(atomicAdd(&p.hdr->ticket, 1u));
            }
            // lane = wc * 16 + cg * 4 + nl: column wc, channel cg, chains nl*4 .. nl*4+3
            int okc = 0;
            const long long nkeys = p.total_tiles * 2 * p.nchunks;
            if (k > 0 && dcheck(p.hdr, ((tile * 2 + (lane >> 4)) * p.nchunks + k - 1) < nkeys, kSiteChunkKey, tk)) {
                const int wc = lane >> 4;
                const long long key = (tile * 2 + wc) * p.nchunks + (k - 1);
                const uint32_t f = ld_acquire_gpu(p.flags + key);
                okc = ((f >> 2) == tag && (f & 3u) == 2u) ? 1 : 0;
                if (okc) {
                    const float4 v = ld_relaxed_gpu_f4(reinterpret_cast<const float4*>(p.pay_incl + key * 64 + (lane & 15) * 4));
                    *reinterpret_cast<float4*>(spec + bi * 128 + (wc * 4 + ((lane >> 2) & 3)) * 16 + (lane & 3) * 4) = v;
                }
            }
            // a column's carry is usable only if all 16 of its lanes found it published
            const unsigned ball = __ballot_sync(0xffffffffu, okc != 0);
            okc = ((ball >> ((lane >> 4) * 16)) & 0xffffu) == 0xffffu ? 1 : 0;
            if ((lane & 15) == 0) spec_ok[bi][lane >> 4] = okc;
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_bar[bi]);
        }
    } else {
        // -------------------------------------------------------------------- consumers
        // lane = s*16 + cg*4 + nl: slice s of the warp, channel cg of the warp's column,
        // chains nl*4 .. nl*4+3 of that channel.
        const int wt = warp / Cfg::kNWC;            // time-warp
        const int wc = warp % Cfg::kNWC;            // channel column
        const int s = lane >> 4, cg = (lane >> 2) & 3, nl = lane & 3;
        const int row = wc * 4 + cg;                // channel row within the tile
        const int g = wt * 2 + s;                   // this lane's 16-byte group (slice) of the chunk
        const int off = row * 128 + ((g ^ row) << 4);
        const int gbase = lane & ~3;
        const bool softplus = p.softplus != 0, has_z = p.has_z != 0;
        const bool lookback_warp = (wt == NWT - 1);

        for (int it = 0;; ++it) {
            const int bi = it % Cfg::kBufs;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[bi], (it / Cfg::kBufs) & 1,
                                                                      p.wait_limit));
            if (!ok) {
                if (lane == 0) report_status(p.hdr, kDevTimeout, 2, blockIdx.x, it, p.wait_limit);
                break;
            }
            const long long tk = ticket_sm[bi];
            if (tk < 0) break;
            const int k = static_cast<int>(tk / p.total_tiles);
            const long long tile = tk % p.total_tiles;
            const int b = static_cast<int>(tile / p.tiles_per_batch);
            const int d = static_cast<int>(tile % p.tiles_per_batch) * 8 + row;
            const bool valid = d < p.dim;
            const uint8_t* st = smem + bi * Cfg::kBuf;
            const float* bcr0 = reinterpret_cast<const float*>(st + 3 * Cfg::kTile) + g * GS * 32 + nl * 4;

            float2 A2[2];
            A2[0] = valid ? f2(p.A[d * 16 + nl * 4] * kLog2e, p.A[d * 16 + nl * 4 + 1] * kLog2e) : f2(0.f, 0.f);
            A2[1] = valid ? f2(p.A[d * 16 + nl * 4 + 2] * kLog2e, p.A[d * 16 + nl * 4 + 3] * kLog2e) : f2(0.f, 0.f);
            const float bias = (valid && p.bias) ? p.bias[d] : 0.f;

            // Step sizes of the slice: lane nl evaluates steps i = r*4 + nl, then the four
            // lanes of the channel exchange them.
            float mine[PER];
#pragma unroll
            for (int r = 0; r < PER; ++r) {
                const int i = r * G + nl;
                const float raw = IoTraits<IO>::to_f32(*reinterpret_cast<const IO*>(st + Cfg::kTile + off + i * ES));
                mine[r] = (k * TC + g * GS + i < p.L) ? step_size(raw, bias, softplus) : 0.f;
            }
            float uf[GS], dt[GS];
            Group16<IO>::unpack(*reinterpret_cast<const uint4*>(st + off), uf);
            float sdt = 0.f;
#pragma unroll
            for (int i = 0; i < GS; ++i) {
                dt[i] = __shfl_sync(0xffffffffu, mine[i / G], gbase | (i % G), 32);
                sdt += dt[i];
            }

            // Pass 1: the slice from a zero state, keeping Abar (the exponentials) and
            // Delta*u of every step in registers; Bbar u = (Delta u) B is recomputed in pass 2.
            float2 av[GS][2], hl[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
            float wv[GS];
#pragma unroll
            for (int i = 0; i < GS; ++i) {
                const float4 Bq = *reinterpret_cast<const float4*>(bcr0 + i * 32);
                const float2 dd = f2(dt[i], dt[i]);
                wv[i] = dt[i] * uf[i];
                const float2 ww = f2(wv[i], wv[i]);
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const float2 arg = __fmul2_rn(dd, A2[jj]);
                    av[i][jj] = f2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                    hl[jj] = __ffma2_rn(av[i][jj], hl[jj], __fmul2_rn(ww, jj ? f2(Bq.z, Bq.w) : f2(Bq.x, Bq.y)));
                }
            }
            // prod Abar over the slice = 2^(A log2e * sum Delta)
            float2 Pl[2];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const float2 arg = __fmul2_rn(f2(sdt, sdt), A2[jj]);
                Pl[jj] = f2(ex2_mufu(arg.x), ex2_mufu(arg.y));
            }

            // Warp-shuffle join of the two slices: slice 1 combines slice 0's pair with its own.
            float2 Pex[2], Hex[2], Pw[2], Hw[2];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const float2 Po = f2(__shfl_xor_sync(0xffffffffu, Pl[jj].x, 16), __shfl_xor_sync(0xffffffffu, Pl[jj].y, 16));
                const float2 Ho = f2(__shfl_xor_sync(0xffffffffu, hl[jj].x, 16), __shfl_xor_sync(0xffffffffu, hl[jj].y, 16));
                Pex[jj] = s ? Po : f2(1.f, 1.f);   // exclusive prefix of this slice inside the warp
                Hex[jj] = s ? Ho : f2(0.f, 0.f);
                Pw[jj] = __fmul2_rn(Pl[jj], Pex[jj]);              // warp aggregate (valid on slice 1)
                Hw[jj] = __ffma2_rn(Pl[jj], Hex[jj], hl[jj]);
            }
            const float sdt_w = sdt + __shfl_xor_sync(0xffffffffu, sdt, 16);
            if (s == 1) {
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    agg[(wt * 8 + row) * 16 + nl * 4 + 2 * jj] = f2(Pw[jj].x, Hw[jj].x);
                    agg[(wt * 8 + row) * 16 + nl * 4 + 2 * jj + 1] = f2(Pw[jj].y, Hw[jj].y);
                }
                if (nl == 0) sdt_sm[wt * 8 + row] = sdt_w;
            }
            named_barrier_sync(1, Cfg::kWarps * 32);

            // Decoupled look-back (the last time-warp of each column; slice-1 lanes carry
            // the payload for their 4 chains, lane 0 polls the flags).
            if (lookback_warp &&
                dcheck(p.hdr, (tile * 2 + wc) * p.nchunks + k < p.total_tiles * 2 * p.nchunks && k < p.nchunks,
                       kSiteChunkKey, tk)) {
                const long long key = (tile * 2 + wc) * p.nchunks + k;
                // unit aggregate: fold the time-warps' pairs in order
                float hu[4], pu[4];
                float sdt_u = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    pu[c] = 1.f;
                    hu[c] = 0.f;
                }
#pragma unroll
                for (int w = 0; w < NWT; ++w) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 ph = agg[(w * 8 + row) * 16 + nl * 4 + c];
                        hu[c] = fmaf(ph.x, hu[c], ph.y);
                        pu[c] *= ph.x;
                    }
                    sdt_u += sdt_sm[w * 8 + row];
                }
                const bool publish = (k != p.debug_skip_chunk);
                // The state before step 0 (the carry-in of chunk 0) of this lane's 4 chains.
                auto initial = [&]() -> float4 {
                    return (p.h0 && valid) ? *reinterpret_cast<const float4*>(
                                                 p.h0 + (static_cast<long long>(b) * p.dim + d) * 16 + nl * 4)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                };
                float hin[4] = {0.f, 0.f, 0.f, 0.f};
                if (k == 0) {
                    const float4 v = initial();
                    hin[0] = v.x; hin[1] = v.y; hin[2] = v.z; hin[3] = v.w;
                }
                const bool have_spec = k > 0 && spec_ok[bi][wc] != 0;
                if (have_spec) {
                    const float4 v = *reinterpret_cast<const float4*>(spec + bi * 128 + row * 16 + nl * 4);
                    hin[0] = v.x; hin[1] = v.y; hin[2] = v.z; hin[3] = v.w;
                } else if (k > 0) {
                    if (publish) {
                        if (s == 1) {
                            *reinterpret_cast<float4*>(p.pay_agg + key * 64 + cg * 16 + nl * 4) =
                                make_float4(hu[0], hu[1], hu[2], hu[3]);
                            if (nl == 0) p.pay_sdt[key * 4 + cg] = sdt_u;
                        }
                        fence_acq_rel_gpu();
                        __syncwarp();
                        if (lane == 0) st_release_gpu(p.flags + key, (tag << 2) | 1u);
                    }
                    // walk back: (px, hx) is the combined pair of the units passed so far
                    float px[4] = {1.f, 1.f, 1.f, 1.f}, hx[4] = {0.f, 0.f, 0.f, 0.f};
                    for (long long j = key - 1, kk = k - 1; kk >= 0; --j, --kk) {
                        uint32_t f = 0, polls = 0;
                        if (lane == 0) {
                            for (;;) {
                                f = ld_acquire_gpu(p.flags + j);
                                if ((f >> 2) == tag && (f & 3u) != 0u) break;
                                if (++polls >= p.spin_limit) {
                                    f = 0;
                                    break;
                                }
                                __nanosleep(64);
                            }
                        }
                        f = __shfl_sync(0xffffffffu, f, 0);
                        if (f == 0) {  // the predecessor never published: record and continue
                            if (lane == 0) report_status(p.hdr, kDevTimeout, 3, static_cast<uint32_t>(tile),
                                                         static_cast<uint32_t>(kk), p.spin_limit);
#pragma unroll
                            for (int c = 0; c < 4; ++c) hin[c] = hx[c];
                            break;
                        }
                        (void)ld_acquire_gpu(p.flags + j);  // order this lane's payload reads after the flag
                        if ((f & 3u) == 2u) {
                            const float4 hi = ld_relaxed_gpu_f4(
                                reinterpret_cast<const float4*>(p.pay_incl + j * 64 + cg * 16 + nl * 4));
                            const float hv[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                            for (int c = 0; c < 4; ++c) hin[c] = fmaf(px[c], hv[c], hx[c]);
                            break;
                        }
                        const float4 ha = ld_relaxed_gpu_f4(
                            reinterpret_cast<const float4*>(p.pay_agg + j * 64 + cg * 16 + nl * 4));
                        const float sj = __ldcg(p.pay_sdt + j * 4 + cg);
                        const float hv[4] = {ha.x, ha.y, ha.z, ha.w};
                        const float a2[4] = {A2[0].x, A2[0].y, A2[1].x, A2[1].y};
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            hx[c] = fmaf(px[c], hv[c], hx[c]);
                            px[c] *= ex2_mufu(a2[c] * sj);
                        }
                        if (kk == 0) {  // walked back over every chunk: apply them to the initial state
                            const float4 v = initial();
                            const float h0v[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int c = 0; c < 4; ++c) hin[c] = fmaf(px[c], h0v[c], hx[c]);
                        }
                    }
                }
                if (publish) {
                    if (s == 1) {
                        float inc[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) inc[c] = fmaf(pu[c], hin[c], hu[c]);
                        *reinterpret_cast<float4*>(p.pay_incl + key * 64 + cg * 16 + nl * 4) =
                            make_float4(inc[0], inc[1], inc[2], inc[3]);
                    }
                    fence_acq_rel_gpu();
                    __syncwarp();
                    if (lane == 0) st_release_gpu(p.flags + key, (tag << 2) | 2u);
                }
                if (s == 1) *reinterpret_cast<float4*>(carry + row * 16 + nl * 4) = make_float4(hin[0], hin[1], hin[2], hin[3]);
            }
            named_barrier_sync(1, Cfg::kWarps * 32);

            // Carry-in of this lane's slice: the unit's carry, the earlier time-warps, and
            // (for slice 1) slice 0.
            float2 h[2];
            {
                const float4 ci = *reinterpret_cast<const float4*>(carry + row * 16 + nl * 4);
                float hc[4] = {ci.x, ci.y, ci.z, ci.w};
                for (int w = 0; w < wt; ++w)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 ph = agg[(w * 8 + row) * 16 + nl * 4 + c];
                        hc[c] = fmaf(ph.x, hc[c], ph.y);
                    }
                h[0] = __ffma2_rn(Pex[0], f2(hc[0], hc[1]), Hex[0]);
                h[1] = __ffma2_rn(Pex[1], f2(hc[2], hc[3]), Hex[1]);
            }

            // Pass 2: the slice again from the true carry-in, with the C contraction.
            float yp[GS];
#pragma unroll
            for (int i = 0; i < GS; ++i) {
                const float4 Bq = *reinterpret_cast<const float4*>(bcr0 + i * 32);
                const float4 Cq = *reinterpret_cast<const float4*>(bcr0 + i * 32 + 16);
                const float2 ww = f2(wv[i], wv[i]);
                h[0] = __ffma2_rn(av[i][0], h[0], __fmul2_rn(ww, f2(Bq.x, Bq.y)));
                h[1] = __ffma2_rn(av[i][1], h[1], __fmul2_rn(ww, f2(Bq.z, Bq.w)));
                float2 acc = __fmul2_rn(f2(Cq.x, Cq.y), h[0]);
                acc = __ffma2_rn(f2(Cq.z, Cq.w), h[1], acc);
                yp[i] = acc.x + acc.y;
            }
            // Reduce-scatter over the four lanes of the channel.
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
            // Epilogue: D skip and silu gate, round, store.
            {
                float ue[PER], ze[PER], yo[PER];
                load_run<IO, PER>(st + off + nl * PER * ES, ue);
                if (has_z) load_run<IO, PER>(st + 2 * Cfg::kTile + off + nl * PER * ES, ze);
                const float Dd = (valid && p.D) ? p.D[d] : 0.f;
#pragma unroll
                for (int r = 0; r < PER; ++r) {
                    float v = fmaf(Dd, ue[r], yp[r]);
                    if (has_z) v *= gate_silu<IO>(ze[r]);
                    yo[r] = v;
                }
                const int t0 = k * TC + g * GS + nl * PER;
                if (valid && dcheck(p.hdr, t0 >= p.L || (static_cast<long long>(b) * p.dim + d) * p.L + t0 <
                                                              static_cast<long long>(p.batch) * p.dim * p.L,
                                    kSiteChunkY, t0)) {
                    IO* yrow = static_cast<IO*>(p.y) + (static_cast<long long>(b) * p.dim + d) * p.L;
                    if (t0 + PER <= p.L) {
                        store_run<IO, PER>(yrow + t0, yo);
                    } else {
#pragma unroll
                        for (int r = 0; r < PER; ++r)
                            if (t0 + r < p.L) yrow[t0 + r] = IoTraits<IO>::from_f32(yo[r]);
                    }
                }
            }
            // The state after the last step of the sequence (steps past L are identities).
            if (valid && p.last_state && k == p.nchunks - 1 && wt == NWT - 1 && s == 1 &&
                dcheck(p.hdr, (static_cast<long long>(b) * p.dim + d) * 16 + 16 <= static_cast<long long>(p.batch) * p.dim * 16,
                       kSiteChunkY, d)) {
                float* dst = p.last_state + (static_cast<long long>(b) * p.dim + d) * 16 + nl * 4;
                *reinterpret_cast<float4*>(dst) = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[bi]);
        }
    }

    // The last CTA of the launch leaves the workspace ready for the next one.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&p.hdr->done, 1u) == gridDim.x - 1) {
            p.hdr->ticket = 0u;
            p.hdr->done = 0u;
            __threadfence();
            atomicExch(&p.hdr->epoch, tag);
        }
    }
}

}  // namespace ssm
