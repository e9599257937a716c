// ssm_api.cu -- host side of the C ABI declared in include/ssm_scan.h: argument
// validation, workspace layout, TMA tensor maps, kernel choice and launches.
// Everything here is marshalling; every step of the scan runs in the kernels.
#include <cstdint>
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ssm_scan.h"
#include "aux_kernels.cuh"
#include "common.cuh"
#include "scan_fwd_chunked.cuh"
#include "scan_fwd_seq.cuh"
#include "scan_bwd.cuh"
#include "scan_fwd_wide.cuh"

namespace {

using ssm::WorkspaceHeader;

constexpr int kAbiVersion = 2;
constexpr uint32_t kDefaultWaitLimit = 1u << 22;
// d_state-16 decode: fp32 state values per thread (4, 8 or 16; 16 / that many threads per channel)
constexpr int kDecodeStatesPerThread = 8;
constexpr uint32_t kDefaultSpinLimit = 1u << 21;  // look-back polls (~64 ns sleep each)

size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }

// d_state values of the forward scan and decode: 16 (the tuned kernels) and the wider states
// of scan_fwd_wide.cuh.
bool dstate_supported(int n) { return n == 16 || n == 32 || n == 64 || n == 128 || n == 256; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace layout:
//   [header 256 B][B/C fp32 rows: batch * L * 128 B]
//   [look-back flags: keys * 4 B][aggregate h: keys * 256 B][aggregate sum Delta: keys * 16 B]
//   [inclusive h: keys * 256 B]
// with keys = (8-channel tiles) * 2 columns * ceil(L / 32) chunks (32 steps is the
// shorter chunk of the two element types, so one size serves both).
struct WsLayout {
    size_t bc_off, flags_off, agg_off, sdt_off, incl_off, total;
    long long keys;
};

constexpr int kMinChunk = 32;

WsLayout ws_layout(int batch, int dim, int64_t L) {
    WsLayout w{};
    const long long tiles = static_cast<long long>(batch) * ((dim + 7) / 8);
    w.keys = tiles * 2 * ((L + kMinChunk - 1) / kMinChunk);
    w.bc_off = sizeof(WorkspaceHeader);
    w.flags_off = w.bc_off + round_up(static_cast<size_t>(batch) * static_cast<size_t>(L) * 128u, 256);
    w.agg_off = w.flags_off + round_up(static_cast<size_t>(w.keys) * 4u, 256);
    w.sdt_off = w.agg_off + static_cast<size_t>(w.keys) * 256u;
    w.incl_off = w.sdt_off + static_cast<size_t>(w.keys) * 16u;
    w.total = w.incl_off + static_cast<size_t>(w.keys) * 256u;
    return w;
}

// ------------------------------------------------------------------ driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D tiled map over a dense (d2, d1, d0) tensor with d0 innermost.
bool make_map_3d(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* ptr, uint64_t d0, uint64_t d1,
                 uint64_t d2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

ssm_status_t check_device(int* sm_count) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_LAUNCH;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return SSM_ERR_LAUNCH;
    if (major != 10) return SSM_ERR_UNSUPPORTED;
    if (sm_count && cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SSM_ERR_LAUNCH;
    return SSM_OK;
}

ssm_status_t launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SSM_OK : SSM_ERR_LAUNCH;
}

// Opt a kernel into the largest dynamic shared memory per block the device allows next
// to its static shared memory, once per (kernel, device); `bytes` is checked against it.
bool ensure_smem_attr(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return false;
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return false;
    const int limit = optin - static_cast<int>(fa.sharedSizeBytes);  // static + dynamic <= opt-in maximum
    if (bytes > limit) return false;
    std::lock_guard<std::mutex> lk(mu);
    if (done.count({kernel, dev})) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, limit) != cudaSuccess) return false;
    done.insert({kernel, dev});
    return true;
}

// ------------------------------------------------------------------ forward launches
// Causal conv1d + SiLU prologue of a forward call (conv_k = 0: none; `u` then holds x).
struct ConvArgs {
    const float *w = nullptr, *b = nullptr, *in = nullptr;
    float* out = nullptr;
    void* u_out = nullptr;
    int k = 0;
};

struct FwdArgs {
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *bias;
    int softplus;
    const float* h0;
    int zoh;
    void* y;
    float* last_state;
    int batch, dim;
    int64_t L;
    ssm_dtype_t io;
    uint8_t* ws;
    cudaStream_t stream;
    int sm_count;
    ConvArgs conv;
};

template <typename IO, int G, int CPL, bool ZOH, bool CONV = false>
const void* seq_kernel_ptr(int stages) {
    switch (stages) {
        case 2: return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 2, ZOH, CONV>);
        case 3: return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 3, ZOH, CONV>);
        default: return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 4, ZOH, CONV>);
    }
}

// Launch plan of the sequential kernel: one persistent CTA per SM (two when the tiles
// do not fit one CTA's warps), each taking an even share of the 8-channel tiles, with
// as deep a TMA ring as shared memory allows.
struct SeqPlan {
    long long total_tiles = 0;
    int tiles_per_batch = 0, grid = 0, max_tiles = 0, stages = 0, threads = 0, smem = 0, warps_per_sm = 0;
    bool ok = false;
};

template <typename IO, int G, int CPL, bool ZOH = false, bool CONV = false>
SeqPlan plan_seq(const FwdArgs& a) {
    using Cfg = ssm::SeqCfg<IO, G, CPL>;
    SeqPlan pl;
    pl.tiles_per_batch = ((a.dim + 7) / 8 + Cfg::kTPW - 1) / Cfg::kTPW * Cfg::kTPW;
    pl.total_tiles = static_cast<long long>(a.batch) * pl.tiles_per_batch;
    // At most kMaxWarps consumer warps, and a round may span at most two batch rows.
    // (tiles are handed out in whole-warp units of kTPW tiles).
    const int tiles_cap = std::min(Cfg::kMaxWarps * Cfg::kCPW / 8 / Cfg::kTPW * Cfg::kTPW,
                                   pl.tiles_per_batch + Cfg::kTPW);
    for (int per_sm = 1; per_sm <= 2 && !pl.ok; ++per_sm) {
        const long long ctas = std::min<long long>(pl.total_tiles, static_cast<long long>(a.sm_count) * per_sm);
        const long long units = pl.total_tiles / Cfg::kTPW;  // tiles in whole-warp units
        int mt = static_cast<int>((units + ctas - 1) / ctas) * Cfg::kTPW;
        if (mt > tiles_cap) {
            if (per_sm == 1) continue;
            mt = tiles_cap;  // several rounds per CTA
        }
        const int budget = (228 * 1024) / per_sm - 1024 - 256;  // per-CTA reserve and static barriers
        const int stages = std::min(4, (budget - 1024) / Cfg::stage_bytes(mt));
        if (stages < 2) continue;
        const int threads = (Cfg::warps_for(mt) + 1) * 32;
        const int smem = Cfg::smem_bytes(mt, stages);
        const void* kern = seq_kernel_ptr<IO, G, CPL, ZOH, CONV>(stages);
        int occ = 0;
        if (!ensure_smem_attr(kern, smem) ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess || occ < per_sm)
            continue;
        pl.grid = static_cast<int>(ctas);
        pl.max_tiles = mt;
        pl.stages = stages;
        pl.threads = threads;
        pl.smem = smem;
        pl.warps_per_sm = per_sm * Cfg::warps_for(mt);
        pl.ok = true;
    }
    return pl;
}

// Relative time of a plan: tiles on the busiest SM, a per-element charge for the
// variant, and a latency penalty below ~10 consumer warps per SM.
template <typename IO, int G, int CPL>
double predict_seq(const FwdArgs& a, const SeqPlan& pl) {
    if (!pl.ok) return 1e300;
    const long long per_sm_ctas = (pl.grid + a.sm_count - 1) / a.sm_count;
    const double rounds = std::ceil(static_cast<double>(pl.total_tiles) / pl.grid / pl.max_tiles);
    const double tiles = static_cast<double>(per_sm_ctas) * pl.max_tiles * rounds;
    // Calibrated on B200 (bf16, d_state 16): ~10 resident consumer warps per SM hide the
    // per-step latencies; two channels per lane or two lanes per channel halve the warps
    // for the same tiles and measured slower at equal warp counts.
    const double cost = CPL == 2 ? 1.3 : G == 8 ? 1.12 : 1.0;
    const double hide = std::min(1.0, pl.warps_per_sm / 10.0);
    return tiles * cost / hide;
}

template <typename IO, int G, int CPL, bool ZOH = false, bool CONV = false>
ssm_status_t launch_seq(const FwdArgs& a, const SeqPlan& pl) {
    using Cfg = ssm::SeqCfg<IO, G, CPL>;
    if (!pl.ok) return SSM_ERR_UNSUPPORTED;
    constexpr int TC = Cfg::kTC;
    constexpr auto sw128 = CU_TENSOR_MAP_SWIZZLE_128B;
    const auto dt = ssm::IoTraits<IO>::kTmaType;
    constexpr int es = ssm::IoTraits<IO>::kBytes;
    CUtensorMap mu, mdl, mz, mbc;
    const uint64_t L = static_cast<uint64_t>(a.L);
    bool ok = make_map_3d(&mu, dt, es, a.u, L, a.dim, a.batch, TC, 8, sw128) &&
              make_map_3d(&mdl, dt, es, a.delta, L, a.dim, a.batch, TC, 8, sw128) &&
              make_map_3d(&mbc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.ws + ws_layout(a.batch, a.dim, a.L).bc_off, 32,
                          L, a.batch, 32, TC, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && a.z) ok = make_map_3d(&mz, dt, es, a.z, L, a.dim, a.batch, TC, 8, sw128);
    if (!a.z) mz = mu;
    if (!ok) return SSM_ERR_LAUNCH;
    ssm::SeqParams p{};
    p.A = a.A;
    p.D = a.D;
    p.bias = a.bias;
    p.h0 = a.h0;
    p.last_state = a.last_state;
    p.y = a.y;
    p.hdr = reinterpret_cast<WorkspaceHeader*>(a.ws);
    p.batch = a.batch;
    p.dim = a.dim;
    p.L = a.L;
    p.tiles_per_batch = pl.tiles_per_batch;
    p.total_tiles = pl.total_tiles;
    p.max_tiles = pl.max_tiles;
    p.softplus = a.softplus;
    p.has_z = a.z != nullptr;
    p.wait_limit = kDefaultWaitLimit;
    p.x = a.u;
    p.conv_w = a.conv.w;
    p.conv_b = a.conv.b;
    p.conv_in = a.conv.in;
    p.conv_out = a.conv.out;
    p.u_out = a.conv.u_out;
    p.conv_k = a.conv.k;
    if (a.L >= (1LL << 31) - 1024) return SSM_ERR_UNSUPPORTED;
    switch (pl.stages) {
        case 2: ssm::scan_fwd_seq_kernel<IO, G, CPL, 2, ZOH, CONV><<<pl.grid, pl.threads, pl.smem, a.stream>>>(mu, mdl, mz, mbc, p); break;
        case 3: ssm::scan_fwd_seq_kernel<IO, G, CPL, 3, ZOH, CONV><<<pl.grid, pl.threads, pl.smem, a.stream>>>(mu, mdl, mz, mbc, p); break;
        default: ssm::scan_fwd_seq_kernel<IO, G, CPL, 4, ZOH, CONV><<<pl.grid, pl.threads, pl.smem, a.stream>>>(mu, mdl, mz, mbc, p); break;
    }
    return launch_status();
}

template <typename IO>
ssm_status_t launch_chunked(const FwdArgs& a, const ssm_fwd_options_t& o) {
    using Cfg = ssm::ChunkCfg<IO>;
    constexpr int TC = Cfg::kTC;
    if (a.L >= (1LL << 31) - 1024) return SSM_ERR_UNSUPPORTED;
    constexpr auto sw128 = CU_TENSOR_MAP_SWIZZLE_128B;
    const auto dt = ssm::IoTraits<IO>::kTmaType;
    constexpr int es = ssm::IoTraits<IO>::kBytes;
    const WsLayout wl = ws_layout(a.batch, a.dim, a.L);
    CUtensorMap mu, mdl, mz, mbc;
    const uint64_t L = static_cast<uint64_t>(a.L);
    bool ok = make_map_3d(&mu, dt, es, a.u, L, a.dim, a.batch, TC, 8, sw128) &&
              make_map_3d(&mdl, dt, es, a.delta, L, a.dim, a.batch, TC, 8, sw128) &&
              make_map_3d(&mbc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.ws + wl.bc_off, 32, L, a.batch, 32, TC,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && a.z) ok = make_map_3d(&mz, dt, es, a.z, L, a.dim, a.batch, TC, 8, sw128);
    if (!a.z) mz = mu;
    if (!ok) return SSM_ERR_LAUNCH;
    auto kern = ssm::scan_fwd_chunked_kernel<IO>;
    if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), Cfg::kSmem)) return SSM_ERR_LAUNCH;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, Cfg::kThreads, Cfg::kSmem) != cudaSuccess ||
        occ < 1)
        return SSM_ERR_LAUNCH;
    ssm::ChunkParams p{};
    p.A = a.A;
    p.D = a.D;
    p.bias = a.bias;
    p.last_state = a.last_state;
    p.y = a.y;
    p.hdr = reinterpret_cast<WorkspaceHeader*>(a.ws);
    p.flags = reinterpret_cast<uint32_t*>(a.ws + wl.flags_off);
    p.pay_agg = reinterpret_cast<float*>(a.ws + wl.agg_off);
    p.pay_sdt = reinterpret_cast<float*>(a.ws + wl.sdt_off);
    p.pay_incl = reinterpret_cast<float*>(a.ws + wl.incl_off);
    p.h0 = a.h0;
    p.batch = a.batch;
    p.dim = a.dim;
    p.L = static_cast<int>(a.L);
    p.tiles_per_batch = (a.dim + 7) / 8;
    p.nchunks = static_cast<int>((a.L + TC - 1) / TC);
    p.total_tiles = static_cast<long long>(a.batch) * p.tiles_per_batch;
    p.total_units = p.total_tiles * p.nchunks;
    p.softplus = a.softplus;
    p.has_z = a.z != nullptr;
    p.wait_limit = kDefaultWaitLimit;
    p.spin_limit = o.spin_limit ? o.spin_limit : kDefaultSpinLimit;
    p.debug_skip_chunk = o.debug_skip_publish;
    const long long grid = std::min<long long>(p.total_units, static_cast<long long>(a.sm_count) * occ);
    kern<<<static_cast<unsigned>(grid), Cfg::kThreads, Cfg::kSmem, a.stream>>>(mu, mdl, mz, mbc, p);
    return launch_status();
}

template <typename IO>
ssm_status_t launch_direct(const FwdArgs& a) {
    ssm::DirectParams p{};
    p.u = a.u;
    p.delta = a.delta;
    p.z = a.z;
    p.bc = reinterpret_cast<const float*>(a.ws + ws_layout(a.batch, a.dim, a.L).bc_off);
    p.A = a.A;
    p.D = a.D;
    p.bias = a.bias;
    p.h0 = a.h0;
    p.y = a.y;
    p.last_state = a.last_state;
    p.batch = a.batch;
    p.dim = a.dim;
    p.L = a.L;
    p.softplus = a.softplus;
    p.zoh = a.zoh;
    p.conv_w = a.conv.w;
    p.conv_b = a.conv.b;
    p.conv_in = a.conv.in;
    p.conv_out = a.conv.out;
    p.u_out = a.conv.u_out;
    p.conv_k = a.conv.k;
    constexpr int G = 2;
    const long long threads = static_cast<long long>(a.batch) * a.dim * G;
    const long long grid = (threads + 127) / 128;
    if (grid > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    ssm::scan_fwd_direct_kernel<IO, G><<<static_cast<unsigned>(grid), 128, 0, a.stream>>>(p);
    return launch_status();
}

// The zero-order-hold and conv-prologue kernels exist for 4 and 8 lanes per channel.
template <typename IO, bool ZOH, bool CONV>
ssm_status_t launch_flagged(const FwdArgs& a, const ssm_fwd_options_t& o) {
    const SeqPlan p4 = plan_seq<IO, 4, 1, ZOH, CONV>(a);
    if constexpr (sizeof(IO) == 2) {
        const SeqPlan p8 = plan_seq<IO, 8, 1, ZOH, CONV>(a);
        const bool use8 = o.lanes_per_channel == 8 ||
                          (o.lanes_per_channel == 0 && predict_seq<IO, 8, 1>(a, p8) < predict_seq<IO, 4, 1>(a, p4));
        if (use8) return launch_seq<IO, 8, 1, ZOH, CONV>(a, p8);
    }
    return launch_seq<IO, 4, 1, ZOH, CONV>(a, p4);
}

template <typename IO>
ssm_status_t launch_pack(const FwdArgs& a) {
    const dim3 grid(static_cast<unsigned>((a.L + 63) / 64), static_cast<unsigned>(a.batch));
    ssm::pack_bc_kernel<IO><<<grid, 256, 0, a.stream>>>(
        static_cast<const IO*>(a.B), static_cast<const IO*>(a.C),
        reinterpret_cast<float*>(a.ws + ws_layout(a.batch, a.dim, a.L).bc_off), a.L);
    return launch_status();
}

template <typename IO>
ssm_status_t launch_forward(const FwdArgs& a, const ssm_fwd_options_t& o) {
    ssm_status_t st = launch_pack<IO>(a);
    if (st != SSM_OK) return st;
    const bool tma_ok = (static_cast<uint64_t>(a.L) * ssm::IoTraits<IO>::kBytes) % 16 == 0 && aligned16(a.u) &&
                        aligned16(a.delta) && aligned16(a.y) && (!a.z || aligned16(a.z));
    int algo = o.algo;
    if (!tma_ok) algo = SSM_ALGO_DIRECT;
    if (algo == SSM_ALGO_DIRECT) return launch_direct<IO>(a);
    if ((a.zoh || a.conv.k > 0) && algo == SSM_ALGO_CHUNKED) return SSM_ERR_UNSUPPORTED;  // plain scan only
    if (algo == SSM_ALGO_AUTO && (a.zoh || a.conv.k > 0)) algo = SSM_ALGO_SEQUENTIAL;
    if (algo == SSM_ALGO_AUTO) {
        // The sequential kernel is faster whenever the channels alone give each SM a few
        // warps (measured on B200: at 5120 channels x 32768 steps it runs at ~1.8x the
        // chunked kernel).  Split the sequence across CTAs only when fewer than 4 warps of
        // 8-lane channels per SM would be resident, and the sequence is long.
        const double warps_per_sm = static_cast<double>(a.batch) * a.dim * 8.0 / 32.0 / a.sm_count;
        const long long chunks = (a.L + ssm::ChunkCfg<IO>::kTC - 1) / ssm::ChunkCfg<IO>::kTC;
        algo = (warps_per_sm < 4.0 && chunks >= 64) ? SSM_ALGO_CHUNKED : SSM_ALGO_SEQUENTIAL;
    }
    if (algo == SSM_ALGO_CHUNKED) return launch_chunked<IO>(a, o);
    // Variants: (lanes per channel G, channels per lane CPL).  lanes_per_channel selects
    // G explicitly (CPL = 1), or G = 4 with CPL = 2 when given as 42.  The zero-order-hold
    // weight is built into the 4- and 8-lane variants only.
    if (a.zoh || a.conv.k > 0) {
        if (a.zoh && a.conv.k > 0) return launch_flagged<IO, true, true>(a, o);
        if (a.zoh) return launch_flagged<IO, true, false>(a, o);
        return launch_flagged<IO, false, true>(a, o);
    }
    const SeqPlan p2 = plan_seq<IO, 2, 1>(a), p4 = plan_seq<IO, 4, 1>(a), p42 = plan_seq<IO, 4, 2>(a);
    SeqPlan p8;
    if constexpr (sizeof(IO) == 2) p8 = plan_seq<IO, 8, 1>(a);
    int G = o.lanes_per_channel;
    if (G == 0) {
        const double t[4] = {predict_seq<IO, 2, 1>(a, p2), predict_seq<IO, 4, 1>(a, p4),
                             sizeof(IO) == 2 ? predict_seq<IO, 8, 1>(a, p8) : 1e300, predict_seq<IO, 4, 2>(a, p42)};
        const int ids[4] = {2, 4, 8, 42};
        int best = 1;
        for (int i = 0; i < 4; ++i)
            if (t[i] < t[best]) best = i;
        G = ids[best];
    }
    if (G == 2) return launch_seq<IO, 2, 1>(a, p2);
    if (G == 4) return launch_seq<IO, 4, 1>(a, p4);
    if (G == 42) return launch_seq<IO, 4, 2>(a, p42);
    if constexpr (sizeof(IO) == 2)
        if (G == 8) return launch_seq<IO, 8, 1>(a, p8);
    return SSM_ERR_INVALID_ARG;
}

// ------------------------------------------------------------------ wider states
template <typename IO, int N>
ssm_status_t launch_wide_n(const FwdArgs& a) {
    float* bc = reinterpret_cast<float*>(a.ws + sizeof(WorkspaceHeader));
    const dim3 pgrid(static_cast<unsigned>((a.L + 31) / 32), static_cast<unsigned>(a.batch), 2 * N / 32);
    ssm::pack_bc_wide_kernel<IO><<<pgrid, dim3(32, 8), 0, a.stream>>>(static_cast<const IO*>(a.B),
                                                                    static_cast<const IO*>(a.C), bc, a.L, N);
    if (cudaGetLastError() != cudaSuccess) return SSM_ERR_LAUNCH;
    ssm::WideParams p{};
    p.u = a.u;
    p.delta = a.delta;
    p.z = a.z;
    p.bc = bc;
    p.A = a.A;
    p.D = a.D;
    p.bias = a.bias;
    p.h0 = a.h0;
    p.y = a.y;
    p.last_state = a.last_state;
    p.batch = a.batch;
    p.dim = a.dim;
    p.L = a.L;
    p.softplus = a.softplus;
    p.zoh = a.zoh;
    using Cfg = ssm::WideCfg<N>;
    auto kern = ssm::scan_fwd_wide_kernel<IO, N>;
    if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), Cfg::kSmem)) return SSM_ERR_LAUNCH;
    const dim3 grid(static_cast<unsigned>((a.dim + Cfg::kCPB - 1) / Cfg::kCPB), static_cast<unsigned>(a.batch));
    kern<<<grid, Cfg::kWarps * 32, Cfg::kSmem, a.stream>>>(p);
    return launch_status();
}

template <typename IO>
ssm_status_t launch_wide(const FwdArgs& a, int n) {
    switch (n) {
        case 32: return launch_wide_n<IO, 32>(a);
        case 64: return launch_wide_n<IO, 64>(a);
        case 128: return launch_wide_n<IO, 128>(a);
        case 256: return launch_wide_n<IO, 256>(a);
    }
    return SSM_ERR_UNSUPPORTED;
}

template <typename IO, int N>
void launch_decode_wide(float* state, const void* u, const void* delta, const float* A, const void* B, const void* C,
                        const float* D, const void* z, const float* bias, int softplus, void* y, int batch, int dim,
                        int zoh, unsigned grid, cudaStream_t s) {
    ssm::state_update_wide_kernel<IO, N><<<grid, 256, 0, s>>>(A, D, bias, state, u, delta, B, C, z, y, batch, dim,
                                                             softplus, zoh);
}

// ------------------------------------------------------------------ backward
// Backward workspace layout:
//   [header 256 B][B/C fp32 rows: batch * L * 128 B][checkpoints: batch * nseg * dim * 64 B]
//   [dB/dC per CTA: batch * ncta * L * 128 B][dA per batch row: batch * dim * 64 B]
//   [dD per batch row: batch * dim * 4 B][ddelta_bias per batch row: batch * dim * 4 B]
struct BwdLayout {
    size_t bc_off, ckpt_off, dbc_off, dA_off, dD_off, dbias_off, total;
    int nseg, ncta;
};

BwdLayout bwd_layout(int batch, int dim, int64_t L) {
    BwdLayout w{};
    w.nseg = static_cast<int>((L + ssm::kBwdSeg - 1) / ssm::kBwdSeg);
    w.ncta = (dim + ssm::kBwdChannels - 1) / ssm::kBwdChannels;
    const size_t B = static_cast<size_t>(batch), D = static_cast<size_t>(dim), Ls = static_cast<size_t>(L);
    w.bc_off = sizeof(WorkspaceHeader);
    w.ckpt_off = w.bc_off + round_up(B * Ls * 128u, 256);
    w.dbc_off = w.ckpt_off + round_up(B * static_cast<size_t>(w.nseg) * D * 64u, 256);
    w.dA_off = w.dbc_off + round_up(B * static_cast<size_t>(w.ncta) * Ls * 128u, 256);
    w.dD_off = w.dA_off + round_up(B * D * 64u, 256);
    w.dbias_off = w.dD_off + round_up(B * D * 4u, 256);
    w.total = w.dbias_off + round_up(B * D * 4u, 256);
    return w;
}

struct BwdArgs {
    const void *u, *delta, *B, *C, *z, *dy;
    const float *A, *D, *bias, *h0, *dlast;
    int softplus;
    void *du, *ddelta, *dz;
    float *dA, *dB, *dC, *dD, *dbias, *dh0;
    int batch, dim;
    int64_t L;
    uint8_t* ws;
    cudaStream_t stream;
};

template <typename IO>
ssm_status_t launch_backward(const BwdArgs& a) {
    const BwdLayout wl = bwd_layout(a.batch, a.dim, a.L);
    uint8_t* bc = a.ws + wl.bc_off;
    {
        // B/C rows for the kernel's ring: bf16 inputs stay bf16 (state pairs), fp32 as rows
        const dim3 grid(static_cast<unsigned>((a.L + 63) / 64), static_cast<unsigned>(a.batch));
        if constexpr (sizeof(IO) == 2)
            ssm::pack_bc_pairs_kernel<<<grid, 256, 0, a.stream>>>(static_cast<const uint16_t*>(a.B),
                                                                  static_cast<const uint16_t*>(a.C),
                                                                  reinterpret_cast<uint32_t*>(bc), a.L);
        else
            ssm::pack_bc_kernel<IO><<<grid, 256, 0, a.stream>>>(static_cast<const IO*>(a.B),
                                                               static_cast<const IO*>(a.C),
                                                               reinterpret_cast<float*>(bc), a.L);
        if (cudaGetLastError() != cudaSuccess) return SSM_ERR_LAUNCH;
    }
    ssm::BwdParams p{};
    p.u = a.u;
    p.delta = a.delta;
    p.z = a.z;
    p.dy = a.dy;
    p.bc = bc;
    p.A = a.A;
    p.D = a.D;
    p.bias = a.bias;
    p.h0 = a.h0;
    p.dlast = a.dlast;
    p.du = a.du;
    p.ddelta = a.ddelta;
    p.dz = a.dz;
    p.dh0 = a.dh0;
    p.ckpt = reinterpret_cast<float*>(a.ws + wl.ckpt_off);
    p.dbc_part = reinterpret_cast<float*>(a.ws + wl.dbc_off);
    p.dA_part = reinterpret_cast<float*>(a.ws + wl.dA_off);
    p.dD_part = reinterpret_cast<float*>(a.ws + wl.dD_off);
    p.dbias_part = reinterpret_cast<float*>(a.ws + wl.dbias_off);
    p.batch = a.batch;
    p.dim = a.dim;
    p.L = a.L;
    p.nseg = wl.nseg;
    p.ncta = wl.ncta;
    p.softplus = a.softplus;
    constexpr int smem = ssm::kBwdSmem;
    auto kern = ssm::scan_bwd_kernel<IO>;
    if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), smem)) return SSM_ERR_LAUNCH;
    kern<<<dim3(static_cast<unsigned>(wl.ncta), static_cast<unsigned>(a.batch)), ssm::kBwdWarps * 32, smem,
           a.stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SSM_ERR_LAUNCH;
    ssm::BwdFinalParams f{};
    f.dbc_part = p.dbc_part;
    f.dA_part = p.dA_part;
    f.dD_part = p.dD_part;
    f.dbias_part = p.dbias_part;
    f.dB = a.dB;
    f.dC = a.dC;
    f.dA = a.dA;
    f.dD = a.dD;
    f.dbias = a.dbias;
    f.batch = a.batch;
    f.dim = a.dim;
    f.ncta = wl.ncta;
    f.L = a.L;
    ssm::scan_bwd_reduce_bc_kernel<<<dim3(static_cast<unsigned>((a.L + 31) / 32), static_cast<unsigned>(a.batch)), 256,
                                     0, a.stream>>>(f);
    const long long n = static_cast<long long>(a.dim) * 16;
    ssm::scan_bwd_reduce_params_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, a.stream>>>(f);
    return launch_status();
}

// Fixed scratch of ssm_selective_scan_fwd_noalloc (header + transposed B/C rows).  In
// host code this name only stands for the array: its device address comes from
// cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSM_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device (nullptr on failure).
void* noalloc_scratch_ptr() {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

int ssm_abi_version(void) { return kAbiVersion; }

const char* ssm_status_string(ssm_status_t s) {
    switch (s) {
        case SSM_OK: return "ok";
        case SSM_ERR_INVALID_ARG: return "invalid argument";
        case SSM_ERR_UNSUPPORTED: return "unsupported configuration";
        case SSM_ERR_LAUNCH: return "CUDA launch or runtime error";
        case SSM_ERR_TIMEOUT: return "device wait timed out";
        case SSM_ERR_WORKSPACE: return "workspace missing or too small";
        case SSM_ERR_SCRATCH_LIMIT: return "problem larger than the fixed scratch of the no-allocation entry point";
    }
    return "unknown status";
}

size_t ssm_selective_scan_workspace_size(int batch, int dim, int dstate, int64_t seqlen) {
    if (batch < 0 || dim < 0 || !dstate_supported(dstate) || seqlen < 0) return 0;
    if (dstate != 16)  // header + B/C rows of 2 * dstate fp32 per step
        return sizeof(WorkspaceHeader) +
               round_up(static_cast<size_t>(batch) * static_cast<size_t>(seqlen) * 8u * dstate, 256);
    return round_up(ws_layout(batch, dim, seqlen).total, 256);
}

ssm_status_t ssm_workspace_init(void* workspace, size_t workspace_bytes, ssm_stream_t stream) {
    if (!workspace || workspace_bytes < sizeof(WorkspaceHeader)) return SSM_ERR_WORKSPACE;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SSM_OK
               : SSM_ERR_LAUNCH;
}

}  // extern "C"

namespace {
ssm_status_t forward_entry(const void* u, const void* delta, const float* A, const void* B, const void* C,
                           const float* D, const void* z, const float* delta_bias, int softplus,
                           const float* initial_state, void* y, float* last_state, int batch, int dim, int dstate,
                           int64_t seqlen, ssm_dtype_t io_dtype, void* workspace, size_t workspace_bytes,
                           const ssm_fwd_options_t* opts, ssm_stream_t stream, const ConvArgs& conv) {
    if (batch < 0 || dim < 0 || seqlen < 0) return SSM_ERR_INVALID_ARG;
    // Tensors with elements must have a pointer; zero-element tensors may be NULL.
    const bool seq_elems = batch > 0 && dim > 0 && seqlen > 0;
    if (seq_elems && (!u || !delta || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    if (dim > 0 && !A) return SSM_ERR_INVALID_ARG;
    if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
    if (!dstate_supported(dstate)) return SSM_ERR_UNSUPPORTED;
    const void* ptrs[] = {u, delta, A, B, C, D, z, delta_bias, initial_state, y, last_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_INVALID_ARG;
    const size_t state_bytes = static_cast<size_t>(batch) * static_cast<size_t>(dim) * dstate * sizeof(float);
    if (initial_state && last_state && state_bytes > 0) {
        // The chunked kernel may still read a channel's initial state after another CTA
        // has written that channel's final state, so the two must not overlap.
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(initial_state), a1 = reinterpret_cast<uintptr_t>(last_state);
        if ((a0 <= a1 ? a1 - a0 : a0 - a1) < state_bytes) return SSM_ERR_INVALID_ARG;
    }
    ssm_fwd_options_t o{SSM_ALGO_AUTO, 0, 0, -1, SSM_DISC_SIMPLIFIED};
    if (opts) o = *opts;
    if (o.algo < SSM_ALGO_AUTO || o.algo > SSM_ALGO_DIRECT) return SSM_ERR_INVALID_ARG;
    if (o.discretization != SSM_DISC_SIMPLIFIED && o.discretization != SSM_DISC_ZOH) return SSM_ERR_INVALID_ARG;
    if (batch == 0 || dim == 0) return SSM_OK;
    if (batch > 65535) return SSM_ERR_UNSUPPORTED;  // batch is a grid y-dimension of the B/C pack
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        workspace_bytes < ssm_selective_scan_workspace_size(batch, dim, dstate, seqlen))
        return SSM_ERR_WORKSPACE;
    int sm_count = 0;
    ssm_status_t st = check_device(&sm_count);
    if (st != SSM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (seqlen == 0) {  // no steps: the final state is the initial one
        if (last_state) {
            const cudaError_t e = initial_state
                                      ? cudaMemcpyAsync(last_state, initial_state, state_bytes,
                                                        cudaMemcpyDeviceToDevice, s)
                                      : cudaMemsetAsync(last_state, 0, state_bytes, s);
            if (e != cudaSuccess) return SSM_ERR_LAUNCH;
        }
        return SSM_OK;
    }
    FwdArgs a{u, delta, B, C, z, A, D, delta_bias, softplus, initial_state, o.discretization == SSM_DISC_ZOH, y,
              last_state, batch, dim, seqlen, io_dtype, static_cast<uint8_t*>(workspace), s, sm_count, conv};
    if (dstate != 16) {
        if (o.algo == SSM_ALGO_CHUNKED || conv.k > 0) return SSM_ERR_UNSUPPORTED;  // d_state 16 only
        return io_dtype == SSM_BF16 ? launch_wide<__nv_bfloat16>(a, dstate) : launch_wide<float>(a, dstate);
    }
    return io_dtype == SSM_BF16 ? launch_forward<__nv_bfloat16>(a, o) : launch_forward<float>(a, o);
}
}  // namespace

extern "C" {

ssm_status_t ssm_selective_scan_fwd_state(const void* u, const void* delta, const float* A, const void* B,
                                          const void* C, const float* D, const void* z, const float* delta_bias,
                                          int softplus, const float* initial_state, void* y, float* last_state,
                                          int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
                                          void* workspace, size_t workspace_bytes, const ssm_fwd_options_t* opts,
                                          ssm_stream_t stream) {
    return forward_entry(u, delta, A, B, C, D, z, delta_bias, softplus, initial_state, y, last_state, batch, dim,
                         dstate, seqlen, io_dtype, workspace, workspace_bytes, opts, stream, ConvArgs{});
}

ssm_status_t ssm_selective_scan_fwd_conv(const void* x, const ssm_conv_t* conv, const void* delta, const float* A,
                                         const void* B, const void* C, const float* D, const void* z,
                                         const float* delta_bias, int softplus, const float* initial_state, void* y,
                                         float* last_state, int batch, int dim, int dstate, int64_t seqlen,
                                         ssm_dtype_t io_dtype, void* workspace, size_t workspace_bytes,
                                         const ssm_fwd_options_t* opts, ssm_stream_t stream) {
    if (!conv || conv->width < 1 || conv->width > 4) return SSM_ERR_INVALID_ARG;
    if (dim > 0 && !conv->weight) return SSM_ERR_INVALID_ARG;
    if (batch > 0 && dim > 0 && seqlen > 0 && conv->u_out && !aligned16(conv->u_out)) return SSM_ERR_INVALID_ARG;
    if (dstate != 16) return SSM_ERR_UNSUPPORTED;
    ConvArgs c;
    c.w = conv->weight;
    c.b = conv->bias;
    c.in = conv->width > 1 ? conv->state_in : nullptr;
    c.out = conv->width > 1 ? conv->state_out : nullptr;
    c.u_out = conv->u_out;
    c.k = conv->width;
    if (seqlen == 0 && c.out && batch > 0 && dim > 0) {  // nothing to scan: the conv state passes through
        ssm_status_t st = forward_entry(x, delta, A, B, C, D, z, delta_bias, softplus, initial_state, y, last_state,
                                        batch, dim, dstate, seqlen, io_dtype, workspace, workspace_bytes, opts,
                                        stream, c);
        if (st != SSM_OK) return st;
        const size_t bytes = static_cast<size_t>(batch) * dim * (c.k - 1) * sizeof(float);
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        cudaError_t e = cudaSuccess;
        if (!c.in) e = cudaMemsetAsync(c.out, 0, bytes, s);
        else if (c.in != c.out) e = cudaMemcpyAsync(c.out, c.in, bytes, cudaMemcpyDeviceToDevice, s);
        return e == cudaSuccess ? SSM_OK : SSM_ERR_LAUNCH;
    }
    return forward_entry(x, delta, A, B, C, D, z, delta_bias, softplus, initial_state, y, last_state, batch, dim,
                         dstate, seqlen, io_dtype, workspace, workspace_bytes, opts, stream, c);
}

ssm_status_t ssm_selective_scan_fwd_ex(const void* u, const void* delta, const float* A, const void* B,
                                       const void* C, const float* D, const void* z, const float* delta_bias,
                                       int softplus, void* y, float* last_state, int batch, int dim, int dstate,
                                       int64_t seqlen, ssm_dtype_t io_dtype, void* workspace,
                                       size_t workspace_bytes, const ssm_fwd_options_t* opts, ssm_stream_t stream) {
    return ssm_selective_scan_fwd_state(u, delta, A, B, C, D, z, delta_bias, softplus, nullptr, y, last_state, batch,
                                        dim, dstate, seqlen, io_dtype, workspace, workspace_bytes, opts, stream);
}

ssm_status_t ssm_selective_scan_fwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                                    const float* D, const void* z, const float* delta_bias, int softplus, void* y,
                                    float* last_state, int batch, int dim, int dstate, int64_t seqlen,
                                    ssm_dtype_t io_dtype, void* workspace, size_t workspace_bytes,
                                    ssm_stream_t stream) {
    return ssm_selective_scan_fwd_ex(u, delta, A, B, C, D, z, delta_bias, softplus, y, last_state, batch, dim,
                                     dstate, seqlen, io_dtype, workspace, workspace_bytes, nullptr, stream);
}

ssm_status_t ssm_state_update(float* state, const void* u, const void* delta, const float* A, const void* B,
                              const void* C, const float* D, const void* z, const float* delta_bias, int softplus,
                              void* y, int batch, int dim, int dstate, ssm_dtype_t io_dtype, ssm_stream_t stream) {
    return ssm_state_update_ex(state, u, delta, A, B, C, D, z, delta_bias, softplus, y, batch, dim, dstate, io_dtype,
                               SSM_DISC_SIMPLIFIED, stream);
}

ssm_status_t ssm_state_update_ex(float* state, const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* D, const void* z, const float* delta_bias, int softplus,
                                 void* y, int batch, int dim, int dstate, ssm_dtype_t io_dtype,
                                 ssm_discretization_t discretization, ssm_stream_t stream) {
    return ssm_state_update_conv(state, nullptr, u, nullptr, nullptr, 0, delta, A, B, C, D, z, delta_bias, softplus, y,
                                 batch, dim, dstate, io_dtype, discretization, stream);
}

ssm_status_t ssm_state_update_conv(float* state, float* conv_state, const void* x, const float* conv_weight,
                                   const float* conv_bias, int conv_width, const void* delta, const float* A,
                                   const void* B, const void* C, const float* D, const void* z,
                                   const float* delta_bias, int softplus, void* y, int batch, int dim, int dstate,
                                   ssm_dtype_t io_dtype, ssm_discretization_t discretization, ssm_stream_t stream) {
    const void* u = x;
    if (conv_width < 0 || conv_width > 4) return SSM_ERR_INVALID_ARG;
    if (conv_width > 0 && batch > 0 && dim > 0 && (!conv_weight || (conv_width > 1 && !conv_state)))
        return SSM_ERR_INVALID_ARG;
    if (conv_width > 0 && dstate != 16) return SSM_ERR_UNSUPPORTED;
    if (batch < 0 || dim < 0) return SSM_ERR_INVALID_ARG;
    if (discretization != SSM_DISC_SIMPLIFIED && discretization != SSM_DISC_ZOH) return SSM_ERR_INVALID_ARG;
    if (batch > 0 && dim > 0 && (!state || !u || !delta || !A || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
    if (!dstate_supported(dstate)) return SSM_ERR_UNSUPPORTED;
    if (!aligned16(state) || !aligned16(A)) return SSM_ERR_INVALID_ARG;
    if (batch == 0 || dim == 0) return SSM_OK;
    if (dstate == 16 && batch > 65535) return SSM_ERR_UNSUPPORTED;  // the batch row is a grid y index
    ssm_status_t st = check_device(nullptr);
    if (st != SSM_OK) return st;
    if (dstate != 16) {
        const int tpc = std::min(dstate / 4, 32);  // threads per channel
        const long long threads = static_cast<long long>(batch) * dim * tpc;
        const long long grid = (threads + 255) / 256;
        if (grid > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        const int zoh = discretization == SSM_DISC_ZOH;
        const unsigned g = static_cast<unsigned>(grid);
#define SSM_DECODE_WIDE(IO_T)                                                                                        \
    switch (dstate) {                                                                                                \
        case 32: launch_decode_wide<IO_T, 32>(state, u, delta, A, B, C, D, z, delta_bias, softplus, y, batch, dim, zoh, g, s); break; \
        case 64: launch_decode_wide<IO_T, 64>(state, u, delta, A, B, C, D, z, delta_bias, softplus, y, batch, dim, zoh, g, s); break; \
        case 128: launch_decode_wide<IO_T, 128>(state, u, delta, A, B, C, D, z, delta_bias, softplus, y, batch, dim, zoh, g, s); break; \
        default: launch_decode_wide<IO_T, 256>(state, u, delta, A, B, C, D, z, delta_bias, softplus, y, batch, dim, zoh, g, s); break; \
    }
        if (io_dtype == SSM_BF16) {
            SSM_DECODE_WIDE(__nv_bfloat16)
        } else {
            SSM_DECODE_WIDE(float)
        }
#undef SSM_DECODE_WIDE
        return launch_status();
    }
    ssm::DecodeParams p{state, u, delta, A, B, C, D, z, delta_bias, y, batch, dim, softplus,
                        discretization == SSM_DISC_ZOH, aligned16(B) && aligned16(C),
                        conv_weight, conv_bias, conv_state, conv_width};
    constexpr int NS = kDecodeStatesPerThread;
    constexpr int TH = ssm::kDecodeThreads;
    const dim3 g(static_cast<unsigned>((static_cast<long long>(dim) * (16 / NS) + TH - 1) / TH),
                 static_cast<unsigned>(batch));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool zoh = discretization == SSM_DISC_ZOH, conv = conv_width > 0;
#define SSM_DECODE(IO_T)                                                                              \
    if (zoh && conv) ssm::state_update_kernel<IO_T, true, true, NS><<<g, TH, 0, s>>>(p);             \
    else if (zoh) ssm::state_update_kernel<IO_T, true, false, NS><<<g, TH, 0, s>>>(p);               \
    else if (conv) ssm::state_update_kernel<IO_T, false, true, NS><<<g, TH, 0, s>>>(p);              \
    else ssm::state_update_kernel<IO_T, false, false, NS><<<g, TH, 0, s>>>(p);
    if (io_dtype == SSM_BF16) {
        SSM_DECODE(__nv_bfloat16)
    } else {
        SSM_DECODE(float)
    }
#undef SSM_DECODE
    return launch_status();
}

ssm_status_t ssm_selective_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B,
                                             const void* C, const float* D, const void* z, const float* delta_bias,
                                             int softplus, void* y, float* last_state, int batch, int dim, int dstate,
                                             int64_t seqlen, ssm_dtype_t io_dtype, ssm_stream_t stream) {
    if (batch < 0 || dim < 0 || seqlen < 0) return SSM_ERR_INVALID_ARG;
    const bool seq_elems = batch > 0 && dim > 0 && seqlen > 0;
    if (seq_elems && (!u || !delta || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    if (dim > 0 && !A) return SSM_ERR_INVALID_ARG;
    if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
    if (dstate != 16) return SSM_ERR_UNSUPPORTED;
    const void* ptrs[] = {u, delta, A, B, C, D, z, delta_bias, y, last_state};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_INVALID_ARG;
    if (batch == 0 || dim == 0) return SSM_OK;
    if (batch > 65535) return SSM_ERR_UNSUPPORTED;
    // The kernels this entry point runs (sequential or direct) use only the header and the
    // B/C rows, i.e. the workspace up to the look-back region: 256 + round_up(batch*L*128, 256).
    if (ws_layout(batch, dim, seqlen).flags_off > SSM_NOALLOC_SCRATCH_BYTES) return SSM_ERR_SCRATCH_LIMIT;
    int sm_count = 0;
    ssm_status_t st = check_device(&sm_count);
    if (st != SSM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (seqlen == 0) {
        if (last_state &&
            cudaMemsetAsync(last_state, 0, static_cast<size_t>(batch) * dim * 16 * sizeof(float), s) != cudaSuccess)
            return SSM_ERR_LAUNCH;
        return SSM_OK;
    }
    uint8_t* scratch = static_cast<uint8_t*>(noalloc_scratch_ptr());
    if (!scratch) return SSM_ERR_LAUNCH;
    // The header (status word) starts every call at zero; the B/C rows are rewritten in full.
    if (cudaMemsetAsync(scratch, 0, sizeof(WorkspaceHeader), s) != cudaSuccess) return SSM_ERR_LAUNCH;
    // Kernels whose scratch is only the header and the B/C rows (no look-back flags).
    const ssm_fwd_options_t o{SSM_ALGO_SEQUENTIAL, 0, 0, -1, SSM_DISC_SIMPLIFIED};
    FwdArgs a{u, delta, B, C, z, A, D, delta_bias, softplus, nullptr, 0, y, last_state, batch, dim, seqlen,
              io_dtype, scratch, s, sm_count};
    return io_dtype == SSM_BF16 ? launch_forward<__nv_bfloat16>(a, o) : launch_forward<float>(a, o);
}

size_t ssm_selective_scan_bwd_workspace_size(int batch, int dim, int dstate, int64_t seqlen) {
    if (batch < 0 || dim < 0 || dstate != 16 || seqlen < 0) return 0;
    return round_up(bwd_layout(batch, dim, seqlen).total, 256);
}

ssm_status_t ssm_selective_scan_bwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                                    const float* D, const void* z, const float* delta_bias, int softplus,
                                    const float* initial_state, const void* dy, const float* dlast_state, void* du,
                                    void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
                                    float* ddelta_bias, float* dinitial_state, int batch, int dim, int dstate,
                                    int64_t seqlen, ssm_dtype_t io_dtype, void* workspace, size_t workspace_bytes,
                                    ssm_stream_t stream) {
    if (batch < 0 || dim < 0 || seqlen < 0) return SSM_ERR_INVALID_ARG;
    const bool seq_elems = batch > 0 && dim > 0 && seqlen > 0;
    if (seq_elems && (!u || !delta || !B || !C || !dy || !du || !ddelta || !dB || !dC || (z && !dz)))
        return SSM_ERR_INVALID_ARG;
    if (dim > 0 && (!A || !dA)) return SSM_ERR_INVALID_ARG;
    if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
    if (dstate != 16) return SSM_ERR_UNSUPPORTED;
    const void* ptrs[] = {u, delta, A, B, C, D, z, delta_bias, initial_state, dy, dlast_state, du, ddelta, dA, dB, dC,
                          dD, dz, ddelta_bias, dinitial_state};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return SSM_ERR_INVALID_ARG;
    if (batch == 0 || dim == 0) return SSM_OK;
    if (batch > 65535) return SSM_ERR_UNSUPPORTED;
    if (seqlen >= (1LL << 31) - 1024) return SSM_ERR_UNSUPPORTED;  // steps are 32-bit in the kernel
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        workspace_bytes < ssm_selective_scan_bwd_workspace_size(batch, dim, dstate, seqlen))
        return SSM_ERR_WORKSPACE;
    ssm_status_t st = check_device(nullptr);
    if (st != SSM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (seqlen == 0) {  // no steps: only the state passes through
        const size_t state_bytes = static_cast<size_t>(batch) * dim * 16 * sizeof(float);
        cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(dim) * 16 * sizeof(float), s);
        if (e == cudaSuccess && dD) e = cudaMemsetAsync(dD, 0, static_cast<size_t>(dim) * sizeof(float), s);
        if (e == cudaSuccess && ddelta_bias)
            e = cudaMemsetAsync(ddelta_bias, 0, static_cast<size_t>(dim) * sizeof(float), s);
        if (e == cudaSuccess && dinitial_state)
            e = dlast_state ? cudaMemcpyAsync(dinitial_state, dlast_state, state_bytes, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(dinitial_state, 0, state_bytes, s);
        return e == cudaSuccess ? SSM_OK : SSM_ERR_LAUNCH;
    }
    BwdArgs a{u, delta, B, C, z, dy, A, D, delta_bias, initial_state, dlast_state, softplus, du, ddelta, dz, dA, dB,
              dC, dD, ddelta_bias, dinitial_state, batch, dim, seqlen, static_cast<uint8_t*>(workspace), s};
    return io_dtype == SSM_BF16 ? launch_backward<__nv_bfloat16>(a) : launch_backward<float>(a);
}

ssm_status_t ssm_read_status(void* workspace, ssm_stream_t stream) {
    if (!workspace) return SSM_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSM_ERR_LAUNCH;
    uint32_t code = 0;
    auto* hdr = static_cast<WorkspaceHeader*>(workspace);
    if (cudaMemcpy(&code, &hdr->status, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess) return SSM_ERR_LAUNCH;
    if (code != 0 && cudaMemset(&hdr->status, 0, sizeof(uint32_t)) != cudaSuccess) return SSM_ERR_LAUNCH;
    return static_cast<ssm_status_t>(code);
}

}  // extern "C"
