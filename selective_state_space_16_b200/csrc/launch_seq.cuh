// launch_seq.cuh -- launch planning of the sequential forward kernel family
// (scan_fwd_seq.cuh): one persistent CTA per SM, lanes per channel chosen by a cost model.
// Included by the fwd_seq_*.cu translation units, each instantiating one element type.
#pragma once

#include <algorithm>
#include <cmath>

#include "host_common.h"
#include "scan_fwd_seq.cuh"

namespace ssmh {

template <typename IO, int G, int CPL, bool ZOH, bool CONV = false, bool CK = false, bool GA = false>
const void* seq_kernel_ptr(int stages) {
    if constexpr (GA) {  // (gathered rows: rings of 3 or 4 stages)
        if (stages == 3) return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 3, ZOH, CONV, CK, true>);
        return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 4, ZOH, CONV, CK, true>);
    } else {
        switch (stages) {
            case 2: return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 2, ZOH, CONV, CK>);
            case 3: return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 3, ZOH, CONV, CK>);
            default: return reinterpret_cast<const void*>(ssm::scan_fwd_seq_kernel<IO, G, CPL, 4, ZOH, CONV, CK>);
        }
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

template <typename IO, int G, int CPL, bool ZOH = false, bool CONV = false, bool CK = false, bool GA = false>
SeqPlan plan_seq(const FwdArgs& a) {
    using Cfg = ssm::SeqCfg<IO, G, CPL>;
    SeqPlan pl;
    pl.tiles_per_batch = ((a.dim + 7) / 8 + Cfg::kTPW - 1) / Cfg::kTPW * Cfg::kTPW;
    pl.total_tiles = static_cast<long long>(a.batch) * pl.tiles_per_batch;
    // At most kMaxWarps consumer warps, and a round may span at most two batch rows.
    // (tiles are handed out in whole-warp units of kTPW tiles).
    const int tiles_cap = std::min(Cfg::kMaxWarps * Cfg::kCPW / 8 / Cfg::kTPW * Cfg::kTPW,
                                   pl.tiles_per_batch + Cfg::kTPW);
    // Attempts: one CTA per SM in one round; two per SM (several rounds when needed); one per SM
    // in several rounds (shapes with more tiles than two CTAs' warps hold, e.g. b8 d5120, where
    // two CTAs of that size do not fit an SM's registers; the GA kernels' ring needs three
    // stages, which two CTAs per SM do not leave room for).
    for (int at = 0; at < 3 && !pl.ok; ++at) {
        const int per_sm = at == 1 ? 2 : 1;
        const long long ctas = std::min<long long>(pl.total_tiles, static_cast<long long>(a.sm_count) * per_sm);
        const long long units = pl.total_tiles / Cfg::kTPW;  // tiles in whole-warp units
        int mt = static_cast<int>((units + ctas - 1) / ctas) * Cfg::kTPW;
        if (mt > tiles_cap) {
            if (at == 0) continue;
            mt = tiles_cap;  // several rounds per CTA
        }
        const int budget = (228 * 1024) / per_sm - 1024 - 256;  // per-CTA reserve and static barriers
        const int info = GA ? Cfg::gather_info_bytes(mt) : 0;  // (gathered rows: one word per row)
        const int stages = std::min(4, (budget - 1024 - info) / Cfg::stage_bytes(mt));
        if (stages < (GA ? 3 : 2)) continue;
        const int threads = (Cfg::warps_for(mt) + 1) * 32;
        const int smem = Cfg::smem_bytes(mt, stages) + info;
        const void* kern = seq_kernel_ptr<IO, G, CPL, ZOH, CONV, CK, GA>(stages);
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

template <typename IO, int G, int CPL, bool ZOH = false, bool CONV = false, bool CK = false, bool GA = false>
ssm_status_t launch_seq(const FwdArgs& a, const SeqPlan& pl) {
    using Cfg = ssm::SeqCfg<IO, G, CPL>;
    if (!pl.ok) return SSM_ERR_UNSUPPORTED;
    constexpr int TC = Cfg::kTC;
    constexpr auto sw128 = CU_TENSOR_MAP_SWIZZLE_128B;
    const auto dt = ssm::IoTraits<IO>::kTmaType;
    constexpr int es = ssm::IoTraits<IO>::kBytes;
    CUtensorMap mu, mdl, mz, mbc;
    const uint64_t L = static_cast<uint64_t>(a.L);
    const uint64_t Lr = static_cast<uint64_t>(a.L_rows ? a.L_rows : a.L);  // row length of u / delta / z
    bool ok = make_map_3d(&mbc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.ws + ws_layout(a.batch, a.dim, a.L).bc_off, 32,
                          L, a.batch, 32, TC, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (GA) {  // the kernel reads u / delta / z itself; the maps are placeholders
        mu = mdl = mz = mbc;
    } else {
        ok = ok && make_map_3d(&mu, dt, es, a.u, Lr, a.dim, a.batch, TC, 8, sw128) &&
             make_map_3d(&mdl, dt, es, a.delta, Lr, a.dim, a.batch, TC, 8, sw128);
        if (ok && a.z) ok = make_map_3d(&mz, dt, es, a.z, Lr, a.dim, a.batch, TC, 8, sw128);
        if (!a.z) mz = mu;
    }
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
    p.x = a.x_orig ? a.x_orig : a.u;  // the caller's x (the conv state-out reads its rows)
    p.conv_w = a.conv.w;
    p.conv_b = a.conv.b;
    p.conv_in = a.conv.in;
    p.conv_out = a.conv.out;
    p.u_out = a.conv.u_out;
    p.conv_k = a.conv.k;
    p.y_vec = a.y_vec;
    p.u_rows = a.u;
    p.dl_rows = a.delta;
    p.z_rows = a.z;
    p.ckpt = a.ckpt;
    p.nseg = static_cast<int>((a.L + 7) / 8);
    if (a.L >= (1LL << 31) - 1024) return SSM_ERR_UNSUPPORTED;
    // With a.pdl the kernel may start while the B/C pack before it is still running (programmatic
    // dependent launch): its prologue and first input copies overlap the pack's tail.
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(static_cast<unsigned>(pl.threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(pl.smem);
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    cudaError_t e;
    if constexpr (GA) {
        if (pl.stages == 3)
            e = cudaLaunchKernelEx(&cfg, ssm::scan_fwd_seq_kernel<IO, G, CPL, 3, ZOH, CONV, CK, true>, mu, mdl, mz, mbc, p);
        else
            e = cudaLaunchKernelEx(&cfg, ssm::scan_fwd_seq_kernel<IO, G, CPL, 4, ZOH, CONV, CK, true>, mu, mdl, mz, mbc, p);
    } else {
        switch (pl.stages) {
            case 2: e = cudaLaunchKernelEx(&cfg, ssm::scan_fwd_seq_kernel<IO, G, CPL, 2, ZOH, CONV, CK>, mu, mdl, mz, mbc, p); break;
            case 3: e = cudaLaunchKernelEx(&cfg, ssm::scan_fwd_seq_kernel<IO, G, CPL, 3, ZOH, CONV, CK>, mu, mdl, mz, mbc, p); break;
            default: e = cudaLaunchKernelEx(&cfg, ssm::scan_fwd_seq_kernel<IO, G, CPL, 4, ZOH, CONV, CK>, mu, mdl, mz, mbc, p); break;
        }
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return SSM_ERR_LAUNCH;
    }
    return launch_status();
}

// The zero-order-hold and conv-prologue kernels exist for 4 and 8 lanes per channel, with and
// without checkpoints (CK).
template <typename IO, bool ZOH, bool CONV, bool CK = false>
ssm_status_t launch_flagged_g(const FwdArgs& a, const ssm_fwd_options_t& o) {
    const SeqPlan p4 = plan_seq<IO, 4, 1, ZOH, CONV, CK>(a);
    if constexpr (sizeof(IO) == 2) {
        const SeqPlan p8 = plan_seq<IO, 8, 1, ZOH, CONV, CK>(a);
        const bool use8 = o.lanes_per_channel == 8 ||
                          (o.lanes_per_channel == 0 && predict_seq<IO, 8, 1>(a, p8) < predict_seq<IO, 4, 1>(a, p4));
        if (use8) return launch_seq<IO, 8, 1, ZOH, CONV, CK>(a, p8);
    }
    return launch_seq<IO, 4, 1, ZOH, CONV, CK>(a, p4);
}

// Plain discretisation without conv: variants (lanes per channel G, channels per lane CPL).
// lanes_per_channel selects G explicitly (CPL = 1), or G = 4 with CPL = 2 when given as 42.
template <typename IO>
ssm_status_t launch_seq_plain(const FwdArgs& a, const ssm_fwd_options_t& o) {
    if (a.ckpt) return launch_seq_ckpt<IO>(a, o);  // the checkpoint-storing kernels (fwd_seq_ckpt_*.cu)
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

// Zero-order hold and / or the conv prologue.
template <typename IO>
ssm_status_t launch_seq_flagged(const FwdArgs& a, const ssm_fwd_options_t& o) {
    if (a.ckpt) return launch_seq_ckpt<IO>(a, o);  // the checkpoint-storing kernels (fwd_seq_ckpt_*.cu)
    if (a.zoh && a.conv.k > 0) return launch_flagged_g<IO, true, true>(a, o);
    if (a.zoh) return launch_flagged_g<IO, true, false>(a, o);
    return launch_flagged_g<IO, false, true>(a, o);
}

// Every discretisation / prologue combination with checkpoints for the backward (4 or 8 lanes
// per channel).  Instantiated only in fwd_seq_ckpt_*.cu (extern below), so that the other
// translation units do not compile these kernels.
template <typename IO>
ssm_status_t launch_seq_ckpt(const FwdArgs& a, const ssm_fwd_options_t& o) {
    if (o.lanes_per_channel != 0 && o.lanes_per_channel != 4 && o.lanes_per_channel != 8) return SSM_ERR_UNSUPPORTED;
    if (a.zoh && a.conv.k > 0) return launch_flagged_g<IO, true, true, true>(a, o);
    if (a.zoh) return launch_flagged_g<IO, true, false, true>(a, o);
    if (a.conv.k > 0) return launch_flagged_g<IO, false, true, true>(a, o);
    return launch_flagged_g<IO, false, false, true>(a, o);
}
extern template ssm_status_t launch_seq_ckpt<__nv_bfloat16>(const FwdArgs&, const ssm_fwd_options_t&);
extern template ssm_status_t launch_seq_ckpt<float>(const FwdArgs&, const ssm_fwd_options_t&);

// Rows of u / delta / z (or x) whose byte length is not a multiple of 16: the GA kernels, which
// gather the rows themselves (4 or 8 lanes per channel, one channel per lane), for every
// discretisation / prologue combination without checkpoints.  Instantiated only in
// fwd_seq_gather_*.cu.
template <typename IO, bool ZOH, bool CONV>
ssm_status_t launch_gather_g(const FwdArgs& a, const ssm_fwd_options_t& o) {
    const SeqPlan p4 = plan_seq<IO, 4, 1, ZOH, CONV, false, true>(a);
    if constexpr (sizeof(IO) == 2) {
        const SeqPlan p8 = plan_seq<IO, 8, 1, ZOH, CONV, false, true>(a);
        const bool use8 = o.lanes_per_channel == 8 ||
                          (o.lanes_per_channel == 0 && predict_seq<IO, 8, 1>(a, p8) < predict_seq<IO, 4, 1>(a, p4));
        if (use8) return launch_seq<IO, 8, 1, ZOH, CONV, false, true>(a, p8);
    }
    return launch_seq<IO, 4, 1, ZOH, CONV, false, true>(a, p4);
}
template <typename IO>
ssm_status_t launch_seq_gather(const FwdArgs& a, const ssm_fwd_options_t& o) {
    if (o.lanes_per_channel != 0 && o.lanes_per_channel != 4 && o.lanes_per_channel != 8) return SSM_ERR_UNSUPPORTED;
    if (a.zoh && a.conv.k > 0) return launch_gather_g<IO, true, true>(a, o);
    if (a.zoh) return launch_gather_g<IO, true, false>(a, o);
    if (a.conv.k > 0) return launch_gather_g<IO, false, true>(a, o);
    return launch_gather_g<IO, false, false>(a, o);
}
extern template ssm_status_t launch_seq_gather<__nv_bfloat16>(const FwdArgs&, const ssm_fwd_options_t&);
extern template ssm_status_t launch_seq_gather<float>(const FwdArgs&, const ssm_fwd_options_t&);

}  // namespace ssmh
