// fwd_chunked.cu -- launcher of the chunked forward kernel (sequence split across CTAs,
// joined by decoupled look-back; scan_fwd_chunked.cuh).
#include <algorithm>

#include "host_common.h"
#include "scan_fwd_chunked.cuh"

namespace ssmh {

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

template ssm_status_t launch_chunked<__nv_bfloat16>(const FwdArgs&, const ssm_fwd_options_t&);
template ssm_status_t launch_chunked<float>(const FwdArgs&, const ssm_fwd_options_t&);

}  // namespace ssmh
