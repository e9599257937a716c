// wide.cu -- launchers of the d_state 32 .. 256 forward scan and decode (scan_fwd_wide.cuh).
#include <algorithm>

#include "host_common.h"
#include "scan_fwd_wide.cuh"

namespace ssmh {

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
    auto kern = a.zoh ? ssm::scan_fwd_wide_kernel<IO, N, true> : ssm::scan_fwd_wide_kernel<IO, N, false>;
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
void decode_wide_n(const DecodeArgs& a, unsigned grid) {
    ssm::state_update_wide_kernel<IO, N><<<grid, 256, 0, a.stream>>>(a.A, a.D, a.bias, a.state, a.u, a.delta, a.B,
                                                                     a.C, a.z, a.y, a.batch, a.dim, a.softplus,
                                                                     a.zoh);
}

template <typename IO>
void decode_wide_io(const DecodeArgs& a, unsigned grid) {
    switch (a.dstate) {
        case 32: decode_wide_n<IO, 32>(a, grid); break;
        case 64: decode_wide_n<IO, 64>(a, grid); break;
        case 128: decode_wide_n<IO, 128>(a, grid); break;
        default: decode_wide_n<IO, 256>(a, grid); break;
    }
}

// d_state 32 .. 256 decode: N/4 (at most 32) threads per channel.
ssm_status_t launch_decode_wide(const DecodeArgs& a, ssm_dtype_t io) {
    const int tpc = std::min(a.dstate / 4, 32);  // threads per channel
    const long long threads = static_cast<long long>(a.batch) * a.dim * tpc;
    const long long grid = (threads + 255) / 256;
    if (grid > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (io == SSM_BF16) decode_wide_io<__nv_bfloat16>(a, static_cast<unsigned>(grid));
    else decode_wide_io<float>(a, static_cast<unsigned>(grid));
    return launch_status();
}

template ssm_status_t launch_wide<__nv_bfloat16>(const FwdArgs&, int);
template ssm_status_t launch_wide<float>(const FwdArgs&, int);

}  // namespace ssmh
