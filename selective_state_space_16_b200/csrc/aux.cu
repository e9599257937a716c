// aux.cu -- launchers of the kernels around the main scans (aux_kernels.cuh): the B/C
// transposes, the direct-load forward and the d_state-16 decode step.
#include <algorithm>

#include "host_common.h"
#include "aux_kernels.cuh"

namespace ssmh {

// d_state-16 decode: fp32 state values per thread (4, 8 or 16; 16 / that many threads per channel)
constexpr int kDecodeStatesPerThread = 8;

template <typename IO>
ssm_status_t launch_pack(const FwdArgs& a) {
    const dim3 grid(static_cast<unsigned>((a.L + 63) / 64), static_cast<unsigned>(a.batch));
    ssm::pack_bc_kernel<IO><<<grid, 256, 0, a.stream>>>(
        static_cast<const IO*>(a.B), static_cast<const IO*>(a.C),
        reinterpret_cast<float*>(a.ws + ws_layout(a.batch, a.dim, a.L).bc_off), a.L,
        reinterpret_cast<WorkspaceHeader*>(a.ws));
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
    p.hdr = reinterpret_cast<WorkspaceHeader*>(a.ws);
    constexpr int G = 2;
    const long long threads = static_cast<long long>(a.batch) * a.dim * G;
    const long long grid = (threads + 127) / 128;
    if (grid > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    ssm::scan_fwd_direct_kernel<IO, G><<<static_cast<unsigned>(grid), 128, 0, a.stream>>>(p);
    return launch_status();
}

// B/C rows for the backward's ring: bf16 inputs stay bf16 (ordered by state pairs), fp32 as
// the forward's fp32 rows.
template <typename IO>
ssm_status_t launch_pack_bwd(const BwdArgs& a, uint8_t* bc) {
    const dim3 grid(static_cast<unsigned>((a.L + 63) / 64), static_cast<unsigned>(a.batch));
    if constexpr (sizeof(IO) == 2)
        ssm::pack_bc_pairs_kernel<<<grid, 256, 0, a.stream>>>(static_cast<const uint16_t*>(a.B),
                                                              static_cast<const uint16_t*>(a.C),
                                                              reinterpret_cast<uint32_t*>(bc), a.L);
    else
        ssm::pack_bc_kernel<IO><<<grid, 256, 0, a.stream>>>(static_cast<const IO*>(a.B), static_cast<const IO*>(a.C),
                                                           reinterpret_cast<float*>(bc), a.L,
                                                           reinterpret_cast<WorkspaceHeader*>(a.ws));
    return launch_status();
}

// d_state-16 decode step: 16 / kDecodeStatesPerThread threads per channel, grid.y = batch row.
template <typename IO>
void decode16_io(const DecodeArgs& a, bool bc_vec) {
    const ssm::DecodeParams p{a.state, a.u, a.delta, a.A, a.B, a.C, a.D, a.z, a.bias, a.y, a.batch, a.dim,
                              a.softplus, a.zoh, bc_vec, a.conv_w, a.conv_b, a.conv_state, a.conv_k};
    constexpr int NS = kDecodeStatesPerThread;
    constexpr int TH = ssm::kDecodeThreads;
    const dim3 g(static_cast<unsigned>((static_cast<long long>(a.dim) * (16 / NS) + TH - 1) / TH),
                 static_cast<unsigned>(a.batch));
    const bool conv = a.conv_k > 0;
    if (a.zoh && conv) ssm::state_update_kernel<IO, true, true, NS><<<g, TH, 0, a.stream>>>(p);
    else if (a.zoh) ssm::state_update_kernel<IO, true, false, NS><<<g, TH, 0, a.stream>>>(p);
    else if (conv) ssm::state_update_kernel<IO, false, true, NS><<<g, TH, 0, a.stream>>>(p);
    else ssm::state_update_kernel<IO, false, false, NS><<<g, TH, 0, a.stream>>>(p);
}

ssm_status_t launch_decode16(const DecodeArgs& a, ssm_dtype_t io) {
    const bool bc_vec = aligned16(a.B) && aligned16(a.C);
    if (io == SSM_BF16) decode16_io<__nv_bfloat16>(a, bc_vec);
    else decode16_io<float>(a, bc_vec);
    return launch_status();
}

template <typename IO>
ssm_status_t launch_pad_rows(const void* const* src, void* const* dst, int narrays, long long rows, int64_t L,
                             int64_t Lp, cudaStream_t stream) {
    ssm::PadArrays arr{};
    for (int i = 0; i < narrays; ++i) {
        arr.src[i] = src[i];
        arr.dst[i] = dst[i];
    }
    const long long chunks = rows * (Lp / (16 / static_cast<long long>(sizeof(IO))));
    const long long grid = std::max<long long>(1, std::min<long long>((chunks + 255) / 256, 148LL * 16));
    ssm::pad_rows_kernel<IO><<<dim3(static_cast<unsigned>(grid), static_cast<unsigned>(narrays)), 256, 0, stream>>>(
        arr, rows, L, Lp);
    return launch_status();
}

template ssm_status_t launch_pad_rows<__nv_bfloat16>(const void* const*, void* const*, int, long long, int64_t,
                                                     int64_t, cudaStream_t);
template ssm_status_t launch_pad_rows<float>(const void* const*, void* const*, int, long long, int64_t, int64_t,
                                             cudaStream_t);
template ssm_status_t launch_pack<__nv_bfloat16>(const FwdArgs&);
template ssm_status_t launch_pack<float>(const FwdArgs&);
template ssm_status_t launch_direct<__nv_bfloat16>(const FwdArgs&);
template ssm_status_t launch_direct<float>(const FwdArgs&);
template ssm_status_t launch_pack_bwd<__nv_bfloat16>(const BwdArgs&, uint8_t*);
template ssm_status_t launch_pack_bwd<float>(const BwdArgs&, uint8_t*);

}  // namespace ssmh

