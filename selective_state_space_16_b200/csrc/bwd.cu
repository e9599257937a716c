// bwd.cu -- launcher of the backward scan (scan_bwd.cuh) and its two reduction kernels.
#include "host_common.h"
#include "scan_bwd.cuh"

namespace ssmh {

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
    w.dcw_off = w.dbias_off + round_up(B * D * 4u, 256);
    w.dcb_off = w.dcw_off + round_up(B * D * 16u, 256);
    w.total = w.dcb_off + round_up(B * D * 4u, 256);
    return w;
}

namespace {
template <typename IO>
using BwdKernel = void (*)(const ssm::BwdParams);

template <typename IO>
BwdKernel<IO> bwd_kernel(bool zoh, bool conv) {
    if (conv) return zoh ? ssm::scan_bwd_kernel<IO, true, true> : ssm::scan_bwd_kernel<IO, false, true>;
    return zoh ? ssm::scan_bwd_kernel<IO, true, false> : ssm::scan_bwd_kernel<IO, false, false>;
}
}  // namespace

template <typename IO>
ssm_status_t launch_backward(const BwdArgs& a) {
    const BwdLayout wl = bwd_layout(a.batch, a.dim, a.L);
    uint8_t* bc = a.ws + wl.bc_off;
    {
        const ssm_status_t st = launch_pack_bwd<IO>(a, bc);
        if (st != SSM_OK) return st;
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
    p.ckpt = a.ckpt ? const_cast<float*>(a.ckpt) : reinterpret_cast<float*>(a.ws + wl.ckpt_off);
    p.ckpt_given = a.ckpt != nullptr;
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
    p.hdr = reinterpret_cast<WorkspaceHeader*>(a.ws);
    p.conv_w = a.conv.w;
    p.conv_b = a.conv.b;
    p.conv_in = a.conv.in;
    p.dconv_out = a.conv.dout;
    p.dconv_in = a.conv.din;
    p.dcw_part = reinterpret_cast<float*>(a.ws + wl.dcw_off);
    p.dcb_part = reinterpret_cast<float*>(a.ws + wl.dcb_off);
    p.conv_k = a.conv.k;
    constexpr int smem = ssm::kBwdSmem;
    auto kern = bwd_kernel<IO>(a.zoh != 0, a.conv.k > 0);
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
    f.dcw_part = p.dcw_part;
    f.dcb_part = p.dcb_part;
    f.dconv_w = a.conv.dw;
    f.dconv_b = a.conv.db;
    f.conv_k = a.conv.k;
    f.batch = a.batch;
    f.dim = a.dim;
    f.ncta = wl.ncta;
    f.L = a.L;
    ssm::scan_bwd_reduce_bc_kernel<<<dim3(static_cast<unsigned>((a.L + 7) / 8), static_cast<unsigned>(a.batch)), 256,
                                     0, a.stream>>>(f);
    const long long n = static_cast<long long>(a.dim) * 16;
    ssm::scan_bwd_reduce_params_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, a.stream>>>(f);
    return launch_status();
}

template ssm_status_t launch_backward<__nv_bfloat16>(const BwdArgs&);
template ssm_status_t launch_backward<float>(const BwdArgs&);

}  // namespace ssmh
