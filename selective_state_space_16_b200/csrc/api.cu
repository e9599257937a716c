// api.cu -- host side of the C ABI declared in include/ssm_scan.h: argument
// validation, kernel choice and dispatch to the launcher of each kernel family
// (host_common.h).  Everything here is marshalling; every step of the scan runs in the
// kernels.
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ssm_scan.h"
#include "host_common.h"

using namespace ssmh;

namespace {

constexpr int kAbiVersion = 3;

// d_state values of the forward scan and decode: 16 (the tuned kernels) and the wider states
// of scan_fwd_wide.cuh.
bool dstate_supported(int n) { return n == 16 || n == 32 || n == 64 || n == 128 || n == 256; }

// Chunk length of the chunked kernel (one 128-byte row of the I/O type).
template <typename IO>
constexpr int chunk_steps() { return 128 / static_cast<int>(sizeof(IO)); }

// Rows of u / delta / z (or x, with the conv prologue) whose byte length is not a multiple of
// 16, which TMA cannot address, staged the second of two ways (the first: the GA kernels gather
// them themselves, see launch_forward): copied into padded rows in the workspace, which the
// sequential kernel then stages with TMA; y (and u_out) go straight to the caller's rows with
// element stores.
template <typename IO>
ssm_status_t launch_forward_padded(const FwdArgs& a, const ssm_fwd_options_t& o) {
    constexpr int64_t E = 16 / static_cast<int64_t>(sizeof(IO));
    const WsLayout wl = ws_layout(a.batch, a.dim, a.L);
    FwdArgs pa = a;
    pa.L_rows = (a.L + E - 1) / E * E;
    pa.y_vec = 0;
    pa.x_orig = a.u;  // with the conv prologue u holds x
    const long long rows = static_cast<long long>(a.batch) * a.dim;
    pa.u = a.ws + wl.pad_off;
    pa.delta = a.ws + wl.pad_off + wl.pad_array;
    if (a.z) pa.z = a.ws + wl.pad_off + 2 * wl.pad_array;
    const void* src[3] = {a.u, a.delta, a.z};
    void* const dst[3] = {const_cast<void*>(pa.u), const_cast<void*>(pa.delta), const_cast<void*>(pa.z)};
    const ssm_status_t st = launch_pad_rows<IO>(src, dst, a.z ? 3 : 2, rows, a.L, pa.L_rows, a.stream);
    if (st != SSM_OK) return st;
    return (a.zoh || a.conv.k > 0) ? launch_seq_flagged<IO>(pa, o) : launch_seq_plain<IO>(pa, o);
}

template <typename IO>
ssm_status_t launch_forward(const FwdArgs& a, const ssm_fwd_options_t& o) {
    ssm_status_t st = launch_pack<IO>(a);
    if (st != SSM_OK) return st;
    const bool tma_ok = (static_cast<uint64_t>(a.L) * sizeof(IO)) % 16 == 0 && aligned16(a.u) &&
                        aligned16(a.delta) && aligned16(a.y) && (!a.z || aligned16(a.z));
    int algo = o.algo;
    if (!tma_ok && (algo == SSM_ALGO_AUTO || algo == SSM_ALGO_SEQUENTIAL)) {
        // Unaligned rows: the sequential kernel either gathers them itself (GA kernels) or
        // stages a padded copy.  Gathering costs the consumer warps ~20% (shared-memory traffic)
        // but saves the copy; measured on B200 it wins when the shape gives every SM about 8 or
        // more 8-channel tiles (b4 d5120 L2047: 0.376 against 0.429 ms) and loses with fewer
        // (b1 d5120 L32767, 4.3 tiles per SM: 2.98 against 2.47 ms).  SEQUENTIAL, and callers
        // without room for padded rows, always gather; checkpoints and 2 lanes per channel or
        // two channels per lane (not built as GA kernels) come from the padded copy.
        const double tiles_per_sm = static_cast<double>(a.batch) * ((a.dim + 7) / 8) / a.sm_count;
        const bool ga_variant = o.lanes_per_channel != 2 && o.lanes_per_channel != 42;
        const bool gather =
            !a.ckpt && ga_variant && (algo == SSM_ALGO_SEQUENTIAL || !a.pad_ok || tiles_per_sm >= 8.0);
        if (!gather) {
            if (!a.pad_ok) return SSM_ERR_UNSUPPORTED;
            return launch_forward_padded<IO>(a, o);
        }
        FwdArgs g = a;
        g.y_vec = 0;
        g.pdl = true;  // launched right after the B/C pack
        const ssm_status_t sg = launch_seq_gather<IO>(g, o);
        if (sg != SSM_ERR_UNSUPPORTED) return sg;
        // no gathering plan fits (shared memory): the padded copy, or without room for it the
        // direct kernel
        return a.pad_ok ? launch_forward_padded<IO>(a, o) : launch_direct<IO>(a);
    }
    if (!tma_ok) algo = SSM_ALGO_DIRECT;
    if (a.ckpt && algo == SSM_ALGO_DIRECT) return SSM_ERR_UNSUPPORTED;  // checkpoints: sequential kernel only
    if (a.ckpt && algo == SSM_ALGO_AUTO) algo = SSM_ALGO_SEQUENTIAL;
    if (algo == SSM_ALGO_DIRECT) return launch_direct<IO>(a);
    if ((a.zoh || a.conv.k > 0) && algo == SSM_ALGO_CHUNKED) return SSM_ERR_UNSUPPORTED;  // plain scan only
    if (algo == SSM_ALGO_AUTO && (a.zoh || a.conv.k > 0)) algo = SSM_ALGO_SEQUENTIAL;
    if (algo == SSM_ALGO_AUTO) {
        // The sequential kernel is faster whenever the channels alone give each SM a few
        // warps (measured on B200: at 5120 channels x 32768 steps it runs at ~1.8x the
        // chunked kernel).  Split the sequence across CTAs only when fewer than 4 warps of
        // 8-lane channels per SM would be resident, and the sequence is long.
        const double warps_per_sm = static_cast<double>(a.batch) * a.dim * 8.0 / 32.0 / a.sm_count;
        const long long chunks = (a.L + chunk_steps<IO>() - 1) / chunk_steps<IO>();
        algo = (warps_per_sm < 4.0 && chunks >= 64) ? SSM_ALGO_CHUNKED : SSM_ALGO_SEQUENTIAL;
    }
    if (algo == SSM_ALGO_CHUNKED) return launch_chunked<IO>(a, o);
    FwdArgs b = a;
    b.pdl = true;  // launched right after the B/C pack
    if (a.zoh || a.conv.k > 0) return launch_seq_flagged<IO>(b, o);
    return launch_seq_plain<IO>(b, o);
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
        case SSM_ERR_BOUNDS: return "device index out of range (debug library check)";
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
    ssm_fwd_options_t o{SSM_ALGO_AUTO, 0, 0, -1, SSM_DISC_SIMPLIFIED, nullptr};
    if (opts) o = *opts;
    if (o.algo < SSM_ALGO_AUTO || o.algo > SSM_ALGO_DIRECT) return SSM_ERR_INVALID_ARG;
    if (o.checkpoints && !aligned16(o.checkpoints)) return SSM_ERR_INVALID_ARG;
    // checkpoints come from the sequential kernel only
    if (o.checkpoints && (o.algo == SSM_ALGO_CHUNKED || o.algo == SSM_ALGO_DIRECT)) return SSM_ERR_UNSUPPORTED;
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
    a.ckpt = o.checkpoints;
    if (dstate != 16) {
        if (o.algo == SSM_ALGO_CHUNKED || conv.k > 0 || o.checkpoints) return SSM_ERR_UNSUPPORTED;  // d_state 16 only
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
    const DecodeArgs da{state, u, delta, B, C, z, A, D, delta_bias, softplus, y, batch, dim, dstate,
                        discretization == SSM_DISC_ZOH, conv_weight, conv_bias, conv_state, conv_width,
                        reinterpret_cast<cudaStream_t>(stream)};
    return dstate == 16 ? launch_decode16(da, io_dtype) : launch_decode_wide(da, io_dtype);
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
    a.pad_ok = false;  // the fixed scratch has no room for padded rows: unaligned rows are gathered
    return io_dtype == SSM_BF16 ? launch_forward<__nv_bfloat16>(a, o) : launch_forward<float>(a, o);
}

size_t ssm_selective_scan_bwd_workspace_size(int batch, int dim, int dstate, int64_t seqlen) {
    if (batch < 0 || dim < 0 || dstate != 16 || seqlen < 0) return 0;
    return round_up(bwd_layout(batch, dim, seqlen).total, 256);
}

ssm_status_t ssm_selective_scan_bwd_ex(const void* u, const void* delta, const float* A, const void* B,
                                       const void* C, const float* D, const void* z, const float* delta_bias,
                                       int softplus, const float* initial_state, const void* dy,
                                       const float* dlast_state, void* du, void* ddelta, float* dA, float* dB,
                                       float* dC, float* dD, void* dz, float* ddelta_bias, float* dinitial_state,
                                       int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
                                       void* workspace, size_t workspace_bytes, const ssm_bwd_options_t* opts,
                                       ssm_stream_t stream) {
    if (batch < 0 || dim < 0 || seqlen < 0) return SSM_ERR_INVALID_ARG;
    ssm_bwd_options_t o{};
    if (opts) o = *opts;
    if (o.discretization != SSM_DISC_SIMPLIFIED && o.discretization != SSM_DISC_ZOH) return SSM_ERR_INVALID_ARG;
    if (o.checkpoints && !aligned16(o.checkpoints)) return SSM_ERR_INVALID_ARG;
    ConvBwdArgs conv;
    if (o.conv) {
        if (o.conv->width < 1 || o.conv->width > 4) return SSM_ERR_INVALID_ARG;
        if (dim > 0 && (!o.conv->weight || !o.dconv_weight)) return SSM_ERR_INVALID_ARG;
        conv.k = o.conv->width;
        conv.w = o.conv->weight;
        conv.b = o.conv->bias;
        conv.in = conv.k > 1 ? o.conv->state_in : nullptr;
        conv.dout = conv.k > 1 ? o.dconv_state_out : nullptr;
        conv.dw = o.dconv_weight;
        conv.db = o.dconv_bias;
        conv.din = conv.k > 1 ? o.dconv_state_in : nullptr;
    }
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
    if (seqlen == 0) {  // no steps: only the state (and the conv's carried inputs) pass through
        const size_t state_bytes = static_cast<size_t>(batch) * dim * 16 * sizeof(float);
        cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(dim) * 16 * sizeof(float), s);
        if (e == cudaSuccess && dD) e = cudaMemsetAsync(dD, 0, static_cast<size_t>(dim) * sizeof(float), s);
        if (e == cudaSuccess && ddelta_bias)
            e = cudaMemsetAsync(ddelta_bias, 0, static_cast<size_t>(dim) * sizeof(float), s);
        if (e == cudaSuccess && dinitial_state)
            e = dlast_state ? cudaMemcpyAsync(dinitial_state, dlast_state, state_bytes, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(dinitial_state, 0, state_bytes, s);
        if (conv.k > 0) {
            const size_t cs_bytes = static_cast<size_t>(batch) * dim * (conv.k - 1) * sizeof(float);
            if (e == cudaSuccess) e = cudaMemsetAsync(conv.dw, 0, static_cast<size_t>(dim) * conv.k * sizeof(float), s);
            if (e == cudaSuccess && conv.db) e = cudaMemsetAsync(conv.db, 0, static_cast<size_t>(dim) * sizeof(float), s);
            if (e == cudaSuccess && conv.din && cs_bytes > 0)
                e = conv.dout ? cudaMemcpyAsync(conv.din, conv.dout, cs_bytes, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(conv.din, 0, cs_bytes, s);
        }
        return e == cudaSuccess ? SSM_OK : SSM_ERR_LAUNCH;
    }
    BwdArgs a{u, delta, B, C, z, dy, A, D, delta_bias, initial_state, dlast_state, softplus, du, ddelta, dz, dA, dB,
              dC, dD, ddelta_bias, dinitial_state, batch, dim, seqlen, static_cast<uint8_t*>(workspace), s,
              o.discretization == SSM_DISC_ZOH, conv, o.checkpoints};
    return io_dtype == SSM_BF16 ? launch_backward<__nv_bfloat16>(a) : launch_backward<float>(a);
}

ssm_status_t ssm_selective_scan_bwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                                    const float* D, const void* z, const float* delta_bias, int softplus,
                                    const float* initial_state, const void* dy, const float* dlast_state, void* du,
                                    void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
                                    float* ddelta_bias, float* dinitial_state, int batch, int dim, int dstate,
                                    int64_t seqlen, ssm_dtype_t io_dtype, void* workspace, size_t workspace_bytes,
                                    ssm_stream_t stream) {
    return ssm_selective_scan_bwd_ex(u, delta, A, B, C, D, z, delta_bias, softplus, initial_state, dy, dlast_state,
                                     du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dinitial_state, batch, dim, dstate,
                                     seqlen, io_dtype, workspace, workspace_bytes, nullptr, stream);
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
