// host_common.h -- host-side pieces shared by the translation units of the library:
// workspace layouts, the argument bundles handed from the C ABI to the launchers, TMA
// tensor-map helpers, and the launcher of every kernel family (each family is compiled in
// its own .cu file so the library builds in parallel).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ssm_scan.h"
#include "common.cuh"

namespace ssmh {

using ssm::WorkspaceHeader;

constexpr uint32_t kDefaultWaitLimit = 1u << 22;  // mbarrier tries before a wait gives up
constexpr uint32_t kDefaultSpinLimit = 1u << 21;  // look-back polls (~64 ns sleep each)

inline size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Forward workspace layout (d_state 16):
//   [header 256 B][B/C fp32 rows: batch * L * 128 B]
//   [look-back flags: keys * 4 B][aggregate h: keys * 256 B][aggregate sum Delta: keys * 16 B]
//   [inclusive h: keys * 256 B]
// with keys = (8-channel tiles) * 2 columns * ceil(L / 32) chunks (32 steps is the shorter
// chunk of the two element types, so one size serves both).
//   [padded rows: 3 arrays of batch * dim * round_up(L, 8) * 4 B, only when L % 8 != 0]
// The padded rows hold u, delta and z copied to rows whose length is a multiple of 16
// bytes (TMA needs 16-byte row strides); sized for fp32, the larger element type.
struct WsLayout {
    size_t bc_off, flags_off, agg_off, sdt_off, incl_off, pad_off, pad_array, total;
    long long keys;
};
constexpr int kMinChunk = 32;

inline bool rows_need_padding(int64_t L) { return L % 8 != 0; }

inline WsLayout ws_layout(int batch, int dim, int64_t L) {
    WsLayout w{};
    const long long tiles = static_cast<long long>(batch) * ((dim + 7) / 8);
    w.keys = tiles * 2 * ((L + kMinChunk - 1) / kMinChunk);
    w.bc_off = sizeof(WorkspaceHeader);
    w.flags_off = w.bc_off + round_up(static_cast<size_t>(batch) * static_cast<size_t>(L) * 128u, 256);
    w.agg_off = w.flags_off + round_up(static_cast<size_t>(w.keys) * 4u, 256);
    w.sdt_off = w.agg_off + static_cast<size_t>(w.keys) * 256u;
    w.incl_off = w.sdt_off + static_cast<size_t>(w.keys) * 16u;
    w.pad_off = round_up(w.incl_off + static_cast<size_t>(w.keys) * 256u, 256);
    w.pad_array = rows_need_padding(L) ? round_up(static_cast<size_t>(batch) * static_cast<size_t>(dim) *
                                                      static_cast<size_t>(round_up(static_cast<size_t>(L), 8)) * 4u,
                                                  256)
                                       : 0;
    w.total = w.pad_off + 3 * w.pad_array;
    return w;
}

// 3-D tiled tensor map over a dense (d2, d1, d0) tensor with d0 innermost (false if the
// driver entry point is missing or the encoding is rejected).
bool make_map_3d(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* ptr, uint64_t d0, uint64_t d1,
                 uint64_t d2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw);

// Opt a kernel into the largest dynamic shared memory per block the device allows next to
// its static shared memory (once per kernel and device); false if `bytes` does not fit.
bool ensure_smem_attr(const void* kernel, int bytes);

// SSM_OK on an sm_100 device (and its SM count), SSM_ERR_UNSUPPORTED on another
// architecture, SSM_ERR_LAUNCH when no device can be queried (or when the fault-injection
// variable SSM_FAKE_LAUNCH_FAILURE is set).
ssm_status_t check_device(int* sm_count);

inline ssm_status_t launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SSM_OK : SSM_ERR_LAUNCH;
}

// Causal conv1d + SiLU prologue of a forward call (k = 0: none; `u` then holds x).
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
    int64_t L_rows = 0;  // row length of u / delta / z when staged into padded rows (0: L)
    int y_vec = 1;       // y rows 16-byte aligned: vector stores of y
    bool pad_ok = true;  // the workspace has room for padded rows (not the no-allocation scratch)
    bool pdl = false;    // the previous launch is the B/C pack: the scan may start early (it waits
                         // for the pack before reading the B/C rows, and reads nothing else it writes)
    float* ckpt = nullptr;  // checkpoints for the backward (batch, ceil(L/8), dim, 16), or null
    const void* x_orig = nullptr;  // conv prologue on padded rows: the caller's x (rows of L)
};

// Backward workspace layout:
//   [header 256 B][B/C rows: batch * L * 128 B][checkpoints: batch * nseg * dim * 64 B]
//   [dB/dC per CTA: batch * ncta * L * 128 B][dA per batch row: batch * dim * 64 B]
//   [dD per batch row: batch * dim * 4 B][ddelta_bias per batch row: batch * dim * 4 B]
//   [conv weight per batch row: batch * dim * 16 B][conv bias per batch row: batch * dim * 4 B]
struct BwdLayout {
    size_t bc_off, ckpt_off, dbc_off, dA_off, dD_off, dbias_off, dcw_off, dcb_off, total;
    int nseg, ncta;
};
BwdLayout bwd_layout(int batch, int dim, int64_t L);

// Conv prologue of a backward call (k = 0: none; `u` then holds x and `du` receives dx).
struct ConvBwdArgs {
    const float *w = nullptr, *b = nullptr, *in = nullptr, *dout = nullptr;
    float *dw = nullptr, *db = nullptr, *din = nullptr;
    int k = 0;
};

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
    int zoh = 0;
    ConvBwdArgs conv;
    const float* ckpt = nullptr;  // the forward's checkpoints (no forward sweep), or null
};

struct DecodeArgs {
    float* state;
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *bias;
    int softplus;
    void* y;
    int batch, dim, dstate;
    int zoh;
    const float *conv_w, *conv_b;
    float* conv_state;
    int conv_k;
    cudaStream_t stream;
};

// ------------------------------------------------------------------ kernel-family launchers
// B/C (batch, 16, L) -> the fp32 rows of the workspace (aux.cu).
template <typename IO> ssm_status_t launch_pack(const FwdArgs& a);
// Direct-load forward (any seqlen / alignment; aux.cu).
template <typename IO> ssm_status_t launch_direct(const FwdArgs& a);
// narrays (<= 3) arrays of rows x L elements -> rows x Lp elements (zero past L) (aux.cu).
template <typename IO> ssm_status_t launch_pad_rows(const void* const* src, void* const* dst, int narrays, long long rows,
                                                    int64_t L, int64_t Lp, cudaStream_t stream);
// Sequence split across CTAs with decoupled look-back (fwd_chunked.cu).
template <typename IO> ssm_status_t launch_chunked(const FwdArgs& a, const ssm_fwd_options_t& o);
// Sequential family, plain discretisation, no conv: picks lanes per channel (fwd_seq_*.cu).
template <typename IO> ssm_status_t launch_seq_plain(const FwdArgs& a, const ssm_fwd_options_t& o);
// Sequential family with the zero-order hold and / or the conv prologue (fwd_seq_flag_*.cu).
template <typename IO> ssm_status_t launch_seq_flagged(const FwdArgs& a, const ssm_fwd_options_t& o);
// Sequential family storing checkpoints for the backward, every variant (fwd_seq_ckpt_*.cu).
template <typename IO> ssm_status_t launch_seq_ckpt(const FwdArgs& a, const ssm_fwd_options_t& o);
template <typename IO> ssm_status_t launch_seq_gather(const FwdArgs& a, const ssm_fwd_options_t& o);
// d_state 32 .. 256 forward (wide.cu).
template <typename IO> ssm_status_t launch_wide(const FwdArgs& a, int n);
// Backward (bwd.cu).
template <typename IO> ssm_status_t launch_backward(const BwdArgs& a);
// B/C rows of the backward's shared-memory ring (aux.cu).
template <typename IO> ssm_status_t launch_pack_bwd(const BwdArgs& a, uint8_t* bc);
// One-token decode: d_state 16 (aux.cu) and 32 .. 256 (wide.cu).
ssm_status_t launch_decode16(const DecodeArgs& a, ssm_dtype_t io);
ssm_status_t launch_decode_wide(const DecodeArgs& a, ssm_dtype_t io);

}  // namespace ssmh
