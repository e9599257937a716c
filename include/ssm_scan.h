/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective state-space scan (S6) library.
 *
 * Sources (web pages on Mamba / selective state-space models; sections as printed):
 *   [Eng]  "Mamba 选择性状态空间模型：亚二次复杂度大语言模型推理工程实践"
 *          (www.ybb.press/ai-agent/15212.html)
 *   [Hist] "AI底层架构的一场革命：Mamba如何用「状态压缩」挑战Transformer的十年统治"
 *          (gitcode.csdn.net/6a278c3f662f9a54cb7b917b.html)
 *   [Card] "Mamba与SSM状态空间模型：一张摘要卡读完万页档案"
 *          (aiqz.cc/article/mamba-ssm-state-space-model.html)
 *   [S4M]  "State Space Models 深度实战：从 S4 到 Mamba 的架构演进与 CUDA 优化"
 *          (www.ybb.press/ai-applications/10137.html)
 *
 * The operation, for every batch row b and channel d (independent of each other):
 *   Delta_t = softplus(delta[b,d,t] + delta_bias[d])          [Eng] §3.2, [Card] 选择性机制
 *   h_t[n]  = exp(Delta_t*A[d,n]) * h_{t-1}[n] + Delta_t*B[b,n,t]*u[b,d,t]
 *             (simplified discretisation Abar = exp(Delta A), Bbar = Delta B,
 *              [Card] 离散化变换 and 选择性机制)
 *   y_t     = (sum_n C[b,n,t]*h_t[n] + D[d]*u[b,d,t]) * silu(z[b,d,t])
 *             ([Eng] §2.2 for C h + D x; [Hist] Mamba Block 数据流 for the SiLU gate)
 *   h_{-1}  = 0 (or a given initial state, ssm_selective_scan_fwd_state);
 *   last_state = h_{L-1}                                         [Eng] §4.2 and §7.2
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory and frees nothing.
 *   - Layouts are dense row-major:  u, delta, z, y: (batch, dim, seqlen);
 *     B, C: (batch, dstate, seqlen);  A: (dim, dstate) fp32;  D, delta_bias: (dim) fp32;
 *     last_state / decode state: (batch, dim, dstate) fp32.
 *   - io_dtype gives the element type of u, delta, z, B, C and y (fp32 or bf16).
 *     A, D, delta_bias and the state are always fp32; arithmetic is fp32.
 *   - Calls are asynchronous on `stream`; errors found before the launch are
 *     returned; errors found on the device (a look-back wait that ran out) are
 *     recorded in the workspace status word and read back by ssm_read_status().
 *   - dstate: the forward scan and decode take 16 (the tuned kernels) or 32, 64, 128, 256 (one
 *     warp per channel; bound by the exponential unit, N per element).  The backward, the
 *     chunked kernel and the no-allocation entry point take 16 only.  Other values return
 *     SSM_ERR_UNSUPPORTED.
 *   - Inputs are never modified, except `state` in ssm_state_update().
 *   - A pointer to a tensor with zero elements (e.g. u when seqlen == 0) may be NULL.
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-identical to cudaStream_t (both are `struct CUstream_st *`); NULL = legacy stream. */
typedef struct CUstream_st* ssm_stream_t;

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad dtype, misaligned pointer    */
    SSM_ERR_UNSUPPORTED = 2,   /* dstate not supported by the call, or the device is not sm_100 */
    SSM_ERR_LAUNCH = 3,        /* a CUDA call or kernel launch failed                           */
    SSM_ERR_TIMEOUT = 4,       /* device: a bounded wait in the kernel gave up (see read_status) */
    SSM_ERR_WORKSPACE = 5,     /* workspace missing or smaller than ssm_selective_scan_workspace_size */
    SSM_ERR_SCRATCH_LIMIT = 6, /* the problem needs more than the fixed scratch of ssm_selective_scan_fwd_noalloc */
    SSM_ERR_BOUNDS = 7         /* device, debug library only: an index range check failed (see below) */
} ssm_status_t;

/*
 * Debug library.  libssm_scan_debug.so is the same library compiled with -DSSM_DEBUG_CHECKS:
 * the kernels range-check their shared-memory offsets, TMA coordinates and global indices,
 * and a failed check records SSM_ERR_BOUNDS in the workspace status word (read back with
 * ssm_read_status) and skips the access instead of touching memory.  It stands in for a
 * memory checker; the release library compiles every check away.
 *
 * Fault injection.  With the environment variable SSM_FAKE_LAUNCH_FAILURE set (to any value),
 * every call that would launch a kernel returns SSM_ERR_LAUNCH before launching anything, as
 * if the launch had failed; it lets callers test their error handling without a GPU fault.
 */

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype_t;

/* Version of this ABI (incremented on any signature change). */
int ssm_abi_version(void);

/* Human-readable name of a status code (static string). */
const char* ssm_status_string(ssm_status_t status);

/*
 * Bytes of device workspace ssm_selective_scan_fwd needs for these sizes (a multiple
 * of 256).  The workspace holds a transposed fp32 copy of B and C, the status word
 * and (dstate 16) the flags and (prod Abar, h) pairs of the inter-CTA chunk carry.
 * Returns 0 for invalid sizes.
 */
size_t ssm_selective_scan_workspace_size(int batch, int dim, int dstate, int64_t seqlen);

/*
 * Zero a workspace before its first use.  After that every call leaves the
 * workspace ready for the next one (its counters and flag epochs are reset by the
 * kernel itself), so this is needed once per allocation.
 */
ssm_status_t ssm_workspace_init(void* workspace, size_t workspace_bytes, ssm_stream_t stream);

/*
 * Full-sequence forward scan (the operation above).
 *   u, delta, B, C, y       required; io_dtype elements.
 *   A                        required; fp32 (dim, dstate).
 *   D, delta_bias            optional fp32 (dim); NULL means 0.
 *   z                        optional io_dtype (batch, dim, seqlen); NULL means no gate.
 *   softplus                 nonzero: Delta = softplus(delta + bias); zero: Delta = delta + bias.
 *   last_state               optional fp32 (batch, dim, dstate) output: the state after step seqlen-1
 *                            (zeros when seqlen == 0).
 *   workspace                device buffer of at least
 *                            ssm_selective_scan_workspace_size(batch, dim, dstate, seqlen) bytes,
 *                            256-byte aligned, zeroed once by ssm_workspace_init().  It must not be
 *                            used by two calls that can overlap on the GPU.
 * All tensor pointers must be 16-byte aligned.  Any seqlen >= 0 is accepted; when
 * seqlen * sizeof(io element) is a multiple of 16 the tiles are staged with TMA straight
 * from u, delta and z (x with the conv prologue).  Otherwise TMA cannot address the rows:
 * the sequential kernel's warps then copy their rows' 16-byte-aligned windows themselves
 * and shift them into place (SSM_ALGO_SEQUENTIAL, the no-allocation entry point, and
 * SSM_ALGO_AUTO on shapes with about 8 or more 8-channel tiles per SM), or u, delta and z
 * are first copied into rows padded to a multiple of 16 bytes inside the workspace (which
 * is sized for this whenever seqlen % 8 != 0: SSM_ALGO_AUTO on smaller shapes, with
 * checkpoints, or with lanes_per_channel 2 or 42); SSM_ALGO_CHUNKED and SSM_ALGO_DIRECT run
 * a direct-load kernel.
 */
ssm_status_t ssm_selective_scan_fwd(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    void* y, float* last_state,
    int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
    void* workspace, size_t workspace_bytes, ssm_stream_t stream);

/* Kernel family for ssm_selective_scan_fwd_ex. */
typedef enum {
    SSM_ALGO_AUTO = 0,        /* pick by shape (what ssm_selective_scan_fwd does)              */
    SSM_ALGO_SEQUENTIAL = 1,  /* each CTA walks all of L for its channels; carry in registers  */
    SSM_ALGO_CHUNKED = 2,     /* L split into chunks across CTAs, joined by decoupled look-back */
    SSM_ALGO_DIRECT = 3       /* no staging: direct global loads (any alignment of seqlen)     */
} ssm_algo_t;

/*
 * Discretisation of the continuous system ([Eng] §2.2).  SIMPLIFIED (the default): Abar = exp(Delta A),
 * Bbar = Delta B ([Card] 离散化变换).  ZOH: the zero-order hold, Bbar = (Delta A)^-1 (exp(Delta A) - 1)
 * Delta B = expm1(Delta A)/A * B for the diagonal A (Delta B when A = 0).  ZOH is supported by the
 * sequential and direct forward kernels, by decode and by ssm_selective_scan_bwd_ex;
 * SSM_ALGO_CHUNKED returns SSM_ERR_UNSUPPORTED for it.
 */
typedef enum { SSM_DISC_SIMPLIFIED = 0, SSM_DISC_ZOH = 1 } ssm_discretization_t;

/* Options of the forward entry points.  Zero-initialise the whole struct: zero means the
 * default for every field (changed in ABI version 2: the discretization field was added; in
 * version 3: the checkpoints field). */
typedef struct {
    int algo;                  /* ssm_algo_t                                                      */
    int lanes_per_channel;     /* SEQUENTIAL: lanes sharing one channel: 2, 4 or 8 (8: bf16 only), or 42 =
                                  4 lanes per channel with each lane holding two channels; 0 = auto    */
    uint32_t spin_limit;       /* CHUNKED: polls before a look-back wait gives up; 0 = default    */
    int debug_skip_publish;    /* CHUNKED, tests only: chunk index whose CTAs never publish; -1 = off */
    int discretization;        /* ssm_discretization_t; 0 = SSM_DISC_SIMPLIFIED                   */
    float* checkpoints;        /* NULL, or fp32 (batch, ceil(seqlen/8), dim, dstate) output: the state
                                  at the start of every 8-step segment (h before step 8s; segment 0:
                                  the initial state), for ssm_selective_scan_bwd_ex, which then skips
                                  its own forward sweep ([Tech] 四.1: keep a little in the forward
                                  pass).  16-byte aligned.  Written by the sequential kernel only
                                  (4 or 8 lanes per channel): d_state 16; SSM_ALGO_AUTO then runs
                                  the sequential kernel, and SSM_ALGO_CHUNKED / SSM_ALGO_DIRECT (or
                                  a direct-load fallback) and lanes_per_channel 2 or 42 return
                                  SSM_ERR_UNSUPPORTED.                                            */
} ssm_fwd_options_t;

/* ssm_selective_scan_fwd with an explicit kernel choice (tuning and tests).  opts may be NULL. */
ssm_status_t ssm_selective_scan_fwd_ex(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    void* y, float* last_state,
    int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
    void* workspace, size_t workspace_bytes, const ssm_fwd_options_t* opts, ssm_stream_t stream);

/*
 * Forward scan from a given state instead of zero: state continuation across the
 * blocks of an over-long sequence ([Eng] §7.2: block-wise processing must carry the
 * state from one block into the next) and reuse of a cached prefix state ([Eng] §6.2).
 * The recurrence above then starts from h_{-1} = initial_state, so that scanning
 * steps [0, L1) and then [L1, L) with initial_state = the first call's last_state
 * gives the scan of [0, L) (up to the fp32 state handed over).
 *   initial_state  optional fp32 (batch, dim, dstate); NULL means zero, and the call is
 *                  then ssm_selective_scan_fwd_ex.  Read only.  It must not overlap
 *                  last_state (SSM_ERR_INVALID_ARG): with the sequence split across CTAs,
 *                  a channel's initial state can still be read after another CTA has
 *                  written that channel's final state.  Use two buffers to chain calls.
 *   seqlen == 0    last_state receives a copy of initial_state (zeros if it is NULL).
 *   opts           as for ssm_selective_scan_fwd_ex; may be NULL.
 * Every other argument, the workspace rules and the errors are those of
 * ssm_selective_scan_fwd.
 */
ssm_status_t ssm_selective_scan_fwd_state(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    const float* initial_state, void* y, float* last_state,
    int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
    void* workspace, size_t workspace_bytes, const ssm_fwd_options_t* opts, ssm_stream_t stream);

/*
 * Causal depthwise conv1d + SiLU in front of the scan: the local-feature step of the Mamba
 * block's x branch ([Hist] Mamba Block 数据流: x -> 1D conv -> SiLU -> S6; [Card] Mamba架构设计),
 *   u[b,d,t] = silu( bias[d] + sum_{k<width} weight[d,k] * x[b,d,t-width+1+k] ),
 * with the inputs before t = 0 taken from state_in (zeros if NULL).
 */
typedef struct {
    const float* weight;    /* (dim, width) fp32, oldest tap first; required                       */
    const float* bias;      /* (dim) fp32, or NULL (0)                                              */
    int width;              /* 1 .. 4                                                               */
    const float* state_in;  /* (batch, dim, width-1) fp32 inputs before t = 0, oldest first, or NULL */
    float* state_out;       /* (batch, dim, width-1) fp32: the last width-1 inputs, or NULL; it may
                               be the same buffer as state_in (each channel reads its state before
                               writing it)                                                          */
    void* u_out;            /* io_dtype (batch, dim, seqlen): u as fed to the scan, or NULL         */
} ssm_conv_t;

/*
 * Forward scan of u = silu(conv(x)) computed on the fly from x (io_dtype, (batch, dim,
 * seqlen), in place of u): the staged x tile is converted in shared memory, so u never makes
 * a round trip through HBM unless u_out asks for it.  u is rounded to io_dtype before the
 * scan (as a separate conv kernel storing u would).  Every other argument as
 * ssm_selective_scan_fwd_state.  d_state 16 only; SSM_ALGO_CHUNKED returns SSM_ERR_UNSUPPORTED.
 */
ssm_status_t ssm_selective_scan_fwd_conv(
    const void* x, const ssm_conv_t* conv, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    const float* initial_state, void* y, float* last_state,
    int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
    void* workspace, size_t workspace_bytes, const ssm_fwd_options_t* opts, ssm_stream_t stream);

/*
 * Backward of the forward scan: the gradients of a loss L with respect to every input,
 * given dy = dL/dy and optionally dlast_state = dL/d last_state.  The forward is
 * recomputed rather than stored ([Tech] 四.1: keep little in the forward pass and
 * rebuild in the backward pass; [S4M] 3.3: forward and backward with the state kept on
 * chip).  With g the gradient reaching h_t and v_t = sum_n C h_t + D u_t:
 *   dz = dy v silu'(z);  dv = dy silu(z);  g += dv C_t;  dC_t += dv h_t;
 *   dDelta_t = sum_n g (A a_t h_{t-1} + B_t u_t);  dB_t += g Delta_t u_t;
 *   du_t = sum_n g Delta_t B_t + D dv;  dA += g Delta_t a_t h_{t-1};  g <- a_t g;
 *   ddelta_t = dDelta_t sigmoid(delta_t + bias) (dDelta_t without softplus);
 *   dD = sum dv u;  ddelta_bias = sum ddelta;  d initial_state = g after step 0.
 * Inputs: as ssm_selective_scan_fwd_state (same values; initial_state may be NULL),
 *   dy                io_dtype (batch, dim, seqlen), required.
 *   dlast_state       optional fp32 (batch, dim, dstate); NULL means 0.
 * Outputs (written, not accumulated; none may overlap another argument):
 *   du, ddelta        io_dtype (batch, dim, seqlen), required.
 *   dz                io_dtype (batch, dim, seqlen); required when z is given, else ignored.
 *   dA                fp32 (dim, dstate), summed over batch rows and steps; required.
 *   dB, dC            fp32 (batch, dstate, seqlen), summed over channels; required.
 *   dD, ddelta_bias   optional fp32 (dim), summed over batch rows and steps (computed
 *                     as if D / delta_bias were given, also when they are NULL).
 *   dinitial_state    optional fp32 (batch, dim, dstate).
 * Every sum is formed in a fixed order: repeated calls give identical results.
 *   workspace         device buffer of at least ssm_selective_scan_bwd_workspace_size()
 *                     bytes, 256-byte aligned; no initialisation needed; must not be used
 *                     by two calls that can overlap on the GPU.
 * Errors as ssm_selective_scan_fwd.  Any seqlen >= 0 and any 16-byte aligned pointers.
 */
size_t ssm_selective_scan_bwd_workspace_size(int batch, int dim, int dstate, int64_t seqlen);

ssm_status_t ssm_selective_scan_bwd(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    const float* initial_state, const void* dy, const float* dlast_state,
    void* du, void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
    float* ddelta_bias, float* dinitial_state,
    int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
    void* workspace, size_t workspace_bytes, ssm_stream_t stream);

/* Options of ssm_selective_scan_bwd_ex.  Zero-initialise the whole struct: all zero (or opts
 * NULL) is ssm_selective_scan_bwd. */
typedef struct {
    int discretization;            /* ssm_discretization_t of the forward; 0 = SSM_DISC_SIMPLIFIED        */
    const ssm_conv_t* conv;        /* the forward's conv prologue, or NULL.  weight, bias, width and
                                      state_in are read; state_out and u_out are ignored.                */
    float* dconv_weight;           /* (dim, width) fp32 output; required with conv                       */
    float* dconv_bias;             /* (dim) fp32 output, or NULL                                          */
    float* dconv_state_in;         /* (batch, dim, width-1) fp32 output: gradient of conv->state_in, or NULL */
    const float* dconv_state_out;  /* (batch, dim, width-1) fp32: gradient reaching conv->state_out (the
                                      carried-out inputs), or NULL (zero)                                 */
    const float* checkpoints;      /* NULL, or the checkpoints a forward call with the same inputs (and
                                      initial state) stored (ssm_fwd_options_t.checkpoints): the
                                      backward then reads them instead of recomputing them          */
} ssm_bwd_options_t;

/*
 * Backward of the zero-order-hold scan and / or of ssm_selective_scan_fwd_conv.  Arguments,
 * workspace (ssm_selective_scan_bwd_workspace_size) and errors as ssm_selective_scan_bwd, and:
 *   discretization = SSM_DISC_ZOH: the gradients of the ZOH scan, where the input weight is
 *     phi B with phi = expm1(Delta A) / A ([Eng] §2.2): dB_t += g phi u_t,
 *     du_t = sum_n g phi B_t + D dv_t, dDelta_t = sum_n g a_t (A h_{t-1} + B_t u_t),
 *     dA += g (Delta_t a_t h_{t-1} + dphi/dA B_t u_t), dphi/dA = (Delta a_t - phi) / A
 *     (its Taylor series where |Delta A| < 1/16).
 *   conv != NULL: `u` is the conv input x (io_dtype (batch, dim, seqlen)) and `du` receives dx.
 *     u = silu(p), p_t = bias + sum_k weight[k] x_{t-width+1+k}, is recomputed from x (rounded to
 *     io_dtype as the forward rounds it) and never stored; with du_t the gradient reaching u
 *     (taken through the rounding unchanged) and dp_t = du_t silu'(p_t):
 *       dx_s = sum_k weight[k] dp_{s+width-1-k} (+ dconv_state_out for the last width-1 inputs),
 *       dconv_weight[d,k] = sum over batch rows and t of dp_t x_{t-width+1+k},
 *       dconv_bias[d] = sum dp_t,  dconv_state_in = dx_s for s = -(width-1) .. -1.
 *     d_state 16.  The conv arrays need no alignment beyond their element type.
 * seqlen == 0: dconv_weight and dconv_bias are zero and dconv_state_in is dconv_state_out.
 */
ssm_status_t ssm_selective_scan_bwd_ex(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    const float* initial_state, const void* dy, const float* dlast_state,
    void* du, void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
    float* ddelta_bias, float* dinitial_state,
    int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype,
    void* workspace, size_t workspace_bytes, const ssm_bwd_options_t* opts, ssm_stream_t stream);

/*
 * One-token decode ([Card] 线性扫描算法: a fixed-size state update per token;
 * [Eng] §6.2).  For every (b, d):  h[n] <- exp(Delta*A[d,n]) h[n] + Delta*B[b,n]*u[b,d],
 * y[b,d] = (sum_n C[b,n] h[n] + D[d] u[b,d]) * silu(z[b,d]), with the fp32 state
 * read, modified and written IN PLACE.
 *   state       fp32 (batch, dim, dstate), in/out; state and A 16-byte aligned.
 *   u, delta, z, y: io_dtype (batch, dim);  B, C: io_dtype (batch, dstate), any alignment
 *   (read as 16-byte vectors when both are 16-byte aligned).
 *   D, delta_bias, z optional as above.  No workspace.
 *   d_state 16: batch <= 65535, else SSM_ERR_UNSUPPORTED.
 */
ssm_status_t ssm_state_update(
    float* state, const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus, void* y,
    int batch, int dim, int dstate, ssm_dtype_t io_dtype, ssm_stream_t stream);

/*
 * One decode step with the conv prologue: u = silu(conv_bias + sum_k conv_weight[d,k] *
 * [conv_state, x]_k) (rounded to io_dtype), then the step of ssm_state_update_ex with u;
 * conv_state (batch, dim, conv_width-1) fp32, oldest first, is shifted in place to end with x.
 * conv_width 0 means no conv (x is u).  d_state 16 with a conv.
 */
ssm_status_t ssm_state_update_conv(
    float* state, float* conv_state, const void* x, const float* conv_weight, const float* conv_bias,
    int conv_width, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus, void* y,
    int batch, int dim, int dstate, ssm_dtype_t io_dtype, ssm_discretization_t discretization,
    ssm_stream_t stream);

/* ssm_state_update with an explicit discretisation (ssm_discretization_t). */
ssm_status_t ssm_state_update_ex(
    float* state, const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus, void* y,
    int batch, int dim, int dstate, ssm_dtype_t io_dtype, ssm_discretization_t discretization,
    ssm_stream_t stream);

/*
 * Forward scan that allocates nothing and takes no workspace.  The pages have no
 * counterpart: this entry point exists for callers that are handed only their input
 * and output buffers -- for example a plugin inside a host framework that owns all
 * device memory and offers no allocator, or a latency-critical loop that cannot
 * afford cudaMalloc, which may synchronise the whole device.  The caller still
 * passes every input and output tensor, with the same meaning, layout and alignment
 * rules as ssm_selective_scan_fwd.
 *
 * Its scratch (a 256-byte header plus the transposed fp32 copy of B and C, i.e.
 * 256 + batch * seqlen * 128 bytes rounded up to 256) lives in one fixed array of
 * SSM_NOALLOC_SCRATCH_BYTES (8 MiB) in the library's device memory: every GPU that
 * loads the library holds that array until the process exits.  Problems that need
 * more return SSM_ERR_SCRATCH_LIMIT before anything is launched.
 *   - The first call on each device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture begins.  The address is kept for the life of the process: after a
 *     cudaDeviceReset (or any reset of the device's primary context) this entry point
 *     must not be called again on that device.
 *   - All calls share the one array: calls whose kernels can overlap on the GPU
 *     (different streams, or different host threads) race on it.  Order them on one
 *     stream or synchronise between them.
 *   - Each call clears the header itself; the B/C region is fully rewritten before
 *     it is read, so nothing left by an earlier call is used.
 * Device-side timeouts are not reported (there is no workspace to read them from).
 */
#define SSM_NOALLOC_SCRATCH_BYTES (8u << 20)
ssm_status_t ssm_selective_scan_fwd_noalloc(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int softplus,
    void* y, float* last_state,
    int batch, int dim, int dstate, int64_t seqlen, ssm_dtype_t io_dtype, ssm_stream_t stream);

/*
 * Synchronise `stream`, return the device-side status recorded in `workspace` by the
 * calls made since the last read (SSM_OK or SSM_ERR_TIMEOUT) and clear it.
 */
ssm_status_t ssm_read_status(void* workspace, ssm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
