/*
 * ssm_oracle.c -- plain fp64 CPU oracle for the selective state-space scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file: only tests/, the smoke check in __graft_entry__.py and the
 * cpu_baseline / reference leg of bench.py use it.  It shares no code, header,
 * constant or helper with the CUDA library; it is written from the pages alone.
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
 *   [Tech] "Transformer架构遭遇颠覆性突破：Mamba模型如何用状态空间重新定义序列建模效率？"
 *          (tech.kj168168.com/?p=3956)
 *
 * What is computed, for every batch row b and channel d independently:
 *   x      = delta[b,d,t] + delta_bias[d]                     ([Eng] §3.2: bias inside softplus)
 *   Delta  = softplus(x)  (or x when softplus is off)         ([Card] 选择性机制; [Eng] §3.2)
 *   h[n]  <- exp(Delta*A[d,n]) * h[n] + Delta*B[b,n,t]*u[b,d,t]
 *            simplified discretisation Abar = exp(Delta A), Bbar = Delta B
 *                                                              ([Card] 离散化变换 and 选择性机制;
 *                                                               [Tech] 二.1)
 *   y      = sum_n C[b,n,t]*h[n]  (the state AFTER the update, [Card] Python 演示;
 *                                   [S4M] 5.2)
 *            + D[d]*u[b,d,t]                                  ([Eng] §2.2; [Tech] 二.1)
 *   y     *= silu(z[b,d,t]) when z is given                   ([Hist] Mamba Block 数据流)
 * The state starts at zero unless h0 is given ([Eng] §7.2; [Card] Python 演示) and
 * the state after the last step is written to last_state ([Eng] §4.2).
 *
 * The backward (oracle_selective_scan_bwd_f64) is the plain definition of the
 * gradients of L = sum dy*y + sum dlast*last_state: the same forward loop, keeping
 * every state, then the chain rule applied to each step in reverse order (the
 * recompute-in-backward scheme of [Tech] 四.1 and [S4M] 3.3, here with everything
 * kept).  oracle_selective_scan_bwd_zoh_f64 does the same for either discretisation,
 * and oracle_causal_conv_silu_bwd_f64 is the chain rule through the conv prologue
 * (u = silu(conv(x))), given the gradient reaching u.  All three are pinned by finite
 * differences of the forward functions.
 *
 * Layouts (all contiguous, row-major): u, delta, z, y: (batch, dim, L);
 * B, C: (batch, dstate, L); A: (dim, dstate); D, delta_bias: (dim);
 * h0 / last_state / decode state: (batch, dim, dstate).
 *
 * Readings taken where the pages are silent:
 *   - D is a per-channel scalar, NULL means 0; z NULL means no gate; delta_bias
 *     NULL means 0.
 *   - softplus is evaluated in the overflow-free form max(x,0) + log1p(exp(-|x|)).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* softplus(x) = log(1 + e^x), written so that neither branch overflows. */
static double softplus_f64(double x)
{
    return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x));
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^{-z})  ([Hist] Mamba Block: SiLU gate). */
static double silu_f64(double z)
{
    return z / (1.0 + exp(-z));
}

/*
 * Input weight of one chain for one step.  Simplified discretisation: Bbar = Delta*B
 * ([Card] 离散化变换).  Zero-order hold ([Eng] §2.2): Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B
 * = expm1(Delta A) / A * B for a diagonal A, whose limit as A -> 0 is Delta*B.  (The page prints
 * the ZOH weight without the Delta in front of B; the reading here is the one that reduces to
 * Delta*B for small Delta*A, as the simplified form on the other pages does.)
 */
static double input_weight(double dt, double a, double b, int zoh)
{
    if (!zoh) return dt * b;
    const double x = dt * a;
    return x == 0.0 ? dt * b : expm1(x) / a * b;
}

/* Step size for one (b, d, t): Delta = softplus(delta + bias) ([Eng] §3.2). */
static double step_size(double delta_raw, const double* delta_bias, int64_t d, int softplus)
{
    double x = delta_raw + (delta_bias ? delta_bias[d] : 0.0);
    return softplus ? softplus_f64(x) : x;
}

/*
 * Full-sequence forward scan.  A plain sequential loop over t and n for every
 * (b, d), as in the sequential scans of [S4M] 5.2 and [Card] Python 演示.
 * Returns 0 on success, -1 on a bad argument.
 */
int oracle_selective_scan_zoh_f64(const double* u, const double* delta, const double* A,
                                  const double* B, const double* C, const double* D,
                                  const double* z, const double* delta_bias, int softplus,
                                  const double* h0, double* y, double* last_state,
                                  int64_t batch, int64_t dim, int64_t dstate, int64_t L, int zoh);

int oracle_selective_scan_f64(const double* u, const double* delta, const double* A,
                              const double* B, const double* C, const double* D,
                              const double* z, const double* delta_bias, int softplus,
                              const double* h0, double* y, double* last_state,
                              int64_t batch, int64_t dim, int64_t dstate, int64_t L)
{
    return oracle_selective_scan_zoh_f64(u, delta, A, B, C, D, z, delta_bias, softplus, h0, y, last_state,
                                         batch, dim, dstate, L, 0);
}

/* As oracle_selective_scan_f64, with the zero-order-hold input weight when zoh != 0. */
int oracle_selective_scan_zoh_f64(const double* u, const double* delta, const double* A,
                                  const double* B, const double* C, const double* D,
                                  const double* z, const double* delta_bias, int softplus,
                                  const double* h0, double* y, double* last_state,
                                  int64_t batch, int64_t dim, int64_t dstate, int64_t L, int zoh)
{
    if (batch < 0 || dim < 0 || dstate < 1 || dstate > 256 || L < 0) return -1;
    if (!u || !delta || !A || !B || !C || !y) return -1;

    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            double h[256];
            const int64_t row = (b * dim + d);
            for (int64_t n = 0; n < dstate; ++n)
                h[n] = h0 ? h0[row * dstate + n] : 0.0;

            for (int64_t t = 0; t < L; ++t) {
                const double ut = u[row * L + t];
                const double dt = step_size(delta[row * L + t], delta_bias, d, softplus);
                double yt = 0.0;
                for (int64_t n = 0; n < dstate; ++n) {
                    const double abar = exp(dt * A[d * dstate + n]);
                    const double bbar = input_weight(dt, A[d * dstate + n], B[(b * dstate + n) * L + t], zoh);
                    h[n] = abar * h[n] + bbar * ut;
                    yt += C[(b * dstate + n) * L + t] * h[n];
                }
                yt += (D ? D[d] : 0.0) * ut;
                if (z) yt *= silu_f64(z[row * L + t]);
                y[row * L + t] = yt;
            }
            if (last_state)
                for (int64_t n = 0; n < dstate; ++n) last_state[row * dstate + n] = h[n];
        }
    }
    return 0;
}

/*
 * One-token decode: the same step body for a single t, reading the state and
 * writing it back ([Card] 线性扫描算法: O(1) per generated token; [Eng] §6.2).
 * state: (batch, dim, dstate) in/out; u, delta, z, y: (batch, dim);
 * B, C: (batch, dstate).
 */
int oracle_state_update_zoh_f64(double* state, const double* u, const double* delta,
                                const double* A, const double* B, const double* C,
                                const double* D, const double* z, const double* delta_bias,
                                int softplus, double* y,
                                int64_t batch, int64_t dim, int64_t dstate, int zoh);

int oracle_state_update_f64(double* state, const double* u, const double* delta,
                            const double* A, const double* B, const double* C,
                            const double* D, const double* z, const double* delta_bias,
                            int softplus, double* y,
                            int64_t batch, int64_t dim, int64_t dstate)
{
    return oracle_state_update_zoh_f64(state, u, delta, A, B, C, D, z, delta_bias, softplus, y, batch, dim,
                                       dstate, 0);
}

/* As oracle_state_update_f64, with the zero-order-hold input weight when zoh != 0. */
int oracle_state_update_zoh_f64(double* state, const double* u, const double* delta,
                                const double* A, const double* B, const double* C,
                                const double* D, const double* z, const double* delta_bias,
                                int softplus, double* y,
                                int64_t batch, int64_t dim, int64_t dstate, int zoh)
{
    if (batch < 0 || dim < 0 || dstate < 1 || dstate > 256) return -1;
    if (!state || !u || !delta || !A || !B || !C || !y) return -1;

    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            const double ut = u[row];
            const double dt = step_size(delta[row], delta_bias, d, softplus);
            double yt = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                double* h = &state[row * dstate + n];
                *h = exp(dt * A[d * dstate + n]) * (*h) +
                     input_weight(dt, A[d * dstate + n], B[b * dstate + n], zoh) * ut;
                yt += C[b * dstate + n] * (*h);
            }
            yt += (D ? D[d] : 0.0) * ut;
            if (z) yt *= silu_f64(z[row]);
            y[row] = yt;
        }
    }
    return 0;
}

/* d silu / dz = sigmoid(z) * (1 + z * (1 - sigmoid(z))). */
static double silu_grad_f64(double z)
{
    const double s = 1.0 / (1.0 + exp(-z));
    return s * (1.0 + z * (1.0 - s));
}

/* d softplus / dx = sigmoid(x). */
static double sigmoid_f64(double x)
{
    return x >= 0.0 ? 1.0 / (1.0 + exp(-x)) : exp(x) / (1.0 + exp(x));
}

/*
 * Derivatives of the input weight per unit B, phi(dt, a) = dt (simplified) or expm1(dt a) / a
 * (zero-order hold, [Eng] §2.2; dt at a = 0):
 *   d phi / d dt = 1 (simplified);  exp(dt a) (ZOH: the derivative of expm1 is exp).
 *   d phi / d a  = 0 (simplified);  (dt a exp(dt a) - expm1(dt a)) / a^2 (ZOH).
 * The ZOH form in a loses digits to cancellation when x = dt a is small, so there it takes the
 * Taylor series of the same function, dt^2 (1/2 + x/3 + x^2/8 + x^3/30 + ...): the k-th term
 * of (x e^x - (e^x - 1)) / x^2 is x^k / (k! (k + 2)), summed to x^3 (the next term,
 * x^4/144, is below 1e-14 relative for |x| < 1e-3).
 */
static double input_weight_ddt(double dt, double a, int zoh)
{
    return zoh ? exp(dt * a) : 1.0;
}

static double input_weight_dA(double dt, double a, int zoh)
{
    if (!zoh) return 0.0;
    const double x = dt * a;
    if (fabs(x) < 1e-3) return dt * dt * (0.5 + x * (1.0 / 3.0 + x * (1.0 / 8.0 + x * (1.0 / 30.0))));
    return (x * exp(x) - expm1(x)) / (a * a);
}

/*
 * Backward of one channel (b, d): the forward loop again, keeping every state, then
 * the chain rule applied to it step by step in reverse order.  Per-channel outputs are
 * written; the sums over channels (dB, dC) and over batch rows (dA, dD, ddelta_bias)
 * are added into the caller's accumulators.
 *   H: (L+1) x dstate scratch (H[0] = initial state, H[t+1] = state after step t);
 *   Dt: L scratch (step sizes).
 */
static void channel_bwd(int64_t b, int64_t d, const double* u, const double* delta, const double* A,
                        const double* B, const double* C, const double* D, const double* z,
                        const double* delta_bias, int softplus, const double* h0, const double* dy,
                        const double* dlast, double* du, double* ddelta, double* dz, double* dh0,
                        double* accB, double* accC, double* accA, double* accD, double* accBias,
                        int64_t dim, int64_t N, int64_t L, double* H, double* Dt, int zoh)
{
    const int64_t row = b * dim + d;
    const double Dd = D ? D[d] : 0.0;
    for (int64_t n = 0; n < N; ++n) H[n] = h0 ? h0[row * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {  /* forward, as oracle_selective_scan_f64 */
        const double ut = u[row * L + t];
        Dt[t] = step_size(delta[row * L + t], delta_bias, d, softplus);
        for (int64_t n = 0; n < N; ++n)
            H[(t + 1) * N + n] = exp(Dt[t] * A[d * N + n]) * H[t * N + n] +
                                 input_weight(Dt[t], A[d * N + n], B[(b * N + n) * L + t], zoh) * ut;
    }
    /* g[n] = dL/dh: the gradient reaching the state, starting from dL/d last_state. */
    double g[256];
    for (int64_t n = 0; n < N; ++n) g[n] = dlast ? dlast[row * N + n] : 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
        const double ut = u[row * L + t], dt = Dt[t];
        /* y = v * silu(z), v = sum_n C h_t + D u */
        double v = Dd * ut;
        for (int64_t n = 0; n < N; ++n) v += C[(b * N + n) * L + t] * H[(t + 1) * N + n];
        double dv = dy[row * L + t];
        if (z) {
            const double zt = z[row * L + t];
            dz[row * L + t] = dy[row * L + t] * v * silu_grad_f64(zt);
            dv *= silu_f64(zt);
        }
        accD[d] += dv * ut;
        double dut = Dd * dv, ddt = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double Bn = B[(b * N + n) * L + t], Cn = C[(b * N + n) * L + t], An = A[d * N + n];
            const double hprev = H[t * N + n], abar = exp(dt * An);
            /* h_t = abar * h_{t-1} + phi * B * u, phi the input weight per unit B */
            const double phi = input_weight(dt, An, 1.0, zoh);
            accC[n * L + t] += dv * H[(t + 1) * N + n];
            g[n] += dv * Cn;                          /* dL/dh_t complete */
            ddt += g[n] * (An * abar * hprev + input_weight_ddt(dt, An, zoh) * Bn * ut);
            accB[n * L + t] += g[n] * phi * ut;
            dut += g[n] * phi * Bn;
            accA[d * N + n] += g[n] * (dt * abar * hprev + input_weight_dA(dt, An, zoh) * Bn * ut);
            g[n] *= abar;                             /* dL/dh_{t-1} through this step */
        }
        du[row * L + t] = dut;
        const double x = delta[row * L + t] + (delta_bias ? delta_bias[d] : 0.0);
        const double dx = softplus ? ddt * sigmoid_f64(x) : ddt;
        ddelta[row * L + t] = dx;
        accBias[d] += dx;
    }
    if (dh0)
        for (int64_t n = 0; n < N; ++n) dh0[row * N + n] = g[n];
}

/*
 * Gradients of the forward scan (reverse-mode differentiation of oracle_selective_scan_f64):
 * given dy = dL/dy (batch, dim, L) and optionally dlast = dL/d last_state (batch, dim, N),
 * writes dL/d of every input: du, ddelta, dz (batch, dim, L; dz only when z is given),
 * dA (dim, N), dB, dC (batch, N, L), dD and ddelta_bias (dim; always written, as if D and
 * delta_bias were present), dh0 (batch, dim, N; optional).  The sums over channels and
 * batch rows are formed per thread and added in thread order, so a run is reproducible
 * for a given thread count.  Returns 0, or -1 on a bad argument or allocation failure.
 */
int oracle_selective_scan_bwd_zoh_f64(const double* u, const double* delta, const double* A,
                                      const double* B, const double* C, const double* D,
                                      const double* z, const double* delta_bias, int softplus,
                                      const double* h0, const double* dy, const double* dlast,
                                      double* du, double* ddelta, double* dA, double* dB, double* dC,
                                      double* dD, double* dz, double* ddelta_bias, double* dh0,
                                      int64_t batch, int64_t dim, int64_t dstate, int64_t L, int zoh);

int oracle_selective_scan_bwd_f64(const double* u, const double* delta, const double* A,
                                  const double* B, const double* C, const double* D,
                                  const double* z, const double* delta_bias, int softplus,
                                  const double* h0, const double* dy, const double* dlast,
                                  double* du, double* ddelta, double* dA, double* dB, double* dC,
                                  double* dD, double* dz, double* ddelta_bias, double* dh0,
                                  int64_t batch, int64_t dim, int64_t dstate, int64_t L)
{
    return oracle_selective_scan_bwd_zoh_f64(u, delta, A, B, C, D, z, delta_bias, softplus, h0, dy, dlast, du,
                                             ddelta, dA, dB, dC, dD, dz, ddelta_bias, dh0, batch, dim, dstate, L, 0);
}

/* As oracle_selective_scan_bwd_f64, for the zero-order-hold input weight when zoh != 0
 * (the gradients of oracle_selective_scan_zoh_f64). */
int oracle_selective_scan_bwd_zoh_f64(const double* u, const double* delta, const double* A,
                                      const double* B, const double* C, const double* D,
                                      const double* z, const double* delta_bias, int softplus,
                                      const double* h0, const double* dy, const double* dlast,
                                      double* du, double* ddelta, double* dA, double* dB, double* dC,
                                      double* dD, double* dz, double* ddelta_bias, double* dh0,
                                      int64_t batch, int64_t dim, int64_t dstate, int64_t L, int zoh)
{
    if (batch < 0 || dim < 0 || dstate < 1 || dstate > 256 || L < 0) return -1;
    if (!u || !delta || !A || !B || !C || !dy || !du || !ddelta || !dA || !dB || !dC || !dD ||
        !ddelta_bias || (z && !dz))
        return -1;
    const int64_t N = dstate;
    int nth = 1;
#ifdef _OPENMP
    nth = omp_get_max_threads();
#endif
    if (nth > dim && dim > 0) nth = (int)dim;
    if (nth < 1) nth = 1;
    const size_t nl = (size_t)N * (size_t)L, dn = (size_t)dim * (size_t)N;
    double* accB = calloc((size_t)nth * nl + 1, sizeof(double));
    double* accC = calloc((size_t)nth * nl + 1, sizeof(double));
    double* accA = calloc((size_t)nth * dn + 1, sizeof(double));
    double* accD = calloc((size_t)nth * (size_t)dim + 1, sizeof(double));
    double* accBias = calloc((size_t)nth * (size_t)dim + 1, sizeof(double));
    int fail = !accB || !accC || !accA || !accD || !accBias;
    for (int64_t b = 0; b < batch && !fail; ++b) {
        memset(accB, 0, (size_t)nth * nl * sizeof(double));
        memset(accC, 0, (size_t)nth * nl * sizeof(double));
        #pragma omp parallel num_threads(nth)
        {
            int tid = 0;
#ifdef _OPENMP
            tid = omp_get_thread_num();
#endif
            double* H = malloc(((size_t)L + 1) * (size_t)N * sizeof(double));
            double* Dt = malloc(((size_t)L + 1) * sizeof(double));
            if (!H || !Dt) {
                #pragma omp atomic write
                fail = 1;
            }
            #pragma omp for schedule(static)
            for (int64_t d = 0; d < dim; ++d)
                if (H && Dt)
                    channel_bwd(b, d, u, delta, A, B, C, D, z, delta_bias, softplus, h0, dy, dlast, du, ddelta,
                                dz, dh0, accB + tid * nl, accC + tid * nl, accA + tid * dn, accD + tid * dim,
                                accBias + tid * dim, dim, N, L, H, Dt, zoh);
            free(H);
            free(Dt);
        }
        for (size_t i = 0; i < nl; ++i) {
            double sb = 0.0, sc = 0.0;
            for (int k = 0; k < nth; ++k) {
                sb += accB[k * nl + i];
                sc += accC[k * nl + i];
            }
            dB[(size_t)b * nl + i] = sb;
            dC[(size_t)b * nl + i] = sc;
        }
    }
    for (size_t i = 0; i < dn && !fail; ++i) {
        double s = 0.0;
        for (int k = 0; k < nth; ++k) s += accA[k * dn + i];
        dA[i] = s;
    }
    for (int64_t d = 0; d < dim && !fail; ++d) {
        double sd = 0.0, sb = 0.0;
        for (int k = 0; k < nth; ++k) {
            sd += accD[k * dim + d];
            sb += accBias[k * dim + d];
        }
        dD[d] = sd;
        ddelta_bias[d] = sb;
    }
    free(accB);
    free(accC);
    free(accA);
    free(accD);
    free(accBias);
    return fail ? -1 : 0;
}

/*
 * Causal depthwise convolution of width K along t, then SiLU: the local-feature step before
 * the scan in the Mamba block ([Hist] Mamba Block 数据流: x -> 1D conv -> SiLU -> S6;
 * [Card] Mamba架构设计):
 *   u[b,d,t] = silu( bias[d] + sum_{k=0}^{K-1} w[d,k] * x[b,d,t-(K-1)+k] )
 * where inputs before t = 0 are x_prev[b,d,0..K-2] (oldest first) when given, else zero.
 * x: (batch, dim, L); w: (dim, K); bias: (dim) or NULL; x_prev: (batch, dim, K-1) or NULL;
 * u: (batch, dim, L) output.  When x_next is given it receives the last K-1 inputs seen
 * (the state that continues the convolution).  Returns 0, or -1 on a bad argument.
 */
int oracle_causal_conv_silu_f64(const double* x, const double* w, const double* bias, const double* x_prev,
                                double* u, double* x_next, int64_t batch, int64_t dim, int64_t L, int64_t K)
{
    if (batch < 0 || dim < 0 || L < 0 || K < 1 || K > 16 || !x || !w || !u) return -1;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            for (int64_t t = 0; t < L; ++t) {
                double acc = bias ? bias[d] : 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    const int64_t s = t - (K - 1) + k;  /* input index, may be negative */
                    double xv = 0.0;
                    if (s >= 0) xv = x[row * L + s];
                    else if (x_prev) xv = x_prev[row * (K - 1) + (K - 1 + s)];
                    acc += w[d * K + k] * xv;
                }
                u[row * L + t] = silu_f64(acc);
            }
            if (x_next)
                for (int64_t j = 0; j < K - 1; ++j) {
                    const int64_t s = L - (K - 1) + j;
                    x_next[row * (K - 1) + j] =
                        s >= 0 ? x[row * L + s] : (x_prev ? x_prev[row * (K - 1) + (K - 1 + s)] : 0.0);
                }
        }
    }
    return 0;
}

/*
 * Backward of oracle_causal_conv_silu_f64: given du = dL/du (batch, dim, L) and optionally
 * dx_next = dL/d x_next (batch, dim, K-1), the gradients of the conv's inputs.  With
 * p[t] = bias + sum_k w[k] xin[t-(K-1)+k] (xin: x_prev before t = 0, then x) and u = silu(p):
 *   dp[t]      = du[t] * silu'(p[t])
 *   dxin[s]   += w[k] * dp[t]          for every (t, k) with s = t-(K-1)+k
 *   dxin[s]   += dx_next[j]            for s = L-(K-1)+j (x_next copies those inputs)
 *   dw[d,k]   += dp[t] * xin[t-(K-1)+k]  (summed over batch rows and t)
 *   dbias[d]  += dp[t]                  (summed over batch rows and t)
 * dx (batch, dim, L) receives dxin[0..L), dx_prev (batch, dim, K-1; optional) dxin[-(K-1)..0).
 * dw (dim, K) and dbias (dim; optional) are written, not accumulated.  The sums over batch
 * rows are formed per channel in batch order.  Returns 0, or -1 on a bad argument.
 */
int oracle_causal_conv_silu_bwd_f64(const double* x, const double* w, const double* bias, const double* x_prev,
                                    const double* du, const double* dx_next, double* dx, double* dw,
                                    double* dbias, double* dx_prev, int64_t batch, int64_t dim, int64_t L,
                                    int64_t K)
{
    if (batch < 0 || dim < 0 || L < 0 || K < 1 || K > 16 || !x || !w || !du || !dx || !dw) return -1;
    int fail = 0;
    #pragma omp parallel for schedule(static)
    for (int64_t d = 0; d < dim; ++d) {
        double gw[16] = {0.0}, gb = 0.0;
        double* dxin = malloc(((size_t)L + (size_t)K) * sizeof(double));  /* index s + (K-1) */
        if (!dxin) {
            #pragma omp atomic write
            fail = 1;
        }
        for (int64_t b = 0; b < batch && dxin; ++b) {
            const int64_t row = b * dim + d;
            for (int64_t i = 0; i < L + K - 1; ++i) dxin[i] = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                double p = bias ? bias[d] : 0.0;
                double xin[16];
                for (int64_t k = 0; k < K; ++k) {
                    const int64_t s = t - (K - 1) + k;
                    xin[k] = s >= 0 ? x[row * L + s] : (x_prev ? x_prev[row * (K - 1) + (K - 1 + s)] : 0.0);
                    p += w[d * K + k] * xin[k];
                }
                const double dp = du[row * L + t] * silu_grad_f64(p);
                gb += dp;
                for (int64_t k = 0; k < K; ++k) {
                    gw[k] += dp * xin[k];
                    dxin[t + k] += w[d * K + k] * dp;       /* s + (K-1) = t + k */
                }
            }
            if (dx_next)
                for (int64_t j = 0; j < K - 1; ++j) dxin[L + j] += dx_next[row * (K - 1) + j];
            for (int64_t s = 0; s < L; ++s) dx[row * L + s] = dxin[s + K - 1];
            if (dx_prev)
                for (int64_t j = 0; j < K - 1; ++j) dx_prev[row * (K - 1) + j] = dxin[j];
        }
        for (int64_t k = 0; k < K; ++k) dw[d * K + k] = gw[k];
        if (dbias) dbias[d] = gb;
        free(dxin);
    }
    return fail ? -1 : 0;
}

/* Number of OpenMP threads the oracle will use (reported beside CPU timings). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Exposed for the pin that checks softplus/silu against library routines. */
double oracle_softplus_f64(double x) { return softplus_f64(x); }
double oracle_silu_f64(double z) { return silu_f64(z); }
