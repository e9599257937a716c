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
 * Layouts (all contiguous, row-major): u, delta, z, y: (batch, dim, L);
 * B, C: (batch, dstate, L); A: (dim, dstate); D, delta_bias: (dim);
 * h0 / last_state / decode state: (batch, dim, dstate).
 *
 * Readings taken where the pages are silent (listed with reasons in the design doc):
 *   - D is a per-channel scalar, NULL means 0; z NULL means no gate; delta_bias
 *     NULL means 0.
 *   - softplus is evaluated in the overflow-free form max(x,0) + log1p(exp(-|x|)).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

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
int oracle_selective_scan_f64(const double* u, const double* delta, const double* A,
                              const double* B, const double* C, const double* D,
                              const double* z, const double* delta_bias, int softplus,
                              const double* h0, double* y, double* last_state,
                              int64_t batch, int64_t dim, int64_t dstate, int64_t L)
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
                    const double bbar = dt * B[(b * dstate + n) * L + t];
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
int oracle_state_update_f64(double* state, const double* u, const double* delta,
                            const double* A, const double* B, const double* C,
                            const double* D, const double* z, const double* delta_bias,
                            int softplus, double* y,
                            int64_t batch, int64_t dim, int64_t dstate)
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
                *h = exp(dt * A[d * dstate + n]) * (*h) + dt * B[b * dstate + n] * ut;
                yt += C[b * dstate + n] * (*h);
            }
            yt += (D ? D[d] : 0.0) * ut;
            if (z) yt *= silu_f64(z[row]);
            y[row] = yt;
        }
    }
    return 0;
}

/* Number of OpenMP threads the oracle will use (reported beside CPU timings). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Exposed for the pin that checks softplus/silu against library routines. */
double oracle_softplus_f64(double x) { return softplus_f64(x); }
double oracle_silu_f64(double z) { return silu_f64(z); }
