/*
 * fp64 CPU oracle for the Mamba-1 selective scan and its one-token state update.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * What it computes (plain definition, no blocking, no reordering):
 *
 *   for every row (b, d), with h[n] = 0 at the start (or a given h0):
 *     for t = 0 .. L-1:
 *       delta = delta_raw[b,d,t] + bias[d]               (bias optional)
 *       delta = softplus(delta) = log(1 + exp(delta))    (if softplus_flag)
 *       for n:  h[n] = exp(delta * A[d,n]) * h[n] + Bbar[n] * u[b,d,t]
 *               Bbar[n] = delta * B[b,n,t]                         (Euler, the default)
 *               Bbar[n] = (exp(delta * A[d,n]) - 1) / A[d,n] * B[b,n,t]   (zero-order hold;
 *                         delta * B[b,n,t] where A[d,n] = 0, the limit)
 *       y = sum_n C[b,n,t] * h[n] + D[d] * u[b,d,t]      (D optional)
 *       y = y * z / (1 + exp(-z))   with z = z[b,d,t]    (gate optional)
 *       out[b,d,t] = y
 *     last_state[b,d,:] = h
 *
 * Sources (web pages, by title and section):
 *  - "Linear Attention vs Softmax Attention: Can RWKV or Mamba Replace
 *    Transformers?", section Implementation, the forward pass of the listed
 *    SelectiveSSMLayer: the step size is softplus of a projection that carries a
 *    bias; A = -exp(A_log); the sequential discretisation loop (A_bar = exp(dt*A),
 *    B_bar = dt*B, h = A_bar*h + B_bar*x, y = h.C + D*x) starts from a zero state;
 *    its output is multiplied by silu of the gate branch.
 *  - "State Space Models in Large Language Models: How Mamba, S4, and Selective
 *    Recurrence Challenge Transformer Attention", section "Mamba: Selective State
 *    Spaces and Hardware-Aware Scans", Dynamic Parameterization: the step is
 *    Softplus(Parameter + Linear(x)), read here as softplus(delta_raw + bias).
 *  - same page, section Discretization, Recurrent View: one recurrence step is
 *    exactly the decode update (oracle_state_update_f64 below).
 *
 *  - "Linear Attention vs Softmax Attention ...", section Core Concepts, item 3,
 *    and "State Space Models in Large Language Models ...", section
 *    Discretization: the zero-order-hold input matrix
 *    (delta A)^-1 (exp(delta A) - I) delta B, which for a diagonal A is
 *    (exp(delta A_n) - 1) / A_n * B_n per state (zoh_flag).
 *
 * Readings where the pages leave a choice open:
 *  - B_bar = delta*B (the page's code) by default; the zero-order-hold form
 *    printed in the pages' equations is the zoh_flag option.
 *  - softplus is the exact log(1 + exp(x)) with no threshold (the listing calls
 *    F.softplus with defaults; the threshold-20 shortcut differs by < 2.1e-9).
 *  - bias absent means 0; D absent means no skip; z absent means no gate.
 *
 * Parity pins (tests/test_oracle_pins.py) tie this file to closed forms and
 * brute force: A = 0 prefix sums, the LTI convolution identity, the fully
 * unrolled sum on tiny inputs, the delta -> 0 and delta -> inf limits,
 * decode-chaining == scan, split-scan == scan, linearity in u, spot values
 * of softplus and silu, and a hand-derived worked example.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact softplus in double: log(1 + exp(x)), evaluated without overflow. */
static double sp_exact(double x)
{
    if (x > 0.0)
        return x + log1p(exp(-x));
    return log1p(exp(x));
}

/* Zero-order-hold input gain (exp(dt * a) - 1) / a, with expm1 so that small
 * dt * a loses nothing to cancellation; its limit dt where a = 0. */
static double zoh_gain(double dt, double a)
{
    if (a == 0.0)
        return dt;
    return expm1(dt * a) / a;
}

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z)). */
static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Selective scan over a batch of rows.  All arrays are dense, C order:
 *   u, delta, z, out : [Bt, D, L]
 *   B, C             : [Bt, N, L]
 *   A                : [D, N]
 *   Dskip, bias      : [D]
 *   h0, last_state   : [Bt, D, N]
 * Nullable: Dskip, z, bias, h0, last_state.  zoh_flag selects the zero-order-hold
 * input gain instead of delta.
 */
void oracle_scan_f64(int64_t Bt, int64_t D, int64_t L, int64_t N,
                     const double *u, const double *delta, const double *A,
                     const double *B, const double *C, const double *Dskip,
                     const double *z, const double *bias, int softplus_flag,
                     int zoh_flag, const double *h0, double *out, double *last_state)
{
    int64_t rows = Bt * D;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t b = r / D, d = r % D;
        double h[64];
        for (int64_t n = 0; n < N; ++n)
            h[n] = h0 ? h0[r * N + n] : 0.0;
        const double *ur = u + r * L;
        const double *dr = delta + r * L;
        const double *zr = z ? z + r * L : NULL;
        const double *Bb = B + b * N * L;
        const double *Cb = C + b * N * L;
        const double *Ad = A + d * N;
        double *yr = out + r * L;
        for (int64_t t = 0; t < L; ++t) {
            double dt = dr[t] + (bias ? bias[d] : 0.0);
            if (softplus_flag)
                dt = sp_exact(dt);
            double x = ur[t];
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double a_bar = exp(dt * Ad[n]);
                double b_bar = dt * Bb[n * L + t];
                if (zoh_flag)
                    b_bar = zoh_gain(dt, Ad[n]) * Bb[n * L + t];
                h[n] = a_bar * h[n] + b_bar * x;
                y += Cb[n * L + t] * h[n];
            }
            if (Dskip)
                y += Dskip[d] * x;
            if (zr)
                y *= silu(zr[t]);
            yr[t] = y;
        }
        if (last_state)
            for (int64_t n = 0; n < N; ++n)
                last_state[r * N + n] = h[n];
    }
}

/*
 * One decode step (the recurrence applied to a single token), state updated in place.
 *   state : [Bt, D, N]      x, dt, z, out : [Bt, D]
 *   A     : [D, N]          B, C          : [Bt, N]
 *   Dskip, bias : [D]       Nullable: Dskip, z, bias.
 */
void oracle_state_update_f64(int64_t Bt, int64_t D, int64_t N, double *state,
                             const double *x, const double *dt_in, const double *A,
                             const double *B, const double *C, const double *Dskip,
                             const double *z, const double *bias, int softplus_flag,
                             int zoh_flag, double *out)
{
    int64_t rows = Bt * D;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t b = r / D, d = r % D;
        double dt = dt_in[r] + (bias ? bias[d] : 0.0);
        if (softplus_flag)
            dt = sp_exact(dt);
        double xv = x[r];
        double *h = state + r * N;
        double y = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double gain = zoh_flag ? zoh_gain(dt, A[d * N + n]) : dt;
            h[n] = exp(dt * A[d * N + n]) * h[n] + gain * B[b * N + n] * xv;
            y += C[b * N + n] * h[n];
        }
        if (Dskip)
            y += Dskip[d] * xv;
        if (z)
            y *= silu(z[r]);
        out[r] = y;
    }
}

/*
 * Causal depthwise 1-D convolution along L, optionally followed by SiLU: the step
 * that feeds the scan its input u in the listed layer ("Linear Attention vs Softmax
 * Attention ...", section Implementation: a grouped Conv1d with one group per
 * channel, kernel size K, padding K - 1, truncated to the first L outputs, then
 * SiLU).  With x = 0 before the start of the sequence:
 *   out[b,d,t] = act(bias[d] + sum_{j=0}^{K-1} w[d,j] * x[b,d,t + j - (K-1)])
 *   x, out : [Bt, D, L]     w : [D, K]     bias : [D] (nullable)
 */
void oracle_causal_conv1d_f64(int64_t Bt, int64_t D, int64_t L, int64_t K,
                              const double *x, const double *w, const double *bias,
                              int silu_flag, double *out)
{
    int64_t rows = Bt * D;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t d = r % D;
        const double *xr = x + r * L;
        const double *wd = w + d * K;
        for (int64_t t = 0; t < L; ++t) {
            double acc = bias ? bias[d] : 0.0;
            for (int64_t j = 0; j < K; ++j) {
                int64_t src = t + j - (K - 1);
                if (src >= 0)
                    acc += wd[j] * xr[src];
            }
            out[r * L + t] = silu_flag ? silu(acc) : acc;
        }
    }
}


/* sigmoid(x) = 1 / (1 + exp(-x)). */
static double sigm(double x)
{
    return 1.0 / (1.0 + exp(-x));
}

/*
 * Gradients of the selective scan (Euler discretisation, zero initial state) with
 * respect to every input, given dout = dLoss/dout.  The forward is the loop of
 * oracle_scan_f64; this is its reverse-mode chain rule written out step by step,
 * from the last step to the first, keeping every state of the forward (the pages'
 * kernel recomputes them: "Mamba selective state space", the hardware-aware scan;
 * here they are simply stored).  Per row, with g[n] = dLoss/dh_t[n]:
 *   gy     = dout_t * silu(z_t)                 dz_t = dout_t * y_t * silu'(z_t)
 *   dD    += gy * u_t                           du_t = gy * D
 *   g[n]  += gy * C_tn                          dC_tn += gy * h_tn
 *   with a = exp(dt A_n):  ddt += g[n] (A_n a h_(t-1)n + B_tn u_t)
 *                          dA_n += g[n] dt a h_(t-1)n,  dB_tn += g[n] dt u_t,
 *                          du_t += g[n] dt B_tn,        g[n] *= a
 *   ddelta_t = ddt * sigmoid(delta_t + bias) (softplus) or ddt;  dbias += ddelta_t
 * dB and dC sum over the channels of a batch; dA, dD and dbias over batches and steps.
 * Outputs are overwritten; nullable: Dskip/dD, z/dz, bias/dbias.  Serial.
 */
void oracle_scan_bwd_f64(int64_t Bt, int64_t D, int64_t L, int64_t N,
                         const double *u, const double *delta, const double *A,
                         const double *B, const double *C, const double *Dskip,
                         const double *z, const double *bias, int softplus_flag,
                         const double *dout, double *du, double *ddelta, double *dA,
                         double *dB, double *dC, double *dD, double *dz, double *dbias)
{
    for (int64_t i = 0; i < D * N; ++i) dA[i] = 0.0;
    for (int64_t i = 0; i < Bt * N * L; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
    if (dD) for (int64_t i = 0; i < D; ++i) dD[i] = 0.0;
    if (dbias) for (int64_t i = 0; i < D; ++i) dbias[i] = 0.0;
    double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N));
    double *dts = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *ys = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double g[64];
    for (int64_t r = 0; r < Bt * D; ++r) {
        int64_t b = r / D, d = r % D;
        const double *ur = u + r * L, *dr = delta + r * L;
        const double *zr = z ? z + r * L : NULL;
        const double *Bb = B + b * N * L, *Cb = C + b * N * L, *Ad = A + d * N;
        /* forward, keeping h_t (hs row t+1; row 0 = h_(-1) = 0), dt_t and y_t */
        for (int64_t n = 0; n < N; ++n) hs[n] = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double step = dr[t] + (bias ? bias[d] : 0.0);
            if (softplus_flag) step = sp_exact(step);
            dts[t] = step;
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double h = exp(step * Ad[n]) * hs[t * N + n] + step * Bb[n * L + t] * ur[t];
                hs[(t + 1) * N + n] = h;
                y += Cb[n * L + t] * h;
            }
            if (Dskip) y += Dskip[d] * ur[t];
            ys[t] = y;
        }
        /* reverse */
        for (int64_t n = 0; n < N; ++n) g[n] = 0.0;
        for (int64_t t = L - 1; t >= 0; --t) {
            double gy = dout[r * L + t];
            if (zr) {
                double s = sigm(zr[t]);
                dz[r * L + t] = dout[r * L + t] * ys[t] * s * (1.0 + zr[t] * (1.0 - s));
                gy *= zr[t] * s;
            }
            double dut = 0.0;
            if (Dskip) {
                dD[d] += gy * ur[t];
                dut = gy * Dskip[d];
            }
            double dt = dts[t], ddt = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                g[n] += gy * Cb[n * L + t];
                dC[b * N * L + n * L + t] += gy * hs[(t + 1) * N + n];
            }
            for (int64_t n = 0; n < N; ++n) {
                double a = exp(dt * Ad[n]);
                double hp = hs[t * N + n];
                ddt += g[n] * (Ad[n] * a * hp + Bb[n * L + t] * ur[t]);
                dA[d * N + n] += g[n] * dt * a * hp;
                dB[b * N * L + n * L + t] += g[n] * dt * ur[t];
                dut += g[n] * dt * Bb[n * L + t];
                g[n] *= a;
            }
            du[r * L + t] = dut;
            double draw = softplus_flag ? ddt * sigm(dr[t] + (bias ? bias[d] : 0.0)) : ddt;
            ddelta[r * L + t] = draw;
            if (dbias) dbias[d] += draw;
        }
    }
    free(hs);
    free(dts);
    free(ys);
}
