/*
 * fp64 reference ("oracle") for the Mamba mixer core and its one-token decode
 * step.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline and reference legs call it; no product code links
 * or calls it, and it shares no source with the CUDA library.
 *
 * It is the plain definition, written out as a sequential loop in double
 * precision with libm exp/log1p, with no blocking, chunking or reordering:
 *
 *   Jamba hybrid SSM-Transformer lesson, section "SSM in one page":
 *       h_t = A h_{t-1} + B x_t,   y_t = C h_t
 *     (the output at t needs only h_{t-1} and x_t: constant memory, O(1) per
 *     token), with A, B, C made data-dependent per token as in Mamba (the
 *     "selective" part) and, for Mamba, a convolution applied to x_t before
 *     the recurrence (section "Mamba-3", on the outer convolution it replaces).
 *   Step size: the reproduction blog's profile section names Delta as the
 *     parameter that sets how fast the state decays.
 *   The discretised form, conv width, activations, skip and gate follow the
 *   problem statement of the mixer core:
 *       u_t   = SiLU(conv_b + sum_k conv_w[k] * x_{t-W+1+k})   (causal, depthwise)
 *       Delta = softplus(dt_t + dt_bias)
 *       h_t[n] = exp(Delta * A[n]) * h_{t-1}[n] + Delta * B_t[n] * u_t
 *       y_t   = (sum_n C_t[n] h_t[n] + D * u_t) * SiLU(z_t)
 *
 * Readings taken where the sources are silent (each is listed with its reason
 * in the design notes):
 *   - conv_w[d, W-1] multiplies the current token (cross-correlation with W-1
 *     tokens of left context), the left context being conv_state_in (raw,
 *     pre-conv x, oldest first) or zeros;
 *   - the skip term D multiplies u, the same conv+SiLU output that enters B x;
 *   - the gate multiplies the sum (C h + D u) by SiLU(z); no norm between the
 *     readout and the gate.  The RMSNorm the pages place inside the Mamba
 *     layer is taken to act on B_t and C_t before the recurrence
 *     (oracle_rmsnorm_rows, at the end of this file), and is optional;
 *   - A is given directly as a (negative) fp32 [D, N] matrix, not as log(-A);
 *   - one B/C group shared by all channels of a sequence;
 *   - softplus(v) = max(v, 0) + log1p(exp(-|v|)), exact for every v.
 *
 * Inputs are the exact values the GPU receives, widened to double; outputs
 * stay unrounded in double.
 *
 * Functions: oracle_mixer_fwd (the forward above), oracle_state_update (its
 * one-token decode step), oracle_rmsnorm_rows (the RMSNorm of B_t and C_t),
 * oracle_matmul_nt (the projections either side of the scan),
 * oracle_ssd_fwd (the Mamba-2 form: one scalar decay per head, grouped B/C)
 * and oracle_m3_fwd (the Mamba-3 form: trapezoidal rule, rotating complex
 * state, several inputs and outputs per state).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define OR_OK 0
#define OR_ERR_ARG 1

static double or_silu(double v) { return v / (1.0 + exp(-v)); }

static double or_softplus(double v) { return fmax(v, 0.0) + log1p(exp(-fabs(v))); }

/*
 * Mixer forward over a whole sequence (prefill).
 *
 *   xz            [B, L, 2D]   x = xz[..., 0:D], z = xz[..., D:2D]
 *   conv_w        [D, W]       conv_b [D] or NULL (= 0)
 *   dt            [B, L, D]    pre-bias step input; dt_bias [D] or NULL (= 0)
 *   A             [D, N]
 *   Bm, Cm        [B, L, N]
 *   Dskip         [D] or NULL (= 0)
 *   h0            [B, D, N] or NULL (= 0)
 *   conv_state_in [B, D, W-1] or NULL (= 0)
 * Outputs (only channels d in [d_begin, d_end) are written):
 *   y             [B, L, D]
 *   h_last        [B, D, N]    state after token L-1
 *   conv_state_out[B, D, W-1]  the last W-1 raw x, oldest first
 *   u_trace, delta_trace [B, L, D] or NULL: u_t and Delta_t, for the checks
 *   pre_trace     [B, L, D] or NULL: the conv output before SiLU
 */
int oracle_mixer_fwd(const double* xz, const double* conv_w, const double* conv_b,
                     const double* dt, const double* dt_bias, const double* A,
                     const double* Bm, const double* Cm, const double* Dskip,
                     const double* h0, const double* conv_state_in,
                     double* y, double* h_last, double* conv_state_out,
                     double* u_trace, double* delta_trace, double* pre_trace,
                     int64_t Bsz, int64_t L, int64_t D, int64_t N, int64_t W,
                     int64_t d_begin, int64_t d_end)
{
    if (Bsz < 0 || L < 0 || D < 1 || N < 1 || N > 256 || W < 1 || W > 64) return OR_ERR_ARG;
    if (d_begin < 0 || d_end > D || d_begin > d_end) return OR_ERR_ARG;
    if (!xz && L > 0) return OR_ERR_ARG;
    if (!conv_w || !dt || !A || !Bm || !Cm || !y || !h_last || !conv_state_out) return OR_ERR_ARG;

    double h[256];
    double win[64]; /* win[0..W-2]: the W-1 previous raw x, oldest first */

    for (int64_t b = 0; b < Bsz; ++b) {
        for (int64_t d = d_begin; d < d_end; ++d) {
            for (int64_t j = 0; j < W - 1; ++j)
                win[j] = conv_state_in ? conv_state_in[(b * D + d) * (W - 1) + j] : 0.0;
            for (int64_t n = 0; n < N; ++n)
                h[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;

            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = b * L + t;
                const double x = xz[row * 2 * D + d];
                const double z = xz[row * 2 * D + D + d];

                /* causal depthwise conv, then SiLU */
                double pre = conv_b ? conv_b[d] : 0.0;
                for (int64_t k = 0; k < W - 1; ++k)
                    pre += conv_w[d * W + k] * win[k];
                pre += conv_w[d * W + (W - 1)] * x;
                const double u = or_silu(pre);

                /* step size */
                const double delta = or_softplus(dt[row * D + d] + (dt_bias ? dt_bias[d] : 0.0));

                /* selective recurrence and readout */
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double dA = exp(delta * A[d * N + n]);
                    const double dBx = delta * Bm[row * N + n] * u;
                    h[n] = dA * h[n] + dBx;
                    acc += Cm[row * N + n] * h[n];
                }
                const double yv = acc + (Dskip ? Dskip[d] : 0.0) * u;
                y[row * D + d] = yv * or_silu(z);

                if (u_trace) u_trace[row * D + d] = u;
                if (delta_trace) delta_trace[row * D + d] = delta;
                if (pre_trace) pre_trace[row * D + d] = pre;

                /* slide the window: drop the oldest, append this token's raw x */
                for (int64_t j = 0; j + 1 < W - 1; ++j) win[j] = win[j + 1];
                if (W > 1) win[W - 2] = x;
            }

            for (int64_t n = 0; n < N; ++n) h_last[(b * D + d) * N + n] = h[n];
            for (int64_t j = 0; j < W - 1; ++j) conv_state_out[(b * D + d) * (W - 1) + j] = win[j];
        }
    }
    return OR_OK;
}

/*
 * One-token state update (decode) for NL independent stacked layers, in place.
 * Written out on its own (not through the forward above) so the two can be
 * checked against each other.
 *
 *   x, z, dt      [NL, B, D]
 *   conv_w        [NL, D, W]; conv_b, dt_bias, Dskip [NL, D] (each may be NULL = 0)
 *   A             [NL, D, N]
 *   Bm, Cm        [NL, B, N]
 *   ssm_state     [NL, B, D, N]   read, then overwritten with the new state
 *   conv_state    [NL, B, D, W-1] read, then overwritten with the shifted window
 *   y             [NL, B, D]
 * Only rows r = (l * B + b) * D + d with r in [r_begin, r_end) are touched.
 */
int oracle_state_update(const double* x, const double* z, const double* dt,
                        const double* conv_w, const double* conv_b,
                        const double* dt_bias, const double* Dskip,
                        const double* A, const double* Bm, const double* Cm,
                        double* ssm_state, double* conv_state, double* y,
                        int64_t NL, int64_t Bsz, int64_t D, int64_t N, int64_t W,
                        int64_t r_begin, int64_t r_end)
{
    if (NL < 0 || Bsz < 0 || D < 1 || N < 1 || W < 1) return OR_ERR_ARG;
    const int64_t rows = NL * Bsz * D;
    if (r_begin < 0 || r_end > rows || r_begin > r_end) return OR_ERR_ARG;
    if (!x || !z || !dt || !conv_w || !A || !Bm || !Cm || !ssm_state || !y) return OR_ERR_ARG;
    if (W > 1 && !conv_state) return OR_ERR_ARG;

    for (int64_t r = r_begin; r < r_end; ++r) {
        const int64_t d = r % D;
        const int64_t lb = r / D;          /* l * B + b */
        const int64_t l = lb / Bsz;
        const int64_t ld = l * D + d;      /* parameter row */

        double* cs = conv_state ? conv_state + r * (W - 1) : NULL;
        double pre = conv_b ? conv_b[ld] : 0.0;
        for (int64_t k = 0; k < W - 1; ++k) pre += conv_w[ld * W + k] * cs[k];
        pre += conv_w[ld * W + (W - 1)] * x[r];
        const double u = or_silu(pre);

        const double delta = or_softplus(dt[r] + (dt_bias ? dt_bias[ld] : 0.0));

        double* h = ssm_state + r * N;
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double dA = exp(delta * A[ld * N + n]);
            h[n] = dA * h[n] + delta * Bm[lb * N + n] * u;
            acc += Cm[lb * N + n] * h[n];
        }
        y[r] = (acc + (Dskip ? Dskip[ld] : 0.0) * u) * or_silu(z[r]);

        for (int64_t k = 0; k + 1 < W - 1; ++k) cs[k] = cs[k + 1];
        if (W > 1) cs[W - 2] = x[r];
    }
    return OR_OK;
}

/*
 * RMSNorm of each row of a [rows, n] matrix, with one weight per column.
 * Jamba deep-dive report, "standard components" list: RMSNorm sits inside the
 * Mamba layer; large-scale-stability section: it is applied to the layer's
 * internal activations.  Reading taken (the pages do not say which
 * activations): the selective parameters B_t and C_t, each normalised over
 * its d_state entries before it enters the recurrence:
 *
 *     out[r, i] = x[r, i] * w[i] / sqrt(mean_j x[r, j]^2 + eps)
 */
int oracle_rmsnorm_rows(const double* x, const double* w, double eps, double* out, int64_t rows, int64_t n)
{
    if (rows < 0 || n < 1 || !x || !w || !out || !(eps >= 0.0)) return OR_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int64_t i = 0; i < n; ++i) ss += x[r * n + i] * x[r * n + i];
        const double inv = 1.0 / sqrt(ss / (double)n + eps);
        for (int64_t i = 0; i < n; ++i) out[r * n + i] = x[r * n + i] * inv * w[i];
    }
    return OR_OK;
}

/*
 * Dense product with the second operand stored row-major as [N, K] (the
 * layout of a projection's weight, one row per output feature):
 *
 *     C[m, n] = sum_k A[m, k] * Bw[n, k]
 *
 * The projections on either side of the selective scan are such products:
 * x_proj maps the conv output u_t (d_inner) to the low-rank step input, B_t
 * and C_t; dt_proj maps the low-rank step input back to d_inner (the Jamba
 * reproduction blog's LoRA section names the low-rank Delta projection, and
 * the JAMBA hybrid-model blog names x_proj and dt_proj).  Only rows m in
 * [m_begin, m_end) are written.
 */
int oracle_matmul_nt(const double* A, const double* Bw, double* C, int64_t M, int64_t N, int64_t K,
                     int64_t m_begin, int64_t m_end)
{
    if (M < 0 || N < 0 || K < 0 || !A || !Bw || !C) return OR_ERR_ARG;
    if (m_begin < 0 || m_end > M || m_begin > m_end) return OR_ERR_ARG;
    for (int64_t m = m_begin; m < m_end; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += A[m * K + k] * Bw[n * K + k];
            C[m * N + n] = acc;
        }
    }
    return OR_OK;
}


/*
 * Mamba-2 form of the selective scan (the variant the lesson's "SSM in one
 * page" section says simplified the state matrix, and its "Mamba-3" section
 * says discretised with Euler's rule).  The state matrix of each head is a
 * scalar times the identity, so one decay per head and token multiplies the
 * whole state; B_t and C_t are shared by the heads of a group:
 *
 *     Delta_t  = softplus(dt_t[h] + dt_bias[h])
 *     h_t[p,n] = exp(Delta_t A[h]) h_{t-1}[p,n] + Delta_t B_t[g,n] x_t[h,p]
 *     y_t[h,p] = (sum_n C_t[g,n] h_t[p,n] + D[h] x_t[h,p]) * SiLU(z_t[h,p])
 *
 * with g = h / (H / G) (heads split into G equal, consecutive groups) and the
 * gate left out when z is NULL.  x is the layer's input after its
 * convolution; channel c = h * P + p.
 *
 *   x, z          [B, L, H*P]  (z may be NULL: no gate)
 *   dt            [B, L, H]    pre-bias step input; dt_bias [H] or NULL (= 0)
 *   A             [H]          negative
 *   Bm, Cm        [B, L, G, N]
 *   Dskip         [H] or NULL (= 0)
 *   h0            [B, H, P, N] or NULL (= 0)
 * Outputs (only channels c in [c_begin, c_end) are written):
 *   y             [B, L, H*P]
 *   h_last        [B, H, P, N]  state after token L-1
 */
int oracle_ssd_fwd(const double* x, const double* z, const double* dt, const double* dt_bias,
                   const double* A, const double* Bm, const double* Cm, const double* Dskip,
                   const double* h0, double* y, double* h_last,
                   int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                   int64_t c_begin, int64_t c_end)
{
    if (Bsz < 0 || L < 0 || H < 1 || P < 1 || N < 1 || N > 256 || G < 1 || H % G != 0) return OR_ERR_ARG;
    const int64_t C = H * P;
    if (c_begin < 0 || c_end > C || c_begin > c_end) return OR_ERR_ARG;
    if ((!x || !dt || !Bm || !Cm) && L > 0) return OR_ERR_ARG;
    if (!A || !y || !h_last) return OR_ERR_ARG;

    double s[256];
    const int64_t heads_per_group = H / G;

    for (int64_t b = 0; b < Bsz; ++b) {
        for (int64_t c = c_begin; c < c_end; ++c) {
            const int64_t h = c / P;
            const int64_t g = h / heads_per_group;
            for (int64_t n = 0; n < N; ++n)
                s[n] = h0 ? h0[(b * C + c) * N + n] : 0.0;

            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = b * L + t;
                const double xv = x[row * C + c];
                const double delta = or_softplus(dt[row * H + h] + (dt_bias ? dt_bias[h] : 0.0));
                const double decay = exp(delta * A[h]);
                const double* Bt = Bm + (row * G + g) * N;
                const double* Ct = Cm + (row * G + g) * N;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    s[n] = decay * s[n] + delta * Bt[n] * xv;
                    acc += Ct[n] * s[n];
                }
                const double yv = acc + (Dskip ? Dskip[h] : 0.0) * xv;
                y[row * C + c] = z ? yv * or_silu(z[row * C + c]) : yv;
            }

            for (int64_t n = 0; n < N; ++n) h_last[(b * C + c) * N + n] = s[n];
        }
    }
    return OR_OK;
}

/*
 * Mamba-3 form (the lesson's "Mamba-3" section: exponential-trapezoidal
 * discretisation, a complex-valued state equivalent to a data-dependent
 * rotary embedding, and multi-input multi-output projections), on the
 * Mamba-2 layout of heads, groups and channels.  Readings (the section gives
 * no formula): the d_state entries of a channel form N/2 complex numbers
 * (entries 2k, 2k+1 = real, imaginary part of pair k); per head h and token t
 *
 *     Delta_t  = softplus(dt_t[h] + dt_bias[h]),  lambda_t = trap_t[h] (0.5 when trap is NULL)
 *     a_t[k]   = exp(Delta_t A[h]) * (cos(Delta_t theta[h,k]) + i sin(Delta_t theta[h,k]))
 *     u_t[k]   = sum_r (B_t[r,g,2k] + i B_t[r,g,2k+1]) x_t[r,c]        (R inputs share the state)
 *     s_t[k]   = a_t[k] (s_{t-1}[k] + (1 - lambda_t) Delta_t u_{t-1}[k]) + lambda_t Delta_t u_t[k]
 *     y_t[r,c] = (sum_k Re(conj(C_t[r,g,k]) s_t[k]) + D[h] x_t[r,c]) * SiLU(z_t[r,c])   (no gate if z is NULL)
 *
 * The state input u enters through a two-tap (trapezoidal) rule inside the
 * recurrence -- at lambda = 1 it is Mamba-2's Euler step, at 1/2 the
 * trapezoid -- and u_{-1} comes from x_prev / B_prev (the token before the
 * call; zero when NULL), so a sequence split into calls continues exactly.
 *
 *   x, z          [B, L, R, H*P]   (z may be NULL)
 *   dt, trap      [B, L, H]        (trap may be NULL)
 *   dt_bias       [H] or NULL;  A [H] (negative);  theta [H, N/2];  Dskip [H] or NULL
 *   Bm, Cm        [B, L, R, G, N]
 *   h0            [B, H, P, N] or NULL
 *   x_prev        [B, R, H*P] or NULL;  B_prev [B, R, G, N] or NULL
 * Outputs (only channels c in [c_begin, c_end) are written):
 *   y             [B, L, R, H*P]
 *   h_last        [B, H, P, N]
 */
int oracle_m3_fwd(const double* x, const double* z, const double* dt, const double* trap, const double* dt_bias,
                  const double* A, const double* theta, const double* Bm, const double* Cm, const double* Dskip,
                  const double* h0, const double* x_prev, const double* B_prev, double* y, double* h_last,
                  int64_t Bsz, int64_t L, int64_t R, int64_t H, int64_t P, int64_t N, int64_t G,
                  int64_t c_begin, int64_t c_end)
{
    if (Bsz < 0 || L < 0 || R < 1 || R > 16 || H < 1 || P < 1 || N < 2 || N > 256 || N % 2 != 0 || G < 1 ||
        H % G != 0)
        return OR_ERR_ARG;
    const int64_t C = H * P, K = N / 2;
    if (c_begin < 0 || c_end > C || c_begin > c_end) return OR_ERR_ARG;
    if ((!x || !dt || !Bm || !Cm) && L > 0) return OR_ERR_ARG;
    if (!A || !theta || !y || !h_last) return OR_ERR_ARG;

    double sr[128], si[128];     /* state, pair k = sr[k] + i si[k] */
    double ur[128], ui[128];     /* u of the previous token */

    for (int64_t b = 0; b < Bsz; ++b) {
        for (int64_t c = c_begin; c < c_end; ++c) {
            const int64_t h = c / P;
            const int64_t g = h * G / H;   /* the head's B/C group: H / G consecutive heads each */
            for (int64_t k = 0; k < K; ++k) {
                sr[k] = h0 ? h0[(b * C + c) * N + 2 * k] : 0.0;
                si[k] = h0 ? h0[(b * C + c) * N + 2 * k + 1] : 0.0;
                ur[k] = 0.0;
                ui[k] = 0.0;
                if (x_prev && B_prev) {
                    for (int64_t r = 0; r < R; ++r) {
                        const double xv = x_prev[(b * R + r) * C + c];
                        const double* Bp = B_prev + ((b * R + r) * G + g) * N;
                        ur[k] += Bp[2 * k] * xv;
                        ui[k] += Bp[2 * k + 1] * xv;
                    }
                }
            }

            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = b * L + t;
                const double delta = or_softplus(dt[row * H + h] + (dt_bias ? dt_bias[h] : 0.0));
                const double lam = trap ? trap[row * H + h] : 0.5;
                const double mag = exp(delta * A[h]);
                for (int64_t k = 0; k < K; ++k) {
                    /* u_t[k] = sum_r B_t[r] pair k * x_t[r] */
                    double vr = 0.0, vi = 0.0;
                    for (int64_t r = 0; r < R; ++r) {
                        const double xv = x[(row * R + r) * C + c];
                        const double* Bt = Bm + ((row * R + r) * G + g) * N;
                        vr += Bt[2 * k] * xv;
                        vi += Bt[2 * k + 1] * xv;
                    }
                    /* s = a (s + (1 - lambda) Delta u_prev) + lambda Delta u */
                    const double pr = sr[k] + (1.0 - lam) * delta * ur[k];
                    const double pi = si[k] + (1.0 - lam) * delta * ui[k];
                    const double ang = delta * theta[h * K + k];
                    const double ar = mag * cos(ang), ai = mag * sin(ang);
                    sr[k] = ar * pr - ai * pi + lam * delta * vr;
                    si[k] = ar * pi + ai * pr + lam * delta * vi;
                    ur[k] = vr;
                    ui[k] = vi;
                }
                for (int64_t r = 0; r < R; ++r) {
                    const double* Ct = Cm + ((row * R + r) * G + g) * N;
                    double acc = 0.0;
                    for (int64_t k = 0; k < K; ++k) acc += Ct[2 * k] * sr[k] + Ct[2 * k + 1] * si[k];
                    const double xv = x[(row * R + r) * C + c];
                    const double yv = acc + (Dskip ? Dskip[h] : 0.0) * xv;
                    const int64_t o = (row * R + r) * C + c;
                    y[o] = z ? yv * or_silu(z[o]) : yv;
                }
            }

            for (int64_t k = 0; k < K; ++k) {
                h_last[(b * C + c) * N + 2 * k] = sr[k];
                h_last[(b * C + c) * N + 2 * k + 1] = si[k];
            }
        }
    }
    return OR_OK;
}
