/*
 * ssm_oracle.c -- plain float64 CPU oracle for the selective scan.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * reference that the CUDA library is checked against.  Only the tests, the
 * smoke check and the bench's CPU-baseline leg may load it; the library
 * itself never calls it, and it shares no code, header or constant with the
 * CUDA sources.
 *
 * Sources followed (web pages on Mamba / Vision Mamba / Mamba2):
 *  - "手写简化版Mamba2：状态空间模型如何突破Transformer长序列瓶颈"
 *    (intelliparadigm.com), sec. 2.2: discrete recurrence
 *    h_t = Abar h_{t-1} + Bbar x_t, y_t = C h_t + D x_t with Abar = exp(dt A)
 *    and the Bbar ~= dt B approximation that Mamba uses (the exact
 *    zero-order-hold Bbar of the same section in the *_zoh functions);
 *    sec. 4.2: dt = softplus(...), A negative;
 *    sec. 4.3: the per-time-step reference scan (state zero-initialised,
 *    elementwise decay over the N states, readout summed over N);
 *    sec. 4.4: skip term y + D u and the SiLU gate y * silu(z);
 *    sec. 3.2: the chunked form -- matrix products inside a chunk, the chunk
 *    end-state passed on by a recurrence between chunks.
 *  - "复现Vision Mamba (Vim)" (news.rkmt.cn), sec. 3.1-3.2: the bidirectional
 *    scan runs the sequence forward, runs it again flipped with its own
 *    parameters, flips that result back and adds the two.
 *
 * Readings where the pages are silent (each applied below):
 *  - softplus(v) = log(1 + exp(v)) evaluated exactly (no threshold);
 *  - the reverse direction runs t = L-1 .. 0 from a zero state; its output is
 *    stored at the original t and its last state is the state after t = 0;
 *  - bidirectional: each direction gates with its own z and the two gated
 *    outputs are summed;
 *  - SSD: A and D are scalars per head, B and C are shared by all heads, the
 *    chunk state is carried across chunks (so the chunked form equals the
 *    sequential recurrence).
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double softplus_exact(double v)
{
    /* log(1 + e^v), written so that large v does not overflow */
    if (v > 0.0)
        return v + log1p(exp(-v));
    return log1p(exp(v));
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* dt' for one (time, channel): softplus(delta + bias) or delta + bias. */
static double dt_of(double delta, const double *bias, int64_t d, int softplus)
{
    double v = delta + (bias ? bias[d] : 0.0);
    return softplus ? softplus_exact(v) : v;
}

/*
 * The input coefficient of one state for one step.  The Mamba2 page,
 * sec. 2.2, discretises h' = A h + B x by zero-order hold (x held constant
 * over the step, the equation integrated exactly):
 *   Abar = exp(dt A),   Bbar = (dt A)^-1 (exp(dt A) - I) dt B,
 * and the scans of sec. 4.3 use the approximation Bbar = dt B.  A is
 * diagonal here, so per state the exact coefficient of B is
 * (exp(dt a) - 1) / a, written with expm1 so that small dt a does not
 * cancel; its limit at a = 0 is dt.
 */
static double bbar_coef(double dt, double a, int zoh)
{
    if (!zoh)
        return dt;
    if (a == 0.0)
        return dt;
    return expm1(dt * a) / a;
}

/*
 * One S6 column (batch b, channel d): the recurrence of sec. 4.3 with the
 * skip term and gate of sec. 4.4 (zoh: the exact zero-order-hold Bbar of
 * sec. 2.2 instead of dt B; see bbar_coef).  The state starts at h0 (N
 * values) or, if h0 is NULL, at zero as in sec. 4.3.  mask (Bsz, L) or NULL: a token with
 * mask 0 is bypassed (Samba page, sec. 2: the state is not updated and the
 * computation is skipped) -- h passes through unchanged and y[t] = 0.
 * Writes y[t] for t in [0, L) and the final state (N values) to hlast if
 * non-NULL.
 */
static void s6_column(int64_t b, int64_t d, int64_t L, int64_t D, int64_t N,
                      const double *x, const double *delta, const double *bias, int softplus,
                      const double *A, const double *Bm, const double *Cm, const double *Dv,
                      const double *z, int reverse, double *y, double *hlast, double *h,
                      const double *h0, const unsigned char *mask, int zoh)
{
    for (int64_t n = 0; n < N; n++)
        h[n] = h0 ? h0[n] : 0.0;
    for (int64_t step = 0; step < L; step++) {
        int64_t t = reverse ? (L - 1 - step) : step;
        int64_t i = (b * L + t) * D + d;            /* (b, t, d) */
        if (mask && !mask[b * L + t]) {
            y[t] = 0.0;
            continue;
        }
        double dt = dt_of(delta[i], bias, d, softplus);
        double acc = 0.0;
        for (int64_t n = 0; n < N; n++) {
            double dA = exp(dt * A[d * N + n]);              /* Abar = exp(dt A) */
            double dBx = bbar_coef(dt, A[d * N + n], zoh) * Bm[(b * L + t) * N + n] * x[i];
                                                              /* Bbar x (dt B x unless zoh) */
            h[n] = dA * h[n] + dBx;
            acc += Cm[(b * L + t) * N + n] * h[n];
        }
        if (Dv)
            acc += Dv[d] * x[i];
        if (z)
            acc *= silu(z[i]);
        y[t] = acc;
    }
    if (hlast)
        for (int64_t n = 0; n < N; n++)
            hlast[n] = h[n];
}

/*
 * Single-direction S6.  x, delta, z: (Bsz, L, D); A: (D, N); Bm, Cm:
 * (Bsz, L, N); delta_bias, Dv: (D) or NULL; z NULL disables the gate.
 * out: (Bsz, L, D); last_state: (Bsz, D, N) or NULL; initial_state:
 * (Bsz, D, N), the state before the first step, or NULL for zero; mask:
 * (Bsz, L) bytes or NULL (see s6_column).
 * cols: list of column ids b*D + d to compute (NULL = every column); only
 * those columns of out / last_state are written.  If accumulate is set the
 * column's output is added to out instead of stored.
 */
static void s6_run(int64_t Bsz, int64_t L, int64_t D, int64_t N,
                   const double *x, const double *delta, const double *delta_bias, int softplus,
                   const double *A, const double *Bm, const double *Cm, const double *Dv,
                   const double *z, int reverse, double *out, double *last_state,
                   const double *initial_state, const unsigned char *mask, const int64_t *cols,
                   int64_t ncols, int nthreads, int accumulate, int zoh)
{
    int64_t total = cols ? ncols : Bsz * D;
#ifdef _OPENMP
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *y = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double *h = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
        for (int64_t k = 0; k < total; k++) {
            int64_t col = cols ? cols[k] : k;
            int64_t b = col / D, d = col % D;
            double *hl = last_state ? last_state + (b * D + d) * N : NULL;
            const double *h0 = initial_state ? initial_state + (b * D + d) * N : NULL;
            s6_column(b, d, L, D, N, x, delta, delta_bias, softplus, A, Bm, Cm, Dv, z,
                      reverse, y, hl, h, h0, mask, zoh);
            for (int64_t t = 0; t < L; t++) {
                int64_t i = (b * L + t) * D + d;
                out[i] = accumulate ? out[i] + y[t] : y[t];
            }
        }
        free(y);
        free(h);
    }
}

void oracle_s6(int64_t Bsz, int64_t L, int64_t D, int64_t N,
               const double *x, const double *delta, const double *delta_bias, int softplus,
               const double *A, const double *Bm, const double *Cm, const double *Dv,
               const double *z, int reverse, double *out, double *last_state,
               const int64_t *cols, int64_t ncols, int nthreads)
{
    s6_run(Bsz, L, D, N, x, delta, delta_bias, softplus, A, Bm, Cm, Dv, z, reverse, out,
           last_state, NULL, NULL, cols, ncols, nthreads, 0, 0);
}

/*
 * oracle_s6 from a given state: initial_state (Bsz, D, N) is h before the
 * first step (before t = 0, or before t = L-1 reversed).  The recurrence
 * of sec. 4.3 depends only on the previous h, which is what lets a long
 * sequence run in pieces and lets inference run one step at a time from a
 * stored state (sec. 5.2).
 */
void oracle_s6_state(int64_t Bsz, int64_t L, int64_t D, int64_t N,
                     const double *x, const double *delta, const double *delta_bias, int softplus,
                     const double *A, const double *Bm, const double *Cm, const double *Dv,
                     const double *z, int reverse, const double *initial_state, double *out,
                     double *last_state, const int64_t *cols, int64_t ncols, int nthreads)
{
    s6_run(Bsz, L, D, N, x, delta, delta_bias, softplus, A, Bm, Cm, Dv, z, reverse, out,
           last_state, initial_state, NULL, cols, ncols, nthreads, 0, 0);
}

/*
 * oracle_s6 with a token mask (Bsz, L): masked tokens are bypassed (Samba
 * page, sec. 2) -- the state passes through unchanged and the output is 0.
 * A scan along another order of the positions (Samba page sec. 3.1, the
 * Mamba-YOLO page sec. 1.2 / 4.4) is this scan on inputs gathered in that
 * order, its outputs scattered back (done by the Python wrapper).
 */
void oracle_s6_masked(int64_t Bsz, int64_t L, int64_t D, int64_t N,
                      const double *x, const double *delta, const double *delta_bias, int softplus,
                      const double *A, const double *Bm, const double *Cm, const double *Dv,
                      const double *z, int reverse, const unsigned char *mask, double *out,
                      double *last_state, const int64_t *cols, int64_t ncols, int nthreads)
{
    s6_run(Bsz, L, D, N, x, delta, delta_bias, softplus, A, Bm, Cm, Dv, z, reverse, out,
           last_state, NULL, mask, cols, ncols, nthreads, 0, 0);
}

/*
 * Vision-Mamba bidirectional scan: forward scan with the *_f parameters plus
 * reversed scan with the *_b parameters; x and delta are shared, each
 * direction adds its own bias, gates with its own z, and the results are
 * summed at the original positions.
 */
void oracle_bidir(int64_t Bsz, int64_t L, int64_t D, int64_t N,
                  const double *x, const double *delta, int softplus,
                  const double *bias_f, const double *A_f, const double *B_f, const double *C_f,
                  const double *D_f, const double *z_f, double *last_f,
                  const double *bias_b, const double *A_b, const double *B_b, const double *C_b,
                  const double *D_b, const double *z_b, double *last_b,
                  double *out, const int64_t *cols, int64_t ncols, int nthreads)
{
    s6_run(Bsz, L, D, N, x, delta, bias_f, softplus, A_f, B_f, C_f, D_f, z_f, 0, out, last_f,
           NULL, NULL, cols, ncols, nthreads, 0, 0);
    s6_run(Bsz, L, D, N, x, delta, bias_b, softplus, A_b, B_b, C_b, D_b, z_b, 1, out, last_b,
           NULL, NULL, cols, ncols, nthreads, 1, 0);
}

/*
 * oracle_s6_state with the exact zero-order-hold input coefficient of the
 * Mamba2 page, sec. 2.2 (bbar_coef) in place of dt B.  initial_state may be
 * NULL (zero).
 */
void oracle_s6_zoh(int64_t Bsz, int64_t L, int64_t D, int64_t N,
                   const double *x, const double *delta, const double *delta_bias, int softplus,
                   const double *A, const double *Bm, const double *Cm, const double *Dv,
                   const double *z, int reverse, const double *initial_state, double *out,
                   double *last_state, const int64_t *cols, int64_t ncols, int nthreads)
{
    s6_run(Bsz, L, D, N, x, delta, delta_bias, softplus, A, Bm, Cm, Dv, z, reverse, out,
           last_state, initial_state, NULL, cols, ncols, nthreads, 0, 1);
}

/* oracle_bidir with the zero-order-hold coefficient in both directions. */
void oracle_bidir_zoh(int64_t Bsz, int64_t L, int64_t D, int64_t N,
                      const double *x, const double *delta, int softplus,
                      const double *bias_f, const double *A_f, const double *B_f, const double *C_f,
                      const double *D_f, const double *z_f, double *last_f,
                      const double *bias_b, const double *A_b, const double *B_b, const double *C_b,
                      const double *D_b, const double *z_b, double *last_b,
                      double *out, const int64_t *cols, int64_t ncols, int nthreads)
{
    s6_run(Bsz, L, D, N, x, delta, bias_f, softplus, A_f, B_f, C_f, D_f, z_f, 0, out, last_f,
           NULL, NULL, cols, ncols, nthreads, 0, 1);
    s6_run(Bsz, L, D, N, x, delta, bias_b, softplus, A_b, B_b, C_b, D_b, z_b, 1, out, last_b,
           NULL, NULL, cols, ncols, nthreads, 1, 1);
}

/*
 * Mamba2 SSD, sequential definition: the S6 recurrence with A[d, n] := A_h
 * for every channel d = (h, p) of head h and every state n, dt per head,
 * B and C shared by all heads.
 * x, z: (Bsz, L, H, P); delta: (Bsz, L, H); A, Dv, bias: (H);
 * Bm, Cm: (Bsz, L, N); out: (Bsz, L, H, P); last_state: (Bsz, H, P, N).
 * cols: ids (b*H + h)*P + p (NULL = all).
 */
void oracle_ssd_seq(int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t N,
                    const double *x, const double *delta, const double *bias, int softplus,
                    const double *A, const double *Bm, const double *Cm, const double *Dv,
                    const double *z, double *out, double *last_state,
                    const int64_t *cols, int64_t ncols, int nthreads)
{
    int64_t total = cols ? ncols : Bsz * H * P;
#ifdef _OPENMP
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *h = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
        for (int64_t k = 0; k < total; k++) {
            int64_t col = cols ? cols[k] : k;
            int64_t p = col % P, hd = (col / P) % H, b = col / (P * H);
            for (int64_t n = 0; n < N; n++)
                h[n] = 0.0;
            for (int64_t t = 0; t < L; t++) {
                int64_t ix = ((b * L + t) * H + hd) * P + p;
                double dt = dt_of(delta[(b * L + t) * H + hd], bias, hd, softplus);
                double dA = exp(dt * A[hd]);
                double acc = 0.0;
                for (int64_t n = 0; n < N; n++) {
                    h[n] = dA * h[n] + dt * Bm[(b * L + t) * N + n] * x[ix];
                    acc += Cm[(b * L + t) * N + n] * h[n];
                }
                if (Dv)
                    acc += Dv[hd] * x[ix];
                if (z)
                    acc *= silu(z[ix]);
                out[ix] = acc;
            }
            if (last_state)
                for (int64_t n = 0; n < N; n++)
                    last_state[((b * H + hd) * P + p) * N + n] = h[n];
        }
        free(h);
    }
}

/*
 * Mamba2 SSD, chunked form (sec. 3.2): the sequence is cut into chunks of Q
 * steps.  For chunk c of head h, with a_k = dt_k A_h and cs_i the inclusive
 * sum of a_k from the chunk start to i:
 *   G[i][j]      = sum_n C_i[n] B_j[n]                       (C B^T)
 *   Ydiag[i][p]  = sum_{j<=i} G[i][j] exp(cs_i - cs_j) dt_j x_j[p]
 *   Yoff[i][p]   = exp(cs_i) sum_n C_i[n] S[p][n]           (state entering c)
 *   Schunk[p][n] = sum_j exp(cs_end - cs_j) dt_j B_j[n] x_j[p]
 *   S           <- exp(cs_end) S + Schunk                   (between chunks)
 *   y = (Ydiag + Yoff + D_h x) * silu(z)
 * The last chunk may be shorter than Q.  Same layouts as oracle_ssd_seq;
 * every (b, h) is computed.
 */
void oracle_ssd_chunked(int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t N, int64_t Q,
                        const double *x, const double *delta, const double *bias, int softplus,
                        const double *A, const double *Bm, const double *Cm, const double *Dv,
                        const double *z, double *out, double *last_state, int nthreads)
{
    int64_t total = Bsz * H;
#ifdef _OPENMP
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)(P * N));
        double *Sc = (double *)malloc(sizeof(double) * (size_t)(P * N));
        double *cs = (double *)malloc(sizeof(double) * (size_t)Q);
        double *dt = (double *)malloc(sizeof(double) * (size_t)Q);
        double *G = (double *)malloc(sizeof(double) * (size_t)(Q * Q));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t bh = 0; bh < total; bh++) {
            int64_t b = bh / H, hd = bh % H;
            for (int64_t k = 0; k < P * N; k++)
                S[k] = 0.0;
            for (int64_t c0 = 0; c0 < L; c0 += Q) {
                int64_t q = (L - c0 < Q) ? (L - c0) : Q;
                double run = 0.0;
                for (int64_t i = 0; i < q; i++) {
                    int64_t t = c0 + i;
                    dt[i] = dt_of(delta[(b * L + t) * H + hd], bias, hd, softplus);
                    run += dt[i] * A[hd];
                    cs[i] = run;
                }
                for (int64_t i = 0; i < q; i++)
                    for (int64_t j = 0; j < q; j++) {
                        double g = 0.0;
                        for (int64_t n = 0; n < N; n++)
                            g += Cm[(b * L + c0 + i) * N + n] * Bm[(b * L + c0 + j) * N + n];
                        G[i * Q + j] = g;
                    }
                for (int64_t i = 0; i < q; i++) {
                    int64_t ti = c0 + i;
                    for (int64_t p = 0; p < P; p++) {
                        double yd = 0.0;
                        for (int64_t j = 0; j <= i; j++) {
                            int64_t tj = c0 + j;
                            yd += G[i * Q + j] * exp(cs[i] - cs[j]) * dt[j] *
                                  x[((b * L + tj) * H + hd) * P + p];
                        }
                        double cS = 0.0;
                        for (int64_t n = 0; n < N; n++)
                            cS += Cm[(b * L + ti) * N + n] * S[p * N + n];
                        double yo = exp(cs[i]) * cS;
                        int64_t ix = ((b * L + ti) * H + hd) * P + p;
                        double y = yd + yo + (Dv ? Dv[hd] * x[ix] : 0.0);
                        if (z)
                            y *= silu(z[ix]);
                        out[ix] = y;
                    }
                }
                for (int64_t p = 0; p < P; p++)
                    for (int64_t n = 0; n < N; n++) {
                        double s = 0.0;
                        for (int64_t j = 0; j < q; j++) {
                            int64_t tj = c0 + j;
                            s += exp(cs[q - 1] - cs[j]) * dt[j] * Bm[(b * L + tj) * N + n] *
                                 x[((b * L + tj) * H + hd) * P + p];
                        }
                        Sc[p * N + n] = s;
                    }
                for (int64_t k = 0; k < P * N; k++)
                    S[k] = exp(cs[q - 1]) * S[k] + Sc[k];
            }
            if (last_state)
                for (int64_t k = 0; k < P * N; k++)
                    last_state[(b * H + hd) * P * N + k] = S[k];
        }
        free(S);
        free(Sc);
        free(cs);
        free(dt);
        free(G);
    }
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
