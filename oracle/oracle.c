/*
 * oracle.c -- plain, slow fp64 CPU reference for the Newton (DEER) and quasi-Newton
 * evaluation of nonlinear RNNs over the whole sequence, its fixed-point variants
 * (Jacobi, Picard, ELK), the linear scans, the adjoint, and the fixed-step simulation
 * of linear ODEs (lsim).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or constant with the CUDA
 * library: it is written from the pages' description of the method.
 *
 * Sources (page title, section):
 *   [DEER]  "Parallelizing non-linear sequential models over the sequence length"
 *           (Lim et al.), summary sections "Approach", "Key results", "Limitations".
 *   [ELK]   "Towards Scalable and Stable Parallelization of Nonlinear RNNs"
 *           (Gonzalez et al., arXiv 2407.19115), Abstract  (quasi-Newton = diagonal Jacobian).
 *   [PARA]  "ParaRNN: Unlocking Parallel Training of Nonlinear RNNs for Large Language
 *           Models", abstract  (one system of equations solved by Newton iterations).
 *   [SEQ]   "Para-Seq" README, sections "Main features" (diagonal ParaGRU,
 *           CIFG/peephole ParaLSTM with 2x2 blocks, vanilla tanh RNN, adjoint
 *           backward, scan-based fixed-step ODE solvers), "Quick example" (lsim) and
 *           "Background" (linearise, then solve the linear recurrence).
 *
 * Readings taken where the pages are silent (each is also listed in the design notes):
 *   - Newton update in the b-form: J_t and f_t are evaluated at the previous iterate,
 *     b_t = f_t - J_t h^(k)_{t-1}, and h^(k+1)_t = J_t h^(k+1)_{t-1} + b_t.
 *   - delta_k = max over every state element of |h^(k+1) - h^(k)|; stop when
 *     delta_k < tol (strict) or k+1 = max_iters; iters counts the updates applied.
 *   - initial iterate h^(0)_t = 0 for t >= 1; h_0 is given.
 *   - ParaLSTM: CIFG (input gate = 1 - forget gate), forget peephole on c_{t-1},
 *     output peephole on the new c_t, no peephole on the candidate, diagonal
 *     recurrent weights; state (c, h) per unit, so each unit has a 2x2 Jacobian.
 *
 * Layouts (row-major, batch first): xproj [B][T][G][H] (G = 3, or 1 for tanh);
 * GRU state [B][T][H]; LSTM state [B][T][H][2] as (c, h); tanh state [B][T][n].
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_GRU = 0, ORC_LSTM = 1, ORC_TANH = 2 };
enum { ORC_SCAN_DIAG = 0, ORC_SCAN_BLOCK2 = 1, ORC_SCAN_DENSE = 2 };

typedef struct {
    int cell;            /* ORC_GRU / ORC_LSTM / ORC_TANH */
    int quasi;           /* keep only the diagonal of the Jacobian in the Newton iteration
                          * [ELK]: tanh (n x n -> diagonal) and LSTM (each 2x2 block -> its
                          * diagonal, the ParaLSTM diagonal scan backend [SEQ]) */
    long B, T, H;        /* H = units (GRU, LSTM) or state size n (tanh) */
    const double *xproj; /* [B][T][G][H]: W x_t + bias per gate (tanh: U x_t + b) */
    const double *a;     /* [3][H] recurrent diagonals: GRU (z,r,c), LSTM (f,g,o) */
    const double *peep;  /* [2][H] LSTM peepholes (w_f, w_o) */
    const double *A;     /* [n][n] tanh recurrent matrix */
    int solver;          /* linearisation used by orc_newton: ORC_NEWTON (the cell's
                          * Jacobian, or its diagonal with quasi), ORC_JACOBI (J = 0),
                          * ORC_PICARD (J = I) ["Para-Seq" README, Main features], or
                          * ORC_ELK (damped step, see orc_newton: the LSTM's full 2x2
                          * blocks, or their diagonals with quasi; GRU's diagonal; for
                          * the tanh RNN the diagonal of its dense Jacobian) */
    double lambda;       /* ELK damping (>= 0; 0 gives the Newton step of the same
                          * linearisation) */
} orc_model;

enum { ORC_NEWTON = 0, ORC_JACOBI = 1, ORC_PICARD = 2, ORC_ELK = 3 };

/* The fixed-point schemes share the Newton loop and differ only in the matrix the step
 * map is linearised with: Jacobi keeps none of it (every step is re-evaluated from
 * the previous iterate), Picard the identity (the update accumulates the increments
 * f(h^(k)_{t-1}) - h^(k)_{t-1} along t). */
static void solver_jacobian(const orc_model *m, long D, double *J)
{
    if (m->solver == ORC_NEWTON || m->solver == ORC_ELK) return;
    for (long i = 0; i < D; ++i)
        for (long j = 0; j < D; ++j) J[i * D + j] = (m->solver == ORC_PICARD && i == j) ? 1.0 : 0.0;
}

void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double sigm(double u) { return 1.0 / (1.0 + exp(-u)); }

static long state_per_unit(const orc_model *m) { return m->cell == ORC_LSTM ? 2 : 1; }

/* ------------------------------------------------------------------------------------
 * Cells.  [SEQ] "Main features": ParaGRU is a diagonal GRU, ParaLSTM a CIFG/peephole
 * LSTM, ParaRNN a vanilla tanh RNN.
 * ---------------------------------------------------------------------------------- */

/* Diagonal ParaGRU, one unit:
 *   z = s(p_z + a_z h), r = s(p_r + a_r h), c = tanh(p_c + a_c (r h)),
 *   f = (1 - z) h + z c.
 * Every operation is elementwise in h, so the Jacobian is one number per unit.
 * dp (optional) receives df/dp_z, df/dp_r, df/dp_c. */
static void gru_unit(double pz, double pr, double pc, double az, double ar, double ac,
                     double h, double *f, double *J, double dp[3])
{
    double z = sigm(pz + az * h);
    double r = sigm(pr + ar * h);
    double c = tanh(pc + ac * (r * h));
    *f = (1.0 - z) * h + z * c;
    double dz = z * (1.0 - z), dr = r * (1.0 - r), dc = 1.0 - c * c;
    /* df/dh = (1-z) + (c-h) dz/dh + z dc/dh, dz/dh = dz a_z, dc/dh = dc a_c (r + h dr a_r) */
    *J = (1.0 - z) + (c - h) * dz * az + z * dc * ac * (r + h * dr * ar);
    if (dp) {
        dp[0] = (c - h) * dz;
        dp[1] = z * dc * ac * h * dr;
        dp[2] = z * dc;
    }
}

/* CIFG + peephole ParaLSTM with diagonal recurrent weights, one unit, state (c, h):
 *   phi = s(p_f + a_f h + w_f c)          forget gate (input gate = 1 - phi)
 *   g   = tanh(p_g + a_g h)               candidate
 *   c'  = phi c + (1 - phi) g
 *   o   = s(p_o + a_o h + w_o c')         output gate, peephole on the new cell
 *   h'  = o tanh(c')
 * J is the 2x2 matrix d(c', h')/d(c, h), row-major.
 * dp (optional) is [2][3]: d(c', h')/d(p_f, p_g, p_o). */
static void lstm_unit(double pf, double pg, double po, double af, double ag, double ao,
                      double wf, double wo, double c, double h, double f[2], double J[4],
                      double dp[6], double *cnew_out)
{
    double phi = sigm(pf + af * h + wf * c);
    double g = tanh(pg + ag * h);
    double cn = phi * c + (1.0 - phi) * g;
    double o = sigm(po + ao * h + wo * cn);
    double tc = tanh(cn);
    f[0] = cn;
    f[1] = o * tc;
    double dphi = phi * (1.0 - phi), dg = 1.0 - g * g, dout = o * (1.0 - o), dtc = 1.0 - tc * tc;
    double dcn_dc = phi + (c - g) * dphi * wf;
    double dcn_dh = (c - g) * dphi * af + (1.0 - phi) * dg * ag;
    double kappa = dout * wo * tc + o * dtc; /* total dh'/dc' through o and tanh */
    J[0] = dcn_dc;
    J[1] = dcn_dh;
    J[2] = kappa * dcn_dc;
    J[3] = dout * ao * tc + kappa * dcn_dh;
    if (dp) {
        double dcn_dpf = (c - g) * dphi, dcn_dpg = (1.0 - phi) * dg;
        dp[0] = dcn_dpf;
        dp[1] = dcn_dpg;
        dp[2] = 0.0;
        dp[3] = kappa * dcn_dpf;
        dp[4] = kappa * dcn_dpg;
        dp[5] = dout * tc;
    }
    if (cnew_out) *cnew_out = cn;
}

/* Vanilla tanh RNN, whole state: f = tanh(A h + p), J = diag(1 - f^2) A.
 * With quasi set, only the diagonal of J is kept [ELK].  J is n x n, row-major. */
static void tanh_step(const orc_model *m, const double *p, const double *h, double *f, double *J)
{
    long n = m->H;
    for (long i = 0; i < n; ++i) {
        double u = p[i];
        for (long j = 0; j < n; ++j) u += m->A[i * n + j] * h[j];
        f[i] = tanh(u);
    }
    for (long i = 0; i < n; ++i) {
        double d = 1.0 - f[i] * f[i];
        for (long j = 0; j < n; ++j) {
            double v = d * m->A[i * n + j];
            J[i * n + j] = (m->quasi && i != j) ? 0.0 : v;
        }
    }
}

/* One unit of a GRU/LSTM at step t of sequence b, from the previous unit state hp. */
static void unit_eval(const orc_model *m, long b, long t, long u, const double *hp, double *f,
                      double *J, double *dp, double *cnew)
{
    long H = m->H;
    const double *p = m->xproj + (b * m->T + t) * 3 * H;
    if (m->cell == ORC_GRU) {
        gru_unit(p[u], p[H + u], p[2 * H + u], m->a[u], m->a[H + u], m->a[2 * H + u], hp[0], f, J,
                 dp);
    } else {
        lstm_unit(p[u], p[H + u], p[2 * H + u], m->a[u], m->a[H + u], m->a[2 * H + u], m->peep[u],
                  m->peep[H + u], hp[0], hp[1], f, J, dp, cnew);
    }
}

/* One step of the whole model at (b, t): f (length D) and the full D x D Jacobian of
 * the step map (D = H, 2H or n).  For GRU/LSTM the Jacobian is placed on its
 * diagonal / 2x2 diagonal blocks in the (c, h)-interleaved state order. */
int orc_step(const orc_model *m, long b, long t, const double *hp, double *f, double *J)
{
    if (m->cell == ORC_TANH) {
        tanh_step(m, m->xproj + (b * m->T + t) * m->H, hp, f, J);
        return 0;
    }
    long S = state_per_unit(m), D = m->H * S;
    memset(J, 0, sizeof(double) * D * D);
    for (long u = 0; u < m->H; ++u) {
        double fu[2], Ju[4];
        unit_eval(m, b, t, u, hp + u * S, fu, Ju, NULL, NULL);
        for (long i = 0; i < S; ++i) {
            f[u * S + i] = fu[i];
            for (long j = 0; j < S; ++j) J[(u * S + i) * D + (u * S + j)] = Ju[i * S + j];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Sequential rollout h_t = f(h_{t-1}, x_t): the "naive sequential application"
 * [PARA] and the ground truth the parallel solve must reproduce [DEER, Approach].
 * ---------------------------------------------------------------------------------- */
int orc_rollout(const orc_model *m, const double *h0, double *h)
{
    long B = m->B, T = m->T, H = m->H;
    if (m->cell == ORC_TANH) {
        long n = H;
#pragma omp parallel for schedule(dynamic, 1)
        for (long b = 0; b < B; ++b) {
            double *J = malloc(sizeof(double) * n * n);
            for (long t = 0; t < T; ++t) {
                const double *hp = t ? h + (b * T + t - 1) * n : (h0 ? h0 + b * n : NULL);
                double *zero = NULL;
                if (!hp) {
                    zero = calloc(n, sizeof(double));
                    hp = zero;
                }
                tanh_step(m, m->xproj + (b * T + t) * n, hp, h + (b * T + t) * n, J);
                free(zero);
            }
            free(J);
        }
        return 0;
    }
    long S = state_per_unit(m);
#pragma omp parallel for schedule(static)
    for (long bu = 0; bu < B * H; ++bu) {
        long b = bu / H, u = bu % H;
        double prev[2] = {0.0, 0.0}, f[2], J[4];
        if (h0)
            for (long s = 0; s < S; ++s) prev[s] = h0[(b * H + u) * S + s];
        for (long t = 0; t < T; ++t) {
            unit_eval(m, b, t, u, prev, f, J, NULL, NULL);
            for (long s = 0; s < S; ++s) {
                h[((b * T + t) * H + u) * S + s] = f[s];
                prev[s] = f[s];
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Newton (DEER) and quasi-Newton iterations [DEER, Approach; PARA; ELK, Abstract].
 * For every t, linearise the cell at the previous iterate: J_t = df/dh (h^(k)_{t-1}),
 * b_t = f(h^(k)_{t-1}) - J_t h^(k)_{t-1}; then solve the linear recurrence
 * h^(k+1)_t = J_t h^(k+1)_{t-1} + b_t sequentially from h_0.
 * The linearisation at step t reads only the previous iterate, so evaluating it just
 * before the recurrence consumes it gives the same numbers as a separate pass.
 * delta_log[k] receives delta_k (up to log_len entries).
 * ---------------------------------------------------------------------------------- */
static double absmax_update(double cur, double v)
{
    if (isnan(v)) return INFINITY;
    v = fabs(v);
    return v > cur ? v : cur;
}

/* ELK ["Towards Scalable and Stable Parallelization of Nonlinear RNNs", Abstract: the
 * Levenberg-Marquardt step computed by Kalman smoothing], for a diagonal linearisation.
 * With x = h^(k+1) - h^(k), a_t the diagonal of J_t and r_t = f_t - h^(k)_t, the damped
 * step minimises
 *     sum_t (x_t - a_t x_{t-1} - r_t)^2 + lambda sum_t x_t^2,    x_0 = 0 (h_0 is given),
 * the Levenberg-Marquardt objective of the stacked residual.  That is the MAP path of
 * the state-space model x_t = a_t x_{t-1} + r_t + w_t, w_t ~ N(0, 1), observed as
 * y_t = 0 = x_t + v_t, v_t ~ N(0, 1/lambda): a Kalman filter forward, then a
 * Rauch-Tung-Striebel smoother backward, one scalar component at a time.  lambda = 0
 * (no observations) returns the quasi-Newton step.  Scratch: 5 T doubles. */
static void elk_component(long T, const double *a, const double *r, double lambda, double *xs, double *work)
{
    double *Pm = work, *mm = work + T, *P = work + 2 * T, *mf = work + 3 * T;
    double Pp = 0.0, mp = 0.0; /* filtered variance and mean before t = 0 (known) */
    for (long t = 0; t < T; ++t) {
        Pm[t] = a[t] * a[t] * Pp + 1.0;           /* predicted variance */
        mm[t] = a[t] * mp + r[t];                 /* predicted mean */
        const double K = lambda * Pm[t] / (1.0 + lambda * Pm[t]); /* gain, Pm / (Pm + 1/lambda) */
        P[t] = (1.0 - K) * Pm[t];
        mf[t] = (1.0 - K) * mm[t];                /* update with the observation 0 */
        Pp = P[t];
        mp = mf[t];
    }
    xs[T - 1] = mf[T - 1];
    for (long t = T - 2; t >= 0; --t) {
        const double G = P[t] * a[t + 1] / Pm[t + 1];
        xs[t] = mf[t] + G * (xs[t + 1] - mm[t + 1]);
    }
}

/* ELK with a 2x2 block linearisation [ELK, Abstract: ELK with the Jacobian itself,
 * quasi-ELK with its diagonal]: the same objective with x_t, r_t in R^2 and J_t the
 * unit's 2x2 Jacobian block (row-major),
 *     sum_t |x_t - J_t x_{t-1} - r_t|^2 + lambda sum_t |x_t|^2,    x_{-1} = 0,
 * the MAP path of x_t = J_t x_{t-1} + r_t + w_t, w_t ~ N(0, I), observed as
 * 0 = x_t + v_t, v_t ~ N(0, I / lambda).  Kalman filter with 2x2 covariances:
 *     Pm_t = J_t P_{t-1} J_t^T + I,  mm_t = J_t m_{t-1} + r_t,
 *     K_t = lambda Pm_t (I + lambda Pm_t)^{-1},  P_t = (I - K_t) Pm_t,  m_t = (I - K_t) mm_t,
 * then the Rauch-Tung-Striebel smoother
 *     x_{T-1} = m_{T-1},  x_t = m_t + G_t (x_{t+1} - mm_{t+1}),  G_t = P_t J_{t+1}^T Pm_{t+1}^{-1}.
 * lambda = 0 gives K = 0 and x = the forward recursion (the Newton step).  Scratch: 12 T. */
static void inv2(const double *M, double *R)
{
    const double det = M[0] * M[3] - M[1] * M[2];
    R[0] = M[3] / det;
    R[1] = -M[1] / det;
    R[2] = -M[2] / det;
    R[3] = M[0] / det;
}
static void mul2(const double *X, const double *Y, double *R) /* R = X Y (2x2, row-major) */
{
    const double r0 = X[0] * Y[0] + X[1] * Y[2], r1 = X[0] * Y[1] + X[1] * Y[3];
    const double r2 = X[2] * Y[0] + X[3] * Y[2], r3 = X[2] * Y[1] + X[3] * Y[3];
    R[0] = r0;
    R[1] = r1;
    R[2] = r2;
    R[3] = r3;
}
static void elk_block2(long T, const double *J, const double *r, double lambda, double *xs, double *work)
{
    double *Pm = work, *mm = work + 4 * T, *P = work + 6 * T, *mf = work + 10 * T;
    double Pp[4] = {0.0, 0.0, 0.0, 0.0}, mp[2] = {0.0, 0.0};
    for (long t = 0; t < T; ++t) {
        const double *Jt = J + 4 * t;
        double JP[4], Jtr[4] = {Jt[0], Jt[2], Jt[1], Jt[3]};
        mul2(Jt, Pp, JP);
        mul2(JP, Jtr, Pm + 4 * t);
        Pm[4 * t] += 1.0;
        Pm[4 * t + 3] += 1.0;
        mm[2 * t] = Jt[0] * mp[0] + Jt[1] * mp[1] + r[2 * t];
        mm[2 * t + 1] = Jt[2] * mp[0] + Jt[3] * mp[1] + r[2 * t + 1];
        double Sm[4] = {lambda * Pm[4 * t] + 1.0, lambda * Pm[4 * t + 1], lambda * Pm[4 * t + 2],
                        lambda * Pm[4 * t + 3] + 1.0}, Si[4], K[4], IK[4];
        inv2(Sm, Si);                       /* (I + lambda Pm)^{-1} */
        mul2(Pm + 4 * t, Si, K);            /* Pm (I + lambda Pm)^{-1} */
        for (int q = 0; q < 4; ++q) K[q] *= lambda;
        IK[0] = 1.0 - K[0];
        IK[1] = -K[1];
        IK[2] = -K[2];
        IK[3] = 1.0 - K[3];
        mul2(IK, Pm + 4 * t, P + 4 * t);
        mf[2 * t] = IK[0] * mm[2 * t] + IK[1] * mm[2 * t + 1];
        mf[2 * t + 1] = IK[2] * mm[2 * t] + IK[3] * mm[2 * t + 1];
        for (int q = 0; q < 4; ++q) Pp[q] = P[4 * t + q];
        mp[0] = mf[2 * t];
        mp[1] = mf[2 * t + 1];
    }
    xs[2 * (T - 1)] = mf[2 * (T - 1)];
    xs[2 * (T - 1) + 1] = mf[2 * (T - 1) + 1];
    for (long t = T - 2; t >= 0; --t) {
        const double *Jn = J + 4 * (t + 1);
        double Jnt[4] = {Jn[0], Jn[2], Jn[1], Jn[3]}, PJ[4], Pmi[4], G[4];
        mul2(P + 4 * t, Jnt, PJ);
        inv2(Pm + 4 * (t + 1), Pmi);
        mul2(PJ, Pmi, G);
        const double e0 = xs[2 * (t + 1)] - mm[2 * (t + 1)], e1 = xs[2 * (t + 1) + 1] - mm[2 * (t + 1) + 1];
        xs[2 * t] = mf[2 * t] + G[0] * e0 + G[1] * e1;
        xs[2 * t + 1] = mf[2 * t + 1] + G[2] * e0 + G[3] * e1;
    }
}

/* Exported for the CPU pins of the block smoother: J [T][4], r [T][2] -> xs [T][2]. */
int orc_elk_block2(long T, const double *J, const double *r, double lambda, double *xs)
{
    double *work = malloc(sizeof(double) * 12 * (T > 0 ? T : 1));
    if (!work) return -1;
    if (T > 0) elk_block2(T, J, r, lambda, xs, work);
    free(work);
    return 0;
}

/* Exported for the CPU pins of the scalar smoother: a [T], r [T] -> xs [T]. */
int orc_elk_scalar(long T, const double *a, const double *r, double lambda, double *xs)
{
    double *work = malloc(sizeof(double) * 5 * (T > 0 ? T : 1));
    if (!work) return -1;
    if (T > 0) elk_component(T, a, r, lambda, xs, work);
    free(work);
    return 0;
}

int orc_newton(const orc_model *m, const double *h0, int max_iters, double tol, double *h_out,
               int *iters_out, double *delta_log, int log_len)
{
    long B = m->B, T = m->T, H = m->H, S = state_per_unit(m);
    long N = (m->cell == ORC_TANH) ? B * T * H : B * T * H * S;
    double *hk = h_out; /* iterate k */
    double *hn = malloc(sizeof(double) * (N > 0 ? N : 1));
    if (!hn) return -1;
    memset(hk, 0, sizeof(double) * N); /* h^(0) = 0 */
    int iters = 0;
    for (int k = 0; k < max_iters; ++k) {
        double delta = 0.0;
        if (m->cell == ORC_TANH && m->solver == ORC_ELK) {
            /* quasi-ELK for the dense tanh RNN: the diagonal of its Jacobian at h^(k),
             * then the same per-unit Kalman smoother as the diagonal cells below */
            long n = H;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : delta)
            for (long b = 0; b < B; ++b) {
                double *J = malloc(sizeof(double) * n * n), *f = malloc(sizeof(double) * n);
                double *a = malloc(sizeof(double) * n * T), *r = malloc(sizeof(double) * n * T);
                double *xs = malloc(sizeof(double) * T), *work = malloc(sizeof(double) * 5 * T);
                double *z0 = calloc(n, sizeof(double));
                const double *pk = h0 ? h0 + b * n : z0; /* h^(k)_{t-1} */
                for (long t = 0; t < T; ++t) {
                    tanh_step(m, m->xproj + (b * T + t) * n, pk, f, J);
                    for (long i = 0; i < n; ++i) {
                        a[i * T + t] = J[i * n + i];
                        r[i * T + t] = f[i] - hk[(b * T + t) * n + i];
                    }
                    pk = hk + (b * T + t) * n;
                }
                double dloc = 0.0;
                for (long i = 0; i < n; ++i) {
                    elk_component(T, a + i * T, r + i * T, m->lambda, xs, work);
                    for (long t = 0; t < T; ++t) {
                        long idx = (b * T + t) * n + i;
                        hn[idx] = hk[idx] + xs[t];
                        dloc = absmax_update(dloc, xs[t]);
                    }
                }
                if (dloc > delta) delta = dloc;
                free(J);
                free(f);
                free(a);
                free(r);
                free(xs);
                free(work);
                free(z0);
            }
        } else if (m->cell == ORC_TANH) {
            long n = H;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : delta)
            for (long b = 0; b < B; ++b) {
                double *J = malloc(sizeof(double) * n * n);
                double *f = malloc(sizeof(double) * n), *bt = malloc(sizeof(double) * n);
                double *z0 = calloc(n, sizeof(double));
                const double *pk = h0 ? h0 + b * n : z0; /* h^(k)_{t-1}   */
                const double *pn = pk;                   /* h^(k+1)_{t-1} */
                double dloc = 0.0;
                for (long t = 0; t < T; ++t) {
                    tanh_step(m, m->xproj + (b * T + t) * n, pk, f, J);
                    solver_jacobian(m, n, J);
                    for (long i = 0; i < n; ++i) { /* b_t = f_t - J_t h^(k)_{t-1} */
                        double s = f[i];
                        for (long j = 0; j < n; ++j) s -= J[i * n + j] * pk[j];
                        bt[i] = s;
                    }
                    double *out = hn + (b * T + t) * n;
                    for (long i = 0; i < n; ++i) { /* h^(k+1)_t = J_t h^(k+1)_{t-1} + b_t */
                        double s = bt[i];
                        for (long j = 0; j < n; ++j) s += J[i * n + j] * pn[j];
                        out[i] = s;
                        dloc = absmax_update(dloc, s - hk[(b * T + t) * n + i]);
                    }
                    pk = hk + (b * T + t) * n;
                    pn = out;
                }
                if (dloc > delta) delta = dloc;
                free(J);
                free(f);
                free(bt);
                free(z0);
            }
        } else if (m->solver == ORC_ELK && S == 2 && !m->quasi) {
            /* ELK with each unit's full 2x2 Jacobian block */
#pragma omp parallel for schedule(static) reduction(max : delta)
            for (long bu = 0; bu < B * H; ++bu) {
                long b = bu / H, u = bu % H;
                double *Jb = malloc(sizeof(double) * T * 4), *r = malloc(sizeof(double) * T * 2);
                double *xs = malloc(sizeof(double) * T * 2), *work = malloc(sizeof(double) * 12 * T);
                double pk[2] = {0.0, 0.0}, f[2], J[4];
                if (h0)
                    for (long s = 0; s < 2; ++s) pk[s] = h0[(b * H + u) * 2 + s];
                for (long t = 0; t < T; ++t) { /* linearise at h^(k): the block, the residual */
                    unit_eval(m, b, t, u, pk, f, J, NULL, NULL);
                    long idx = ((b * T + t) * H + u) * 2;
                    for (int q = 0; q < 4; ++q) Jb[4 * t + q] = J[q];
                    for (long s = 0; s < 2; ++s) {
                        r[2 * t + s] = f[s] - hk[idx + s];
                        pk[s] = hk[idx + s];
                    }
                }
                elk_block2(T, Jb, r, m->lambda, xs, work);
                double dloc = 0.0;
                for (long t = 0; t < T; ++t)
                    for (long s = 0; s < 2; ++s) {
                        long idx = ((b * T + t) * H + u) * 2 + s;
                        hn[idx] = hk[idx] + xs[2 * t + s];
                        dloc = absmax_update(dloc, xs[2 * t + s]);
                    }
                if (dloc > delta) delta = dloc;
                free(Jb);
                free(r);
                free(xs);
                free(work);
            }
        } else if (m->solver == ORC_ELK) {
            /* ELK on a diagonal linearisation (ParaGRU; the ParaLSTM's block diagonal with
             * quasi set): one scalar smoother per state component */
#pragma omp parallel for schedule(static) reduction(max : delta)
            for (long bu = 0; bu < B * H; ++bu) {
                long b = bu / H, u = bu % H;
                double *a = malloc(sizeof(double) * T * S), *r = malloc(sizeof(double) * T * S);
                double *xs = malloc(sizeof(double) * T), *work = malloc(sizeof(double) * 5 * T);
                double pk[2] = {0.0, 0.0}, f[2], J[4];
                if (h0)
                    for (long s = 0; s < S; ++s) pk[s] = h0[(b * H + u) * S + s];
                for (long t = 0; t < T; ++t) { /* linearise at h^(k): diagonal of J, residual */
                    unit_eval(m, b, t, u, pk, f, J, NULL, NULL);
                    long idx = ((b * T + t) * H + u) * S;
                    for (long s = 0; s < S; ++s) {
                        a[s * T + t] = J[s * S + s];
                        r[s * T + t] = f[s] - hk[idx + s];
                        pk[s] = hk[idx + s];
                    }
                }
                double dloc = 0.0;
                for (long s = 0; s < S; ++s) {
                    elk_component(T, a + s * T, r + s * T, m->lambda, xs, work);
                    for (long t = 0; t < T; ++t) {
                        long idx = ((b * T + t) * H + u) * S + s;
                        hn[idx] = hk[idx] + xs[t];
                        dloc = absmax_update(dloc, xs[t]);
                    }
                }
                if (dloc > delta) delta = dloc;
                free(a);
                free(r);
                free(xs);
                free(work);
            }
        } else {
#pragma omp parallel for schedule(static) reduction(max : delta)
            for (long bu = 0; bu < B * H; ++bu) {
                long b = bu / H, u = bu % H;
                double pk[2] = {0.0, 0.0}, pn[2], f[2], J[4], bt[2];
                if (h0)
                    for (long s = 0; s < S; ++s) pk[s] = h0[(b * H + u) * S + s];
                pn[0] = pk[0];
                pn[1] = pk[1];
                double dloc = 0.0;
                for (long t = 0; t < T; ++t) {
                    unit_eval(m, b, t, u, pk, f, J, NULL, NULL);
                    if (m->quasi && S == 2) { /* diagonal of the 2x2 block: c and h decouple */
                        J[1] = 0.0;
                        J[2] = 0.0;
                    }
                    solver_jacobian(m, S, J);
                    long idx = ((b * T + t) * H + u) * S;
                    for (long i = 0; i < S; ++i) {
                        double s = f[i];
                        for (long j = 0; j < S; ++j) s -= J[i * S + j] * pk[j];
                        bt[i] = s;
                    }
                    double nw[2];
                    for (long i = 0; i < S; ++i) {
                        double s = bt[i];
                        for (long j = 0; j < S; ++j) s += J[i * S + j] * pn[j];
                        nw[i] = s;
                    }
                    for (long i = 0; i < S; ++i) {
                        dloc = absmax_update(dloc, nw[i] - hk[idx + i]);
                        hn[idx + i] = nw[i];
                        pk[i] = hk[idx + i];
                        pn[i] = nw[i];
                    }
                }
                if (dloc > delta) delta = dloc;
            }
        }
        double *tmp = hk;
        hk = hn;
        hn = tmp;
        iters = k + 1;
        if (delta_log && k < log_len) delta_log[k] = delta;
        if (delta < tol) break;
    }
    if (hk != h_out) {
        memcpy(h_out, hk, sizeof(double) * N);
        free(hk);
    } else {
        free(hn);
    }
    *iters_out = iters;
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Linear recurrences solved sequentially [SEQ, Main features: dense, diagonal and
 * 2x2 block associative scans, plus reverse adjoint scans].
 *   forward:  out_t = J_t out_{t-1} + b_t,        out_{-1} = c (h0, or 0)
 *   reverse:  out_t = b_t + J_{t+1}^T out_{t+1},  out_{T-1} = b_{T-1} + c
 * kind: diag J [B][T][N]; block2 J [B][T][N][2][2] with b [B][T][N][2];
 *       dense J [B][T][N][N] with b [B][T][N].
 * ---------------------------------------------------------------------------------- */
int orc_linear_scan(int kind, long B, long T, long N, const double *J, const double *bb,
                    const double *c0, double *out, int reverse)
{
    if (kind == ORC_SCAN_DENSE) {
#pragma omp parallel for schedule(dynamic, 1)
        for (long b = 0; b < B; ++b) {
            double *carry = calloc(N, sizeof(double));
            if (c0) memcpy(carry, c0 + b * N, sizeof(double) * N);
            for (long s = 0; s < T; ++s) {
                long t = reverse ? T - 1 - s : s;
                double *o = out + (b * T + t) * N;
                const double *bv = bb + (b * T + t) * N;
                for (long i = 0; i < N; ++i) {
                    double acc = bv[i];
                    if (!reverse) {
                        const double *Jt = J + (b * T + t) * N * N;
                        for (long j = 0; j < N; ++j) acc += Jt[i * N + j] * carry[j];
                    } else if (s == 0) {
                        acc += carry[i];
                    } else {
                        const double *Jn = J + (b * T + t + 1) * N * N;
                        for (long j = 0; j < N; ++j) acc += Jn[j * N + i] * carry[j];
                    }
                    o[i] = acc;
                }
                memcpy(carry, o, sizeof(double) * N);
            }
            free(carry);
        }
        return 0;
    }
    long E = (kind == ORC_SCAN_BLOCK2) ? 2 : 1;
#pragma omp parallel for schedule(static)
    for (long bn = 0; bn < B * N; ++bn) {
        long b = bn / N, n = bn % N;
        double carry[2] = {0.0, 0.0};
        if (c0)
            for (long e = 0; e < E; ++e) carry[e] = c0[(b * N + n) * E + e];
        for (long s = 0; s < T; ++s) {
            long t = reverse ? T - 1 - s : s;
            long vi = ((b * T + t) * N + n) * E;
            double o[2];
            if (!reverse) {
                const double *Jt = J + ((b * T + t) * N + n) * E * E;
                for (long i = 0; i < E; ++i) {
                    double acc = bb[vi + i];
                    for (long j = 0; j < E; ++j) acc += Jt[i * E + j] * carry[j];
                    o[i] = acc;
                }
            } else if (s == 0) {
                for (long i = 0; i < E; ++i) o[i] = bb[vi + i] + carry[i];
            } else {
                const double *Jn = J + ((b * T + t + 1) * N + n) * E * E;
                for (long i = 0; i < E; ++i) {
                    double acc = bb[vi + i];
                    for (long j = 0; j < E; ++j) acc += Jn[j * E + i] * carry[j];
                    o[i] = acc;
                }
            }
            for (long i = 0; i < E; ++i) {
                out[vi + i] = o[i];
                carry[i] = o[i];
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Adjoint backward at given states h [SEQ, Main features: "optional adjoint
 * backward"; DEER, Surprising findings: one linear solve for the gradient].
 * For L = sum_t <g_t, h_t>:  lambda_t = g_t + J_{t+1}^T lambda_{t+1}, lambda_T = g_T,
 * with every J evaluated at the given states.  Then
 *   grad_xproj_t = (df_t/dp_t)^T lambda_t,  grad_theta = sum_{b,t} (df_t/dtheta)^T lambda_t,
 *   grad_h0 = J_0^T lambda_0   (0-based time).
 * grad_params rows: GRU (a_z, a_r, a_c); LSTM (a_f, a_g, a_o, w_f, w_o).
 * GRU / LSTM only.
 * ---------------------------------------------------------------------------------- */
int orc_adjoint(const orc_model *m, const double *h0, const double *h, const double *g,
                double *grad_xproj, double *grad_params, double *grad_h0)
{
    if (m->cell == ORC_TANH) return -1;
    long B = m->B, T = m->T, H = m->H, S = state_per_unit(m);
    long NP = (m->cell == ORC_GRU) ? 3 : 5;
#pragma omp parallel for schedule(static)
    for (long u = 0; u < H; ++u) {
        double gp[5] = {0, 0, 0, 0, 0};
        for (long b = 0; b < B; ++b) {
            double mu[2] = {0.0, 0.0}; /* J_{t+1}^T lambda_{t+1} */
            for (long t = T - 1; t >= 0; --t) {
                double hp[2] = {0.0, 0.0};
                for (long s = 0; s < S; ++s)
                    hp[s] = t ? h[((b * T + t - 1) * H + u) * S + s]
                              : (h0 ? h0[(b * H + u) * S + s] : 0.0);
                double lam[2];
                for (long s = 0; s < S; ++s) lam[s] = g[((b * T + t) * H + u) * S + s] + mu[s];
                double f[2], J[4], dp[6], cn = 0.0;
                unit_eval(m, b, t, u, hp, f, J, dp, &cn);
                double gx[3];
                for (long q = 0; q < 3; ++q) {
                    double acc = 0.0;
                    for (long s = 0; s < S; ++s) acc += dp[s * 3 + q] * lam[s];
                    gx[q] = acc;
                    grad_xproj[((b * T + t) * 3 + q) * H + u] = acc;
                }
                if (m->cell == ORC_GRU) {
                    /* a_z, a_r enter as a h next to p_z, p_r; a_c as a_c (r h) next to p_c */
                    double r = sigm(m->xproj[((b * T + t) * 3 + 1) * H + u] + m->a[H + u] * hp[0]);
                    gp[0] += gx[0] * hp[0];
                    gp[1] += gx[1] * hp[0];
                    gp[2] += gx[2] * r * hp[0];
                } else {
                    /* a_f, a_g, a_o multiply h_{t-1}; w_f multiplies c_{t-1}; w_o the new c_t */
                    gp[0] += gx[0] * hp[1];
                    gp[1] += gx[1] * hp[1];
                    gp[2] += gx[2] * hp[1];
                    gp[3] += gx[0] * hp[0];
                    gp[4] += gx[2] * cn;
                }
                for (long j = 0; j < S; ++j) {
                    double acc = 0.0;
                    for (long i = 0; i < S; ++i) acc += J[i * S + j] * lam[i];
                    mu[j] = acc;
                }
            }
            for (long s = 0; s < S; ++s) grad_h0[(b * H + u) * S + s] = mu[s];
        }
        for (long q = 0; q < NP; ++q) grad_params[q * H + u] = gp[q];
    }
    return 0;
}

/* Final residual r = max over (b, t, state element) of |h_t - f(h_{t-1}, x_t)|. */
double orc_residual(const orc_model *m, const double *h0, const double *h)
{
    long B = m->B, T = m->T, H = m->H;
    double res = 0.0;
    if (m->cell == ORC_TANH) {
        long n = H;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : res)
        for (long b = 0; b < B; ++b) {
            double *J = malloc(sizeof(double) * n * n), *f = malloc(sizeof(double) * n);
            double *z0 = calloc(n, sizeof(double));
            double rl = 0.0;
            for (long t = 0; t < T; ++t) {
                const double *hp = t ? h + (b * T + t - 1) * n : (h0 ? h0 + b * n : z0);
                tanh_step(m, m->xproj + (b * T + t) * n, hp, f, J);
                for (long i = 0; i < n; ++i) rl = absmax_update(rl, h[(b * T + t) * n + i] - f[i]);
            }
            if (rl > res) res = rl;
            free(J);
            free(f);
            free(z0);
        }
        return res;
    }
    long S = state_per_unit(m);
#pragma omp parallel for schedule(static) reduction(max : res)
    for (long bu = 0; bu < B * H; ++bu) {
        long b = bu / H, u = bu % H;
        double rl = 0.0;
        for (long t = 0; t < T; ++t) {
            double hp[2] = {0.0, 0.0}, f[2], J[4];
            for (long s = 0; s < S; ++s)
                hp[s] = t ? h[((b * T + t - 1) * H + u) * S + s] : (h0 ? h0[(b * H + u) * S + s] : 0.0);
            unit_eval(m, b, t, u, hp, f, J, NULL, NULL);
            for (long s = 0; s < S; ++s) rl = absmax_update(rl, h[((b * T + t) * H + u) * S + s] - f[s]);
        }
        if (rl > res) res = rl;
    }
    return res;
}

/* ------------------------------------------------------------------ lsim
 * Fixed-step simulation of a linear time-invariant system, dx/dt = A x + B u,
 * y = C x + D u ("Para-Seq" README, Quick example and the `src.ode_solvers` row of
 * Main features: scan-based fixed-step linear simulation).  The continuous system
 * arrives already discretised over one step (Ad, G0, G1; see oracle/__init__.py):
 *   x_0 = x0 (zero when absent),
 *   x_k = Ad x_{k-1} + G0 u_{k-1} + G1 u_k      for k = 1 .. T-1,
 *   y_k = C x_k + D u_k                          for k = 0 .. T-1.
 * Plain sequential loop in time, OpenMP over the independent input sequences.
 * Layouts (row-major): Ad [n,n], G0 and G1 [n,m], C [p,n], D [p,m] or NULL,
 * U [B,T,m], x0 [B,n] or NULL, y [B,T,p], x [B,T,n] or NULL. */
void orc_lti_sim(long B, long T, int n, int m, int p, const double *Ad, const double *G0, const double *G1,
                 const double *C, const double *D, const double *U, const double *x0, double *y, double *x)
{
#pragma omp parallel for schedule(static)
    for (long b = 0; b < B; ++b) {
        double *cur = calloc((size_t)n, sizeof(double)), *nxt = calloc((size_t)n, sizeof(double));
        const double *ub = U + (size_t)b * T * m;
        if (x0)
            for (int i = 0; i < n; ++i) cur[i] = x0[(size_t)b * n + i];
        for (long k = 0; k < T; ++k) {
            const double *uk = ub + (size_t)k * m;
            if (k > 0) {
                const double *up = uk - m;
                for (int i = 0; i < n; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < n; ++j) acc += Ad[i * n + j] * cur[j];
                    for (int q = 0; q < m; ++q) acc += G0[i * m + q] * up[q] + G1[i * m + q] * uk[q];
                    nxt[i] = acc;
                }
                double *t = cur;
                cur = nxt;
                nxt = t;
            }
            for (int r = 0; r < p; ++r) {
                double acc = 0.0;
                for (int j = 0; j < n; ++j) acc += C[r * n + j] * cur[j];
                if (D)
                    for (int q = 0; q < m; ++q) acc += D[r * m + q] * uk[q];
                y[((size_t)b * T + k) * p + r] = acc;
            }
            if (x)
                for (int i = 0; i < n; ++i) x[((size_t)b * T + k) * n + i] = cur[i];
        }
        free(cur);
        free(nxt);
    }
}
