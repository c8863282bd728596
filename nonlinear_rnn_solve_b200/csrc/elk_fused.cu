// elk_fused.cu -- ELK and quasi-ELK for the ParaGRU and the ParaLSTM: the Newton
// iteration damped by Levenberg-Marquardt, with the damped step computed by parallel
// Kalman filtering and smoothing ("Towards Scalable and Stable Parallelization of
// Nonlinear RNNs", Abstract: ELK with the Jacobian, quasi-ELK with its diagonal;
// "Para-Seq" README, Main features: ELK and quasi-ELK).
//
// Per unit the state x_t has S components (GRU: 1; LSTM: (c, h) with the full 2x2
// Jacobian block, or its diagonal for quasi-ELK).  With J_t the step's Jacobian block,
// r_t = f_t - h^(k)_t and x = h^(k+1) - h^(k), the damped step minimises
//     sum_t |x_t - J_t x_{t-1} - r_t|^2 + lambda sum_t |x_t|^2      (x_{-1} = 0):
// the smoothed mean of x_t = J_t x_{t-1} + r_t + w_t, w ~ N(0, I), observed as 0 with
// noise covariance I / lambda.  Every iteration is two passes over the tiles:
//   F  (forward in time) the Kalman filter as one associative scan whose element
//      carries the conditional mean and covariance together (the parallel filter of
//      Sarkka and Garcia-Fernandez, "Temporal Parallelization of Bayesian Smoothers",
//      2021).  With g = 1 / (1 + lambda) and k = lambda g a step's element is
//      A = g J, b = g r, C = g I, eta = -k J^T r, Jn = k J^T J; the filtered (m, P)
//      after a prefix is its composition applied to (0, 0).  A tile publishes its
//      aggregate and the (m, P) after its last step (decoupled look-back).
//   S  (backward in time) each tile re-linearises, re-runs the filter inside the tile
//      from the (m, P) its predecessor published in F, forms the smoother's affine
//      maps x_t = G_t x_{t+1} + m_t - G_t (J_{t+1} m_t + r_{t+1}) with
//      G_t = P_t J_{t+1}^T (J_{t+1} P_t J_{t+1}^T + I)^{-1} (G = 0 at the sequence's
//      last step), scans them backward (look-back across the later tiles) and writes
//      h^(k+1) = h^(k) + x.
// Nothing per step goes through global memory between the passes: only the tiles'
// published values and each tile's first-step (J, r), which the gain of the step
// before the tile needs after the later tile has rewritten its states.
#include <string.h>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"
#include "newton_common.cuh"

namespace prn {
namespace {

// ---------------------------------------------------------------- S x S algebra (S = 1, 2)
template <int S> __device__ __forceinline__ void mat_mul(const float *X, const float *Y, float *R) {  // R = X Y
    if (S == 1) {
        R[0] = X[0] * Y[0];
    } else {
        const float r0 = fmaf(X[0], Y[0], X[1] * Y[2]), r1 = fmaf(X[0], Y[1], X[1] * Y[3]);
        const float r2 = fmaf(X[2], Y[0], X[3] * Y[2]), r3 = fmaf(X[2], Y[1], X[3] * Y[3]);
        R[0] = r0, R[1 % (S * S)] = r1, R[2 % (S * S)] = r2, R[3 % (S * S)] = r3;
    }
}
template <int S> __device__ __forceinline__ void mat_mul_t(const float *X, const float *Y, float *R) {  // R = X Y^T
    if (S == 1) {
        R[0] = X[0] * Y[0];
    } else {
        const float r0 = fmaf(X[0], Y[0], X[1] * Y[1]), r1 = fmaf(X[0], Y[2], X[1] * Y[3]);
        const float r2 = fmaf(X[2], Y[0], X[3] * Y[1]), r3 = fmaf(X[2], Y[2], X[3] * Y[3]);
        R[0] = r0, R[1 % (S * S)] = r1, R[2 % (S * S)] = r2, R[3 % (S * S)] = r3;
    }
}
template <int S> __device__ __forceinline__ void mat_tmul(const float *X, const float *Y, float *R) {  // R = X^T Y
    if (S == 1) {
        R[0] = X[0] * Y[0];
    } else {
        const float r0 = fmaf(X[0], Y[0], X[2] * Y[2]), r1 = fmaf(X[0], Y[1], X[2] * Y[3]);
        const float r2 = fmaf(X[1], Y[0], X[3] * Y[2]), r3 = fmaf(X[1], Y[1], X[3] * Y[3]);
        R[0] = r0, R[1 % (S * S)] = r1, R[2 % (S * S)] = r2, R[3 % (S * S)] = r3;
    }
}
template <int S> __device__ __forceinline__ void mat_vec(const float *X, const float *v, float *r) {  // r = X v
    if (S == 1) {
        r[0] = X[0] * v[0];
    } else {
        const float r0 = fmaf(X[0], v[0], X[1] * v[S - 1]), r1 = fmaf(X[2 % (S * S)], v[0], X[3 % (S * S)] * v[S - 1]);
        r[0] = r0, r[S - 1] = r1;
    }
}
template <int S> __device__ __forceinline__ void mat_tvec(const float *X, const float *v, float *r) {  // r = X^T v
    if (S == 1) {
        r[0] = X[0] * v[0];
    } else {
        const float r0 = fmaf(X[0], v[0], X[2 % (S * S)] * v[S - 1]), r1 = fmaf(X[1], v[0], X[3 % (S * S)] * v[S - 1]);
        r[0] = r0, r[S - 1] = r1;
    }
}
// R = X^{-1}, with the hardware reciprocal (a few ulp; the matrices inverted here are
// I + (positive semi-definite) x (positive semi-definite) products, far from singular)
template <int S> __device__ __forceinline__ void mat_inv(const float *X, float *R) {
    if (S == 1) {
        R[0] = rcp_hw(X[0]);
    } else {
        const float id = rcp_hw(fmaf(X[0], X[3 % (S * S)], -X[1] * X[2 % (S * S)]));
        const float r0 = X[3 % (S * S)] * id, r1 = -X[1] * id, r2 = -X[2 % (S * S)] * id, r3 = X[0] * id;
        R[0] = r0, R[1 % (S * S)] = r1, R[2 % (S * S)] = r2, R[3 % (S * S)] = r3;
    }
}
template <int S> __device__ __forceinline__ void add_ident(float *X, float s) {
    X[0] += s;
    if (S == 2) X[3 % (S * S)] += s;
}

// ---------------------------------------------------------------- filter element
// (A, b, C, eta, Jn) of a run of steps; composition o after i:
//   M = (I + C_i Jn_o)^{-1},  A = A_o M A_i,  b = A_o M (b_i + C_i eta_o) + b_o,
//   C = A_o M C_i A_o^T + C_o,  eta = (M A_i)^T (eta_o - Jn_o b_i) + eta_i,
//   Jn = (M A_i)^T Jn_o A_i + Jn_i.
// A constant (A = 0, Jn = 0) holds a known filtered state: b = m, C = P.  The carry of
// the scan is (m [S], P [S x S]).
template <int S> struct KElem {
    static constexpr int N = S * S;
    static constexpr int oA = 0, ob = N, oC = N + S, oe = 2 * N + S, oJ = 2 * N + 2 * S;
    static constexpr int kFloats = 3 * N + 2 * S;
    float v[kFloats];
    __device__ __forceinline__ static KElem zero() {
        KElem r;
#pragma unroll
        for (int q = 0; q < kFloats; ++q) r.v[q] = 0.f;
        return r;
    }
    __device__ __forceinline__ static KElem ident() {
        KElem r = zero();
        add_ident<S>(r.v + oA, 1.f);
        return r;
    }
    __device__ __forceinline__ static KElem cst(const float *x) {
        KElem r = zero();
#pragma unroll
        for (int q = 0; q < S; ++q) r.v[ob + q] = x[q];
#pragma unroll
        for (int q = 0; q < N; ++q) r.v[oC + q] = x[S + q];
        return r;
    }
    __device__ __forceinline__ void apply(const float *x, float *y) const;
    __device__ __forceinline__ KElem shfl_up(unsigned off) const {
        KElem r;
#pragma unroll
        for (int q = 0; q < kFloats; ++q) r.v[q] = __shfl_up_sync(0xffffffffu, v[q], off);
        return r;
    }
    __device__ __forceinline__ KElem shfl_down(unsigned off) const {
        KElem r;
#pragma unroll
        for (int q = 0; q < kFloats; ++q) r.v[q] = __shfl_down_sync(0xffffffffu, v[q], off);
        return r;
    }
    __device__ __forceinline__ void to_floats(float *f) const {
#pragma unroll
        for (int q = 0; q < kFloats; ++q) f[q] = v[q];
    }
    __device__ __forceinline__ static KElem from_floats(const float *f) {
        KElem r;
#pragma unroll
        for (int q = 0; q < kFloats; ++q) r.v[q] = f[q];
        return r;
    }
    __device__ __forceinline__ static bool const_floats(const float *f) {
        bool z = true;
#pragma unroll
        for (int q = 0; q < N; ++q) z = z && f[oA + q] == 0.f && f[oJ + q] == 0.f;
        return z;
    }
    __device__ __forceinline__ static void const_value(const float *f, float *x) {
#pragma unroll
        for (int q = 0; q < S; ++q) x[q] = f[ob + q];
#pragma unroll
        for (int q = 0; q < N; ++q) x[S + q] = f[oC + q];
    }
};

template <int S> __device__ __forceinline__ KElem<S> compose(const KElem<S> &i, const KElem<S> &o) {
    using K = KElem<S>;
    constexpr int N = S * S;
    float M[N], AM[N], MA[N], t[N];
    mat_mul<S>(i.v + K::oC, o.v + K::oJ, t);
    add_ident<S>(t, 1.f);
    mat_inv<S>(t, M);
    mat_mul<S>(o.v + K::oA, M, AM);
    mat_mul<S>(M, i.v + K::oA, MA);
    K r;
    mat_mul<S>(AM, i.v + K::oA, r.v + K::oA);
    float w[S], w2[S];
    mat_vec<S>(i.v + K::oC, o.v + K::oe, w);
#pragma unroll
    for (int q = 0; q < S; ++q) w[q] += i.v[K::ob + q];
    mat_vec<S>(AM, w, w2);
#pragma unroll
    for (int q = 0; q < S; ++q) r.v[K::ob + q] = w2[q] + o.v[K::ob + q];
    mat_mul<S>(AM, i.v + K::oC, t);
    mat_mul_t<S>(t, o.v + K::oA, r.v + K::oC);
#pragma unroll
    for (int q = 0; q < N; ++q) r.v[K::oC + q] += o.v[K::oC + q];
    mat_vec<S>(o.v + K::oJ, i.v + K::ob, w);
#pragma unroll
    for (int q = 0; q < S; ++q) w[q] = o.v[K::oe + q] - w[q];
    mat_tvec<S>(MA, w, w2);
#pragma unroll
    for (int q = 0; q < S; ++q) r.v[K::oe + q] = w2[q] + i.v[K::oe + q];
    mat_mul<S>(o.v + K::oJ, i.v + K::oA, t);
    mat_tmul<S>(MA, t, r.v + K::oJ);
#pragma unroll
    for (int q = 0; q < N; ++q) r.v[K::oJ + q] += i.v[K::oJ + q];
    return r;
}

template <int S> __device__ __forceinline__ void KElem<S>::apply(const float *x, float *y) const {
    const KElem r = compose(cst(x), *this);
    const_value(r.v, y);
}

// The element of one step from its Jacobian block J and residual r.
template <int S>
__device__ __forceinline__ KElem<S> step_elem(const float *J, const float *r, float g, float k) {
    using K = KElem<S>;
    K e;
#pragma unroll
    for (int q = 0; q < S * S; ++q) {
        e.v[K::oA + q] = g * J[q];
        e.v[K::oC + q] = 0.f;
    }
    add_ident<S>(e.v + K::oC, g);
#pragma unroll
    for (int q = 0; q < S; ++q) e.v[K::ob + q] = g * r[q];
    float w[S];
    mat_tvec<S>(J, r, w);
#pragma unroll
    for (int q = 0; q < S; ++q) e.v[K::oe + q] = -k * w[q];
    mat_tmul<S>(J, J, e.v + K::oJ);
#pragma unroll
    for (int q = 0; q < S * S; ++q) e.v[K::oJ + q] *= k;
    return e;
}

// One filter step from (m, P): Pm = J P J^T + I, mm = J m + r, W = (I + lambda Pm)^{-1},
// P <- W Pm, m <- W mm.
template <int S> __device__ __forceinline__ void filter_step(const float *J, const float *r, float lam, float *m,
                                                             float *P) {
    constexpr int N = S * S;
    float JP[N], Pm[N], t[N], W[N], mm[S];
    mat_mul<S>(J, P, JP);
    mat_mul_t<S>(JP, J, Pm);
    add_ident<S>(Pm, 1.f);
    mat_vec<S>(J, m, mm);
#pragma unroll
    for (int q = 0; q < S; ++q) mm[q] += r[q];
#pragma unroll
    for (int q = 0; q < N; ++q) t[q] = lam * Pm[q];
    add_ident<S>(t, 1.f);
    mat_inv<S>(t, W);
    mat_mul<S>(W, Pm, P);
    mat_vec<S>(W, mm, m);
}

// The smoother's affine map of step t from the filtered (m, P) at t and the next
// step's (J, r): G = P J^T (J P J^T + I)^{-1}, g = m - G (J m + r).
template <int S> __device__ __forceinline__ Aff<S> smoother_elem(const float *m, const float *P, const float *Jn,
                                                                 const float *rn) {
    constexpr int N = S * S;
    float JP[N], Pm[N], Pmi[N], PJt[N], G[N], mm[S], gm[S];
    mat_mul<S>(Jn, P, JP);
    mat_mul_t<S>(JP, Jn, Pm);
    add_ident<S>(Pm, 1.f);
    mat_inv<S>(Pm, Pmi);
    mat_mul_t<S>(P, Jn, PJt);
    mat_mul<S>(PJt, Pmi, G);
    mat_vec<S>(Jn, m, mm);
#pragma unroll
    for (int q = 0; q < S; ++q) mm[q] += rn[q];
    mat_vec<S>(G, mm, gm);
    float d[S];
#pragma unroll
    for (int q = 0; q < S; ++q) d[q] = m[q] - gm[q];
    return make_aff<S>(G, d);
}

struct ElkFArgs {
    NewtonDiagArgs A;  // A.agg / A.inc: pass F's look-back
    float lambda;
    unsigned long long *aggS, *incS;  // pass S's look-back
    float *firstJR;                   // [ntiles][C][S*S + S]: each tile's first step (J, r)
};

// Bounded read of a published word with this epoch (the pass that wrote it is behind a
// grid barrier, so it is normally there on the first poll).
__device__ __forceinline__ bool read_tagged(const unsigned long long *p, unsigned epoch, float *v,
                                            const NewtonDiagArgs &A) {
    unsigned long long t0 = 0;
    for (int polls = 0;; ++polls) {
        const unsigned long long w = ld_relaxed_u64(p);
        if ((unsigned)w == epoch) {
            *v = __uint_as_float((unsigned)(w >> 32));
            return true;
        }
        if (ld_relaxed_int(&A.ctl->abort)) return false;
        if (polls == 4) t0 = gtimer();
        if (polls > 4) {
            if (gtimer() - t0 > A.dbg.wait_ns) {
                raise_status(A.sticky, A.ctl, kStTimeout, true);
                return false;
            }
            __nanosleep(32);
        }
    }
}

// Linearise the L steps t0 .. t0 + L - 1 of unit u at h^(k) (k = 0: h^(0) = 0): J, r
// per step (J = I, r = 0 past the sequence or the units; the LSTM's block diagonal
// for quasi-ELK) and h^(k) of the steps in cur.
template <class Cell, int L, int IN>
__device__ __forceinline__ void linearise(const NewtonDiagArgs &A, const Cell &cell, const Proj<IN> &pj, int b, int u,
                                          bool uv, int t0, int k, float (*J)[Cell::S * Cell::S],
                                          float (*r)[Cell::S], float (*cur)[Cell::S]) {
    constexpr int S = Cell::S;
    float hp[S];
#pragma unroll
    for (int j = 0; j < S; ++j) hp[j] = 0.f;
    if (uv) {
        if (t0 == 0) {
            if (A.h0) load_state<S>(A.h0, (size_t)b * A.H + u, hp);
        } else if (k > 0 && t0 - 1 < A.T) {
            load_state<S>(A.h, ((size_t)b * A.T + (t0 - 1)) * A.H + u, hp);
        }
    }
#pragma unroll
    for (int i = 0; i < L; ++i) {
        const int t = t0 + i;
        const bool v = uv && t < A.T;
        float p[3], f[S], Jt[S * S];
#pragma unroll
        for (int j = 0; j < S; ++j) cur[i][j] = 0.f;
        if (k > 0 && v) load_state<S>(A.h, ((size_t)b * A.T + t) * A.H + u, cur[i]);
        pj.get(b, v ? t : 0, u, p);
        cell.eval(p, hp, f, Jt);
        apply_jmode<S>(A.jmode, Jt);
#pragma unroll
        for (int q = 0; q < S * S; ++q) J[i][q] = v ? Jt[q] : (q % (S + 1) == 0 ? 1.f : 0.f);
#pragma unroll
        for (int j = 0; j < S; ++j) {
            r[i][j] = v ? f[j] - cur[i][j] : 0.f;
            hp[j] = cur[i][j];
        }
    }
}

template <class Cell, int C, int L, int IN, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) elk_fused_kernel(const ElkFArgs E) {
    constexpr int S = Cell::S, N = S * S, SC = S + N, SUB = kThreads / C, TCH = SUB * L;
    using KE = KElem<S>;
    using AE = Aff<S>;
    const NewtonDiagArgs &A = E.A;
    __shared__ ScanSmem<SC, C, kThreads, KE> smk;
    __shared__ ScanSmem<S, C, kThreads, AE> sma;
    __shared__ float s_first[SUB][C][N + S];  // each thread's first step (J, r)
    __shared__ float s_swap[kThreads][AE::kFloats];
    __shared__ unsigned s_red[kThreads / 32];
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = (A.H + C - 1) / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    const float lam = E.lambda, g = 1.f / (1.f + lam), kk = lam * g;
    LookBack<SC> lbF{A.agg, A.inc};
    LookBack<S> lbS{E.aggS, E.incS};
    if (tid == 0) s_fail = 0;
    __syncthreads();

    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epF = A.epoch0 + 2u * (unsigned)k + 1u, epS = epF + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;

        // ---------------- pass F: the filter, forward in time
        {
            TileWalk tw(nseq);
            for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
                const int chunk = tw.chunk, b = tw.seq / nct;
                const int u = (tw.seq % nct) * C + c;
                const bool uv = u < A.H;
                const int t0 = chunk * TCH + s * L;
                Cell cell;
                cell.load(A.a, A.peep, A.H, uv ? u : 0);
                Proj<IN> pj;
                pj.load(A, uv ? u : 0);
                float J[L][N], r[L][S], cur[L][S];
                linearise<Cell, L, IN>(A, cell, pj, b, uv ? u : 0, uv, t0, k, J, r, cur);
                KE e = KE::ident();
#pragma unroll
                for (int i = 0; i < L; ++i)
                    if (uv && t0 + i < A.T) e = compose(e, step_elem<S>(J[i], r[i], g, kk));
                if (s == 0 && uv && t0 < A.T) {
                    float *fj = E.firstJR + ((size_t)tile * C + c) * (N + S);
#pragma unroll
                    for (int q = 0; q < N; ++q) fj[q] = J[0][q];
#pragma unroll
                    for (int q = 0; q < S; ++q) fj[N + q] = r[0][q];
                }
                KE excl, total;
                cta_scan<SC, C, kThreads, KE>(e, smk, excl, total);
                if (tid < 32) {
                    float base[SC];
#pragma unroll
                    for (int q = 0; q < SC; ++q) base[q] = 0.f;
                    if (!look_back<SC, C, kThreads, KE>(lbF, smk, total, tile, chunk, nseq, epF, base, A.ctl,
                                                         A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();
                if (s_fail) return;
            }
        }
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;

        // ---------------- pass S: the smoother, backward in time, and the update
        float my_max = 0.f;
        {
            TileWalk tw(nseq);
            for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
                const int chunk = tw.chunk;                 // scan order: descending time
                const int tc = nchunk - 1 - chunk;          // time chunk
                const int b = tw.seq / nct;
                const int u = (tw.seq % nct) * C + c;
                const bool uv = u < A.H;
                const int t0 = tc * TCH + s * L;           // thread s holds time sub-chunk s
                Cell cell;
                cell.load(A.a, A.peep, A.H, uv ? u : 0);
                Proj<IN> pj;
                pj.load(A, uv ? u : 0);
                float J[L][N], r[L][S], cur[L][S];
                linearise<Cell, L, IN>(A, cell, pj, b, uv ? u : 0, uv, t0, k, J, r, cur);
#pragma unroll
                for (int q = 0; q < N; ++q) s_first[s][c][q] = J[0][q];
#pragma unroll
                for (int q = 0; q < S; ++q) s_first[s][c][N + q] = r[0][q];
                // the filter inside the tile, from the state the preceding tile published
                KE e = KE::ident();
#pragma unroll
                for (int i = 0; i < L; ++i)
                    if (uv && t0 + i < A.T) e = compose(e, step_elem<S>(J[i], r[i], g, kk));
                KE fexcl, ftotal;
                cta_scan<SC, C, kThreads, KE>(e, smk, fexcl, ftotal);
                if (tid < C) {
                    if (tc == 0) {
#pragma unroll
                        for (int q = 0; q < SC; ++q) smk.carry[c][q] = 0.f;
                    } else {
                        const long ptile = (long)(tc - 1) * nseq + tw.seq;  // its index in pass F
#pragma unroll
                        for (int q = 0; q < SC; ++q) {
                            float v = 0.f;
                            if (!read_tagged(lbF.inc + (ptile * C + c) * SC + q, epF, &v, A)) s_fail = 1;
                            smk.carry[c][q] = v;
                        }
                    }
                }
                __syncthreads();
                if (s_fail) return;
                float mP[SC];
                fexcl.apply(smk.carry[c], mP);
                // the next step's (J, r) for this thread's last step
                float Jn[N], rn[S];
                bool have_next = t0 + L < A.T;
                if (s + 1 < SUB) {
#pragma unroll
                    for (int q = 0; q < N; ++q) Jn[q] = s_first[s + 1][c][q];
#pragma unroll
                    for (int q = 0; q < S; ++q) rn[q] = s_first[s + 1][c][N + q];
                } else if (have_next && uv) {
                    const float *fj = E.firstJR + (((size_t)(tc + 1) * nseq + tw.seq) * C + c) * (N + S);
#pragma unroll
                    for (int q = 0; q < N; ++q) Jn[q] = fj[q];
#pragma unroll
                    for (int q = 0; q < S; ++q) rn[q] = fj[N + q];
                } else {
#pragma unroll
                    for (int q = 0; q < N; ++q) Jn[q] = 0.f;
#pragma unroll
                    for (int q = 0; q < S; ++q) rn[q] = 0.f;
                }
                // filtered (m, P) step by step, each step's smoother map; J[i], r[i] become
                // the map's matrix and offset
#pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int t = t0 + i;
                    const bool v = uv && t < A.T;
                    filter_step<S>(J[i], r[i], lam, mP, mP + S);
                    AE m;
                    if (!v) {
                        m = AE::ident();
                    } else if (t + 1 >= A.T) {
                        float zero[N], mv[S];
#pragma unroll
                        for (int q = 0; q < N; ++q) zero[q] = 0.f;
#pragma unroll
                        for (int q = 0; q < S; ++q) mv[q] = mP[q];
                        m = make_aff<S>(zero, mv);
                    } else {
                        m = smoother_elem<S>(mP, mP + S, i + 1 < L ? J[(i + 1) % L] : Jn,
                                             i + 1 < L ? r[(i + 1) % L] : rn);
                    }
                    float mf[AE::kFloats];
                    m.to_floats(mf);
#pragma unroll
                    for (int q = 0; q < N; ++q) J[i][q] = mf[q];
#pragma unroll
                    for (int q = 0; q < S; ++q) r[i][q] = mf[N + q];
                }
                // this thread's maps composed in scan order (descending time)
                AE sagg = AE::ident();
#pragma unroll
                for (int i = L - 1; i >= 0; --i) sagg = compose(sagg, make_aff<S>(J[i], r[i]));
                // the scan runs in descending time: thread s's aggregate takes position
                // SUB - 1 - s, and the exclusive prefix returns the same way
                float af[AE::kFloats];
                sagg.to_floats(af);
#pragma unroll
                for (int q = 0; q < AE::kFloats; ++q) s_swap[(SUB - 1 - s) * C + c][q] = af[q];
                __syncthreads();
                AE mine = AE::from_floats(s_swap[tid]);
                AE sexcl, stotal;
                cta_scan<S, C, kThreads, AE>(mine, sma, sexcl, stotal);
                if (tid < 32) {
                    const float base[S] = {};
                    if (!look_back<S, C, kThreads, AE>(lbS, sma, stotal, tile, chunk, nseq, epS, base, A.ctl,
                                                       A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();  // the swap slots are read; the carry is in sma.carry
                if (s_fail) return;
                sexcl.to_floats(af);
#pragma unroll
                for (int q = 0; q < AE::kFloats; ++q) s_swap[tid][q] = af[q];
                __syncthreads();
                const AE ex = AE::from_floats(s_swap[(SUB - 1 - s) * C + c]);
                float x[S];
                ex.apply(sma.carry[c], x);  // x at the step after this thread's last
#pragma unroll
                for (int i = L - 1; i >= 0; --i) {
                    const int t = t0 + i;
                    make_aff<S>(J[i], r[i]).apply(x, x);
                    if (uv && t < A.T) {
                        float hn[S];
#pragma unroll
                        for (int j = 0; j < S; ++j) {
                            hn[j] = cur[i][j] + x[j];
                            const float ad = fabsf(x[j]);
                            my_max = (ad > my_max || isnan(x[j])) ? ad : my_max;
                        }
                        store_state<S>(A.h, ((size_t)b * A.T + t) * A.H + u, hn);
                    }
                }
                __syncthreads();  // s_first, s_swap and the scan buffers are reused
            }
        }
        const unsigned bits = block_max_bits(my_max, s_red);
        if (tid == 0) atomicMax(&A.ctl->delta_bits[k % 3], bits);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        const unsigned dbits = ld_acquire(&A.ctl->delta_bits[k % 3]);
        last_delta = __uint_as_float(dbits);
        iters = k + 1;
        if (blockIdx.x == 0 && tid == 0 && A.dbg.delta_log && k < A.dbg.delta_log_cap)
            A.dbg.delta_log[k] = last_delta;
        if (dbits >= 0x7f800000u) {
            if (blockIdx.x == 0 && tid == 0) atomicOr(A.sticky, kStNonfinite);
            stop_all = true;
            break;
        }
        if (last_delta < A.tol) break;
    }
    if (A.residual_out && !stop_all)
        if (!residual_pass<Cell, C, L, IN>(A, s_red)) return;
    if (blockIdx.x == 0 && tid == 0) {
        *A.iters_out = iters;
        if (A.delta_out) *A.delta_out = last_delta;
        if (!stop_all && A.tol > 0.f && iters == A.max_iters && !(last_delta < A.tol))
            atomicOr(A.sticky, kStNotConverged);
    }
}

int pick_units(int H) {
    if (H >= 32) return 32;
    int c = 1;
    while (c < H) c <<= 1;
    return c;
}

// Steps per thread: 8 (scalar state), 4 (2x2 blocks: the per-step maps stay in registers).
template <class Cell, int IN> const void *elk_fused_by_C(int C) {
    constexpr int L = Cell::S == 1 ? 8 : 4;
    constexpr int MINB = Cell::S == 1 ? 2 : 1;
    switch (C) {
        case 1: return reinterpret_cast<const void *>(&elk_fused_kernel<Cell, 1, L, IN, MINB>);
        case 2: return reinterpret_cast<const void *>(&elk_fused_kernel<Cell, 2, L, IN, MINB>);
        case 4: return reinterpret_cast<const void *>(&elk_fused_kernel<Cell, 4, L, IN, MINB>);
        case 8: return reinterpret_cast<const void *>(&elk_fused_kernel<Cell, 8, L, IN, MINB>);
        case 16: return reinterpret_cast<const void *>(&elk_fused_kernel<Cell, 16, L, IN, MINB>);
        default: return reinterpret_cast<const void *>(&elk_fused_kernel<Cell, 32, L, IN, MINB>);
    }
}

}  // namespace

// ELK on the ParaGRU and the ParaLSTM (jmode 0: the full 2x2 blocks; 1: their diagonal).
int elk_plan(const NewtonDiagReq &r, int num_sms, Plan *plan) {
    const int S = r.cell == 1 ? 2 : 1;
    const int C = pick_units(r.H);
    const bool fused = r.xproj == nullptr;
    const void *kern = S == 1 ? (fused ? elk_fused_by_C<GruCell, -1>(C) : elk_fused_by_C<GruCell, 0>(C))
                              : (fused ? elk_fused_by_C<LstmCell, -1>(C) : elk_fused_by_C<LstmCell, 0>(C));
    const int L = S == 1 ? 8 : 4;
    const int TCH = (kThreads / C) * L;
    const long nseq = (long)r.B * ((r.H + C - 1) / C);
    const int N = S * S, SC = S + N;
    plan->ntiles = nseq * ((r.T + TCH - 1) / TCH);
    if (plan->ntiles > 0x7fffffffL) return 1;
    plan->kernel = kern;
    plan->variant = C;
    plan->C = C;
    plan->S = S;
    plan->tch = TCH;
    plan->dyn_smem = 0;
    plan->threads = kThreads;
    plan->agg_words = (size_t)plan->ntiles * C * (3 * N + 2 * S);  // pass F: filter aggregates
    plan->inc_words = (size_t)plan->ntiles * C * SC;               // pass F: (m, P) after each tile
    // pass S's look-back (aggregates, inclusive values) and the tiles' first-step (J, r)
    plan->side_bytes = (size_t)plan->ntiles * C * ((S * S + S) + S) * sizeof(unsigned long long) +
                       (size_t)plan->ntiles * C * (N + S) * sizeof(float);
    plan->epochs = 2u * (unsigned)r.max_iters + 1u;
    plan->grid = occupancy_grid(plan->kernel, kThreads, 0, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t elk_launch(const NewtonDiagReq &r, float lambda, const Plan &plan, const Work &w, const DbgHost &dbg,
                       cudaStream_t st) {
    ElkFArgs E;
    memset(&E, 0, sizeof(E));
    NewtonDiagArgs &A = E.A;
    A.B = r.B;
    A.T = r.T;
    A.H = r.H;
    A.in = r.in;
    A.jmode = r.jmode;
    A.xproj = r.xproj;
    A.x = r.x;
    A.W = r.W;
    A.bias = r.bias;
    A.a = r.a;
    A.peep = r.peep;
    A.h0 = r.h0;
    A.h = r.h;
    A.max_iters = r.max_iters;
    A.tol = r.tol;
    A.iters_out = r.iters_out;
    A.delta_out = r.delta_out;
    A.residual_out = r.residual_out;
    A.ctl = w.ctl;
    A.sticky = w.sticky;
    A.agg = w.agg;
    A.inc = w.inc;
    A.side = nullptr;
    A.epoch0 = w.epoch0;
    A.dbg.wait_ns = dbg.wait_ns;
    A.dbg.skip_tile = dbg.skip_tile;
    A.dbg.delta_log = dbg.delta_log;
    A.dbg.delta_log_cap = dbg.delta_log_cap;
    A.dbg.no_halo = 1;
    const int S = plan.S, C = plan.C;
    const size_t nt = (size_t)plan.ntiles * C;
    E.lambda = lambda;
    E.aggS = reinterpret_cast<unsigned long long *>(w.side);
    E.incS = E.aggS + nt * (S * S + S);
    E.firstJR = reinterpret_cast<float *>(E.incS + nt * S);
    void *args[] = {&E};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(kThreads), args, 0, st);
}

}  // namespace prn
