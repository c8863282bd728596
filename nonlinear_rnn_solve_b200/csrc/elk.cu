// elk.cu -- ELK: the Newton iteration stabilised by Levenberg-Marquardt damping, with
// the damped step computed by parallel Kalman smoothing ("Towards Scalable and Stable
// Parallelization of Nonlinear RNNs", Abstract; "Para-Seq" README, Main features: ELK
// and quasi-ELK), for the diagonal linearisations: ParaGRU (its Jacobian is diagonal)
// the ParaLSTM with each 2x2 block reduced to its diagonal, and the dense tanh RNN with
// the diagonal of its Jacobian (quasi-ELK).
//
// Every state component is a scalar channel (LSTM: c and h of a unit are two channels).
// With a_t the diagonal Jacobian entry, r_t = f_t - h^(k)_t and x = h^(k+1) - h^(k), the
// damped step minimises sum_t (x_t - a_t x_{t-1} - r_t)^2 + lambda sum_t x_t^2 (x_0 = 0):
// the smoothed mean of x_t = a_t x_{t-1} + r_t + w_t, w ~ N(0, 1), observed as 0 with
// noise variance 1/lambda.  One persistent cooperative kernel runs every iteration in
// three scan phases separated by grid barriers:
//   A  filter variance: P_t = (a_t^2 P + 1) / (lambda (a_t^2 P + 1) + 1), a Moebius map
//      of P_{t-1}; as the projective vector (u, v), P = u / v, it is the linear map
//      M_t = [[a^2, 1], [lambda a^2, lambda + 1]]: a 2x2 scan from (0, 1) whose
//      compositions are rescaled (PAff2);
//   B  filter mean: m_t = (1 - K_t)(a_t m_{t-1} + r_t), K_t = lambda Pm_t / (1 + lambda
//      Pm_t), Pm_t = a_t^2 P_{t-1} + 1: a diagonal affine scan from 0;
//   C  smoother (reverse in time): s_t = G_t s_{t+1} + m_t - G_t (a_{t+1} m_t + r_{t+1}),
//      G_t = P_t a_{t+1} / Pm_{t+1}, s_{T-1} = m_{T-1}; then h^(k+1)_t = h^(k)_t + s_t.
// Each phase is the chunked scan of the Newton kernels (thread-serial, warp shuffles,
// shared memory, decoupled look-back) with its own epoch; a_t, r_t, P_t and m_t pass
// between phases through a scratch buffer.
#include <string.h>

#include <algorithm>
#include <type_traits>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"
#include "newton_common.cuh"

namespace prn {

// A 2x2 linear map, or a constant (offset only), acting on projective vectors (u, v)
// that stand for P = u / v: every composition and image is rescaled so its largest
// entry is 1, which leaves the represented ratio unchanged and keeps products of many
// steps in range (an unscaled product of the per-step maps decays geometrically).
// Scan compositions only ever combine linear maps with each other or with constants,
// so the rescaling is always exact projectively.
struct PAff2 {
    float a00, a01, a10, a11, d0, d1;
    static constexpr int kFloats = 6;
    __device__ __forceinline__ static PAff2 ident() { return {1.f, 0.f, 0.f, 1.f, 0.f, 0.f}; }
    __device__ __forceinline__ static PAff2 cst(const float *v) { return {0.f, 0.f, 0.f, 0.f, v[0], v[1]}; }
    __device__ __forceinline__ void apply(const float *x, float *y) const {
        float y0 = fmaf(a00, x[0], fmaf(a01, x[1], d0));
        float y1 = fmaf(a10, x[0], fmaf(a11, x[1], d1));
        const float mx = fmaxf(fabsf(y0), fabsf(y1));
        if (mx > 0.f && mx < 3.0e38f) {
            y0 /= mx;
            y1 /= mx;
        }
        y[0] = y0;
        y[1] = y1;
    }
    __device__ __forceinline__ PAff2 shfl_up(unsigned off) const {
        const unsigned m = 0xffffffffu;
        return {__shfl_up_sync(m, a00, off), __shfl_up_sync(m, a01, off), __shfl_up_sync(m, a10, off),
                __shfl_up_sync(m, a11, off), __shfl_up_sync(m, d0, off),  __shfl_up_sync(m, d1, off)};
    }
    __device__ __forceinline__ PAff2 shfl_down(unsigned off) const {
        const unsigned m = 0xffffffffu;
        return {__shfl_down_sync(m, a00, off), __shfl_down_sync(m, a01, off), __shfl_down_sync(m, a10, off),
                __shfl_down_sync(m, a11, off), __shfl_down_sync(m, d0, off),  __shfl_down_sync(m, d1, off)};
    }
    __device__ __forceinline__ void to_floats(float *v) const {
        v[0] = a00; v[1] = a01; v[2] = a10; v[3] = a11; v[4] = d0; v[5] = d1;
    }
    __device__ __forceinline__ static PAff2 from_floats(const float *v) { return {v[0], v[1], v[2], v[3], v[4], v[5]}; }
    __device__ __forceinline__ static bool const_floats(const float *v) {
        return v[0] == 0.f && v[1] == 0.f && v[2] == 0.f && v[3] == 0.f;
    }
    __device__ __forceinline__ static void const_value(const float *v, float *x) {
        x[0] = v[4];
        x[1] = v[5];
    }
};
__device__ __forceinline__ PAff2 compose(const PAff2 &i, const PAff2 &o) {
    PAff2 r;
    r.a00 = fmaf(o.a00, i.a00, o.a01 * i.a10);
    r.a01 = fmaf(o.a00, i.a01, o.a01 * i.a11);
    r.a10 = fmaf(o.a10, i.a00, o.a11 * i.a10);
    r.a11 = fmaf(o.a10, i.a01, o.a11 * i.a11);
    r.d0 = fmaf(o.a00, i.d0, fmaf(o.a01, i.d1, o.d0));
    r.d1 = fmaf(o.a10, i.d0, fmaf(o.a11, i.d1, o.d1));
    const float mx = fmaxf(fmaxf(fmaxf(fabsf(r.a00), fabsf(r.a01)), fmaxf(fabsf(r.a10), fabsf(r.a11))),
                           fmaxf(fabsf(r.d0), fabsf(r.d1)));
    if (mx > 0.f && mx < 3.0e38f) {
        const float s = 1.f / mx;
        r.a00 *= s;
        r.a01 *= s;
        r.a10 *= s;
        r.a11 *= s;
        r.d0 *= s;
        r.d1 *= s;
    }
    return r;
}

struct ElkArgs {
    NewtonDiagArgs A;
    float lambda;
    float *sa, *sr, *sP, *sm;  // [B, T, D] scratch, D = H * S
    const float *Amat;         // tanh RNN: recurrent matrix [n, n] (A.H = n)
};

// Cell tag of the dense tanh RNN, h_t = tanh(A h_{t-1} + p_t): its linearisation (the
// Jacobian's diagonal (1 - f^2) A_ii and r = f - h^(k)) needs the whole state row, so
// a pass over rows writes a and r to the scratch before the scans read them.
struct TanhLin {
    static constexpr int S = 1;
};
constexpr int kElkMaxN = 64;

// The tanh RNN at the iterate in h (k = 0: h^(0) = 0): per row (b, t) and unit i,
// f = tanh(p_t + sum_j A_ij h_{t-1,j}); writes a = (1 - f^2) A_ii and r = f - h_t, or
// (residual) folds |h_t - f| into my_max.  sAt: A transposed in shared memory with
// rows padded to n4 = n rounded up to a multiple of 4 (zeros beyond n).  A thread
// takes four consecutive units of one row: per j one 16-byte load of A's column
// entries and one (four-j) state load feed four multiply-adds.
// IN = 0: p from xproj [B, T, n]; IN = -1: p = bias + W x_t (W [n, in], in <= 8).
template <int IN>
__device__ void tanh_lin_pass(const ElkArgs &E, const float *sAt, int n4, int k, bool residual, float &my_max) {
    const NewtonDiagArgs &A = E.A;
    const int n = A.H;
    const int tpr = n4 / 4, rpc = kThreads / tpr;  // threads per row, rows per CTA and pass
    const int lr = threadIdx.x / tpr, i0 = (threadIdx.x - lr * tpr) * 4;
    const long nrows = (long)A.B * A.T;
    const bool have_h = k > 0 || residual;
    for (long row0 = (long)blockIdx.x * rpc; row0 < nrows; row0 += (long)gridDim.x * rpc) {
        const long row = row0 + lr;
        if (lr >= rpc || row >= nrows) continue;
        const long b = row / A.T, t = row - b * A.T;
        const float *hp = t == 0 ? (A.h0 ? A.h0 + b * n : nullptr) : (have_h ? A.h + (row - 1) * n : nullptr);
        float z[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            z[u] = 0.f;
            if (i < n) {
                if (IN == 0) {
                    z[u] = A.xproj[row * n + i];
                } else {
                    z[u] = A.bias ? A.bias[i] : 0.f;
                    for (int q = 0; q < A.in; ++q) z[u] = fmaf(A.W[(size_t)i * A.in + q], A.x[row * A.in + q], z[u]);
                }
            }
        }
        if (hp) {
            auto col = [&](int j, float hj) {
                const float4 a4 = *reinterpret_cast<const float4 *>(sAt + j * n4 + i0);
                z[0] = fmaf(a4.x, hj, z[0]);
                z[1] = fmaf(a4.y, hj, z[1]);
                z[2] = fmaf(a4.z, hj, z[2]);
                z[3] = fmaf(a4.w, hj, z[3]);
            };
            if (n % 4 == 0) {  // rows of h start on 16 bytes (h, h0 16-byte aligned)
                for (int j = 0; j < n; j += 4) {
                    const float4 h4 = *reinterpret_cast<const float4 *>(hp + j);
                    col(j, h4.x);
                    col(j + 1, h4.y);
                    col(j + 2, h4.z);
                    col(j + 3, h4.w);
                }
            } else {
                for (int j = 0; j < n; ++j) col(j, hp[j]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            if (i >= n) break;
            const float f = tanhf(z[u]);
            const float cur = have_h ? A.h[row * n + i] : 0.f;
            if (residual) {
                const float ad = fabsf(cur - f);
                my_max = (ad > my_max || isnan(ad)) ? ad : my_max;
            } else {
                E.sa[row * n + i] = (1.f - f * f) * sAt[i * n4 + i];
                E.sr[row * n + i] = f - cur;
            }
        }
    }
}

template <class Cell, int C, int L, int IN>
__global__ void __launch_bounds__(kThreads, 2) elk_kernel(const ElkArgs E) {
    const NewtonDiagArgs &A = E.A;
    constexpr int S = Cell::S;
    constexpr int SUB = kThreads / C, TCH = SUB * L;
    constexpr bool kTanh = std::is_same<Cell, TanhLin>::value;
    __shared__ __align__(16) float s_At[kTanh ? kElkMaxN * kElkMaxN : 4];
    const int n4 = (A.H + 3) & ~3;  // tanh: padded row length of s_At
    __shared__ ScanSmem<2, C, kThreads, PAff2> sm2;
    __shared__ ScanSmem<1, C> sm1;
    __shared__ unsigned s_red[kThreads / 32];
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int D = A.H * S;
    const int nct = (D + C - 1) / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    const float lam = E.lambda;
    LookBack<2> lb2{A.agg, A.inc};
    LookBack<1> lb1{A.agg, A.inc};
    if (tid == 0) s_fail = 0;
    if (kTanh)
        for (int e = tid; e < n4 * n4; e += kThreads) {
            const int j = e / n4, i = e % n4;  // s_At[j][i] = A[i][j]
            s_At[e] = (i < A.H && j < A.H) ? E.Amat[i * A.H + j] : 0.f;
        }
    __syncthreads();

    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned ep = A.epoch0 + 3u * (unsigned)k;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        if constexpr (kTanh) {  // linearise the whole iterate first
            float unused = 0.f;
            tanh_lin_pass<IN>(E, s_At, n4, k, false, unused);
            if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        }

        // ---------------- phase A: linearise, filter variance
        {
            TileWalk tw(nseq);
            for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
                const int chunk = tw.chunk, b = tw.seq / nct;
                const int ch = (tw.seq % nct) * C + c;  // channel: unit ch / S, component ch % S
                const bool cv = ch < D;
                const int u = cv ? ch / S : 0, q = cv ? ch % S : 0;
                const int t0 = chunk * TCH + s * L;
                float av[L];
                PAff2 e = PAff2::ident();
                if constexpr (kTanh) {  // a_t from the linearisation pass
#pragma unroll
                    for (int i = 0; i < L; ++i) {
                        const int t = t0 + i;
                        const bool v = cv && t < A.T;
                        const float aq = v ? E.sa[((size_t)b * A.T + t) * D + ch] : 0.f;
                        av[i] = aq;
                        const float a2 = aq * aq;
                        e = compose(e, v ? PAff2{a2, 1.f, lam * a2, lam + 1.f, 0.f, 0.f} : PAff2::ident());
                    }
                } else {
                    Cell cell;
                    cell.load(A.a, A.peep, A.H, u);
                    Proj<IN> pj;
                    pj.load(A, u);
                    float hp[S];
#pragma unroll
                    for (int j = 0; j < S; ++j) hp[j] = 0.f;
                    if (t0 == 0) {
                        if (A.h0) load_state<S>(A.h0, (size_t)b * A.H + u, hp);
                    } else if (k > 0 && t0 - 1 < A.T) {
                        load_state<S>(A.h, ((size_t)b * A.T + (t0 - 1)) * A.H + u, hp);
                    }
#pragma unroll
                    for (int i = 0; i < L; ++i) {
                        const int t = t0 + i;
                        const bool v = cv && t < A.T;
                        float p[3], cur[S], f[S], J[S * S];
                        pj.get(b, v ? t : 0, u, p);
#pragma unroll
                        for (int j = 0; j < S; ++j) cur[j] = 0.f;
                        if (k > 0 && v) load_state<S>(A.h, ((size_t)b * A.T + t) * A.H + u, cur);
                        cell.eval(p, hp, f, J);
                        float fq = f[0], cq = cur[0], aq = J[0];
#pragma unroll
                        for (int j = 1; j < S; ++j)
                            if (q == j) {
                                fq = f[j];
                                cq = cur[j];
                                aq = J[j * S + j];
                            }
#pragma unroll
                        for (int j = 0; j < S; ++j) hp[j] = cur[j];
                        av[i] = v ? aq : 0.f;
                        if (v) {
                            const size_t o = ((size_t)b * A.T + t) * D + ch;
                            E.sa[o] = aq;
                            E.sr[o] = fq - cq;
                        }
                        // M_t (identity outside the sequence)
                        const float a2 = aq * aq;
                        e = compose(e, v ? PAff2{a2, 1.f, lam * a2, lam + 1.f, 0.f, 0.f} : PAff2::ident());
                    }
                }
                PAff2 excl, total;
                cta_scan<2, C, kThreads, PAff2>(e, sm2, excl, total);
                if (tid < 32) {
                    const float base[2] = {0.f, 1.f};  // P = 0 before the first step
                    if (!look_back<2, C, kThreads, PAff2>(lb2, sm2, total, tile, chunk, nseq, ep + 1u, base, A.ctl,
                                                          A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();
                if (s_fail) return;
                float uv[2];
                excl.apply(sm2.carry[c], uv);
#pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int t = t0 + i;
                    if (!(cv && t < A.T)) continue;
                    const float a2 = av[i] * av[i];
                    const float nu = fmaf(a2, uv[0], uv[1]), nv = fmaf(lam * a2, uv[0], (lam + 1.f) * uv[1]);
                    const float mx = fmaxf(fabsf(nu), fabsf(nv));
                    uv[0] = nu / mx;
                    uv[1] = nv / mx;
                    E.sP[((size_t)b * A.T + t) * D + ch] = nu / nv;
                }
                __syncthreads();
            }
        }
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;

        // ---------------- phase B: filter mean
        {
            TileWalk tw(nseq);
            for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
                const int chunk = tw.chunk, b = tw.seq / nct;
                const int ch = (tw.seq % nct) * C + c;
                const bool cv = ch < D;
                const int t0 = chunk * TCH + s * L;
                float Pprev = (cv && t0 > 0 && t0 - 1 < A.T) ? E.sP[((size_t)b * A.T + t0 - 1) * D + ch] : 0.f;
                float cr[L], dr[L];
                Aff<1> e = Aff<1>::ident();
#pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int t = t0 + i;
                    const bool v = cv && t < A.T;
                    cr[i] = 1.f;
                    dr[i] = 0.f;
                    if (v) {
                        const size_t o = ((size_t)b * A.T + t) * D + ch;
                        const float a = E.sa[o], r = E.sr[o];
                        const float Pm = fmaf(a * a, Pprev, 1.f);
                        const float omk = 1.f / (1.f + lam * Pm);  // 1 - K
                        cr[i] = omk * a;
                        dr[i] = omk * r;
                        Pprev = E.sP[o];
                    }
                    e = compose(e, Aff<1>{cr[i], dr[i]});
                }
                Aff<1> excl, total;
                cta_scan<1, C>(e, sm1, excl, total);
                if (tid < 32) {
                    const float base[1] = {0.f};
                    if (!look_back<1, C>(lb1, sm1, total, tile, chunk, nseq, ep + 2u, base, A.ctl, A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();
                if (s_fail) return;
                float m;
                excl.apply(sm1.carry[c], &m);
#pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int t = t0 + i;
                    m = fmaf(cr[i], m, dr[i]);
                    if (cv && t < A.T) E.sm[((size_t)b * A.T + t) * D + ch] = m;
                }
                __syncthreads();
            }
        }
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;

        // ---------------- phase C: smoother (scan order = descending time), update
        float my_max = 0.f;
        {
            TileWalk tw(nseq);
            for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
                const int chunk = tw.chunk, b = tw.seq / nct;
                const int ch = (tw.seq % nct) * C + c;
                const bool cv = ch < D;
                const int u = cv ? ch / S : 0, q = cv ? ch % S : 0;
                const int tbase = (nchunk - 1 - chunk) * TCH + (SUB - 1 - s) * L;  // earliest step of the thread
                float gr[L], br[L];
                Aff<1> e = Aff<1>::ident();
#pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int t = tbase + (L - 1 - i);  // scan step i is time t
                    const bool v = cv && t < A.T;
                    gr[i] = 1.f;
                    br[i] = 0.f;
                    if (v) {
                        const size_t o = ((size_t)b * A.T + t) * D + ch;
                        const float P = E.sP[o], mt = E.sm[o];
                        if (t + 1 < A.T) {
                            const size_t o1 = o + D;
                            const float a1 = E.sa[o1], r1 = E.sr[o1];
                            const float G = P * a1 / fmaf(a1 * a1, P, 1.f);
                            gr[i] = G;
                            br[i] = mt - G * fmaf(a1, mt, r1);
                        } else {
                            gr[i] = 0.f;  // s_{T-1} = m_{T-1}
                            br[i] = mt;
                        }
                    }
                    e = compose(e, Aff<1>{gr[i], br[i]});
                }
                Aff<1> excl, total;
                cta_scan<1, C>(e, sm1, excl, total);
                if (tid < 32) {
                    const float base[1] = {0.f};
                    if (!look_back<1, C>(lb1, sm1, total, tile, chunk, nseq, ep + 3u, base, A.ctl, A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();
                if (s_fail) return;
                float sv;
                excl.apply(sm1.carry[c], &sv);
#pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int t = tbase + (L - 1 - i);
                    sv = fmaf(gr[i], sv, br[i]);
                    if (cv && t < A.T) {
                        float* hq = A.h + (((size_t)b * A.T + t) * A.H + u) * S + q;
                        const float cur = k > 0 ? *hq : 0.f;
                        *hq = cur + sv;
                        const float ad = fabsf(sv);
                        my_max = (ad > my_max || isnan(sv)) ? ad : my_max;
                    }
                }
                __syncthreads();
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
    if (A.residual_out && !stop_all) {
        if constexpr (kTanh) {
            float my_res = 0.f;
            tanh_lin_pass<IN>(E, s_At, n4, 1, true, my_res);
            const unsigned bits = block_max_bits(my_res, s_red);
            if (tid == 0) atomicMax(&A.ctl->res_bits, bits);
            if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
            if (blockIdx.x == 0 && tid == 0) {
                const unsigned rb = ld_acquire(&A.ctl->res_bits);
                *A.residual_out = __uint_as_float(rb);
                if (rb >= 0x7f800000u) atomicOr(A.sticky, kStNonfinite);
            }
        } else {
            if (!residual_pass<Cell, C, L, IN>(A, s_red)) return;
        }
    }
    if (blockIdx.x == 0 && tid == 0) {
        *A.iters_out = iters;
        if (A.delta_out) *A.delta_out = last_delta;
        if (!stop_all && A.tol > 0.f && iters == A.max_iters && !(last_delta < A.tol))
            atomicOr(A.sticky, kStNotConverged);
    }
}

namespace {

int pick_C(int D) {
    if (D >= 32) return 32;
    int c = 1;
    while (c < D) c <<= 1;
    return c;
}

// Steps per thread: 16 for tiles of 32 channels (wide states: a 64-step tile would
// spend most of its time in the look-back), 8 for narrower ones (long sequences of
// few channels, where 8 measured faster).
constexpr int kElkL = 8, kElkLWide = 16;
int elk_L(int C) { return C == 32 ? kElkLWide : kElkL; }

template <class Cell, int IN> const void *elk_by_C(int C) {
    switch (C) {
        case 1: return reinterpret_cast<const void *>(&elk_kernel<Cell, 1, kElkL, IN>);
        case 2: return reinterpret_cast<const void *>(&elk_kernel<Cell, 2, kElkL, IN>);
        case 4: return reinterpret_cast<const void *>(&elk_kernel<Cell, 4, kElkL, IN>);
        case 8: return reinterpret_cast<const void *>(&elk_kernel<Cell, 8, kElkL, IN>);
        case 16: return reinterpret_cast<const void *>(&elk_kernel<Cell, 16, kElkL, IN>);
        default: return reinterpret_cast<const void *>(&elk_kernel<Cell, 32, kElkLWide, IN>);
    }
}

}  // namespace

namespace {

// Tiles, workspace and grid of an ELK solve over D scalar channels per sequence.
int elk_plan_common(const void *kernel, long B, long T, int D, int C, int max_iters, int num_sms, Plan *plan) {
    const int TCH = (kThreads / C) * elk_L(C);
    const long nseq = B * ((D + C - 1) / C);
    plan->ntiles = nseq * ((T + TCH - 1) / TCH);
    plan->kernel = kernel;
    plan->variant = C;
    plan->C = C;
    plan->dyn_smem = 0;
    plan->agg_words = (size_t)plan->ntiles * C * 6;  // phase A: 2x2 blocks; B, C reuse them
    plan->inc_words = (size_t)plan->ntiles * C * 2;
    plan->side_bytes = 4 * (size_t)B * T * D * sizeof(float);  // a, r, P, m
    plan->epochs = 3u * (unsigned)max_iters + 1u;
    plan->grid = occupancy_grid(plan->kernel, kThreads, 0, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t elk_launch_common(ElkArgs &E, long D, float lambda, const Plan &plan, const Work &w, const DbgHost &dbg,
                              cudaStream_t st) {
    NewtonDiagArgs &A = E.A;
    A.ctl = w.ctl;
    A.sticky = w.sticky;
    A.agg = w.agg;
    A.inc = w.inc;
    A.side = w.side;
    A.epoch0 = w.epoch0;
    A.dbg.wait_ns = dbg.wait_ns;
    A.dbg.skip_tile = dbg.skip_tile;
    A.dbg.delta_log = dbg.delta_log;
    A.dbg.delta_log_cap = dbg.delta_log_cap;
    A.dbg.no_halo = 1;
    const size_t n = (size_t)A.B * A.T * D;
    E.lambda = lambda;
    E.sa = w.side;
    E.sr = w.side + n;
    E.sP = w.side + 2 * n;
    E.sm = w.side + 3 * n;
    void *args[] = {&E};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(kThreads), args, 0, st);
}

}  // namespace

int elk_tanh_plan(const NewtonTanhReq &r, int num_sms, Plan *plan) {
    if (r.n > kElkMaxN) return 1;
    const int C = pick_C(r.n);
    const void *k = r.xproj ? elk_by_C<TanhLin, 0>(C) : elk_by_C<TanhLin, -1>(C);
    return elk_plan_common(k, r.B, r.T, r.n, C, r.max_iters, num_sms, plan);
}

cudaError_t elk_tanh_launch(const NewtonTanhReq &r, float lambda, const Plan &plan, const Work &w,
                            const DbgHost &dbg, cudaStream_t st) {
    ElkArgs E;
    memset(&E, 0, sizeof(E));
    NewtonDiagArgs &A = E.A;
    A.B = r.B;
    A.T = r.T;
    A.H = r.n;
    A.in = r.in;
    A.xproj = r.xproj;
    A.x = r.x;
    A.W = r.W;
    A.bias = r.bias;
    A.h0 = r.h0;
    A.h = r.h;
    A.max_iters = r.max_iters;
    A.tol = r.tol;
    A.iters_out = r.iters_out;
    A.delta_out = r.delta_out;
    A.residual_out = r.residual_out;
    E.Amat = r.A;
    return elk_launch_common(E, r.n, lambda, plan, w, dbg, st);
}

}  // namespace prn
