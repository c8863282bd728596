// adjoint.cu -- adjoint backward of the Newton-solved recurrence for ParaGRU and
// ParaLSTM ("Para-Seq" README, Main features: optional adjoint backward, reverse
// adjoint scans; DEER summary, Surprising findings: the gradient needs one linear
// solve, no backpropagation through the Newton iterations).
//
// For L = sum_t <g_t, h_t>, with every Jacobian evaluated at the given states,
//   lambda_t = g_t + mu_{t+1},   mu_t = J_t^T lambda_t,   mu_T = 0,
// so mu obeys the reverse linear recurrence mu_t = J_t^T mu_{t+1} + J_t^T g_t: one
// reverse scan.  The epilogue forms grad_xproj_t = (df_t/dp_t)^T lambda_t, reduces
// the recurrent-parameter gradients and writes grad_h0 = mu_0.
#include "cells.cuh"
#include "common.cuh"
#include "internal.h"

namespace prn {

struct AdjArgs {
    int B, T, H;
    const float *xproj, *a, *peep, *h0, *h, *g;
    float *gx, *gp, *gh0;
    Ctl *ctl;
    int *sticky;
    unsigned long long *agg, *inc;
    unsigned epoch0;
    Dbg dbg;
};

template <int S>
__device__ __forceinline__ void ld_state(const float *p, size_t idx, float *v) {
    if (S == 1) {
        v[0] = p[idx];
    } else {
        float2 u = *reinterpret_cast<const float2 *>(p + idx * 2);
        v[0] = u.x;
        v[S - 1] = u.y;
    }
}

template <class Cell, int C, int L>
__global__ void __launch_bounds__(kThreads, 2) adjoint_kernel(const AdjArgs A) {
    constexpr int S = Cell::S;
    constexpr int NF = S == 1 ? 2 : 3;   // parameter factors per step
    constexpr int NP = Cell::NPAR;
    constexpr int SUB = kThreads / C;
    constexpr int TCH = SUB * L;
    __shared__ ScanSmem<S, C> sm;
    __shared__ float s_gp[kThreads][NP];
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = (A.H + C - 1) / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    LookBack<S> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;
    TileWalk tw(nseq);
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
        const int chunk = tw.chunk;  // scan order: from the end of time
        const int seq = tw.seq;
        const int b = seq / nct;
        const int h = (seq % nct) * C + c;
        const bool cv = h < A.H;
        const int hh = cv ? h : 0;
        const int tbase = (nchunk - 1 - chunk) * TCH + (SUB - 1 - s) * L;
        Cell cell;
        cell.load(A.a, A.peep, A.H, hh);
        float Jm[L][S * S], gg[L][S], dp[L][3 * S], fac[L][NF];
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = tbase + (L - 1 - i);  // scan step i is time t (descending)
            const bool v = cv && t < A.T;
            const int tt = v ? t : 0;
            float p[3], hp[S];
            const float *q = A.xproj + ((size_t)b * A.T + tt) * 3 * A.H + hh;
            p[0] = q[0];
            p[1] = q[A.H];
            p[2] = q[2 * A.H];
#pragma unroll
            for (int k = 0; k < S; ++k) hp[k] = 0.f;
            if (tt == 0) {
                if (A.h0) ld_state<S>(A.h0, (size_t)b * A.H + hh, hp);
            } else {
                ld_state<S>(A.h, ((size_t)b * A.T + tt - 1) * A.H + hh, hp);
            }
            float gv[S];
            ld_state<S>(A.g, ((size_t)b * A.T + tt) * A.H + hh, gv);
            cell.partials(p, hp, Jm[i], dp[i], fac[i]);
#pragma unroll
            for (int k = 0; k < S; ++k) gg[i][k] = v ? gv[k] : 0.f;
            if (!v) {
#pragma unroll
                for (int k = 0; k < S * S; ++k) Jm[i][k] = (k % (S + 1)) == 0 ? 1.f : 0.f;
#pragma unroll
                for (int k = 0; k < 3 * S; ++k) dp[i][k] = 0.f;
#pragma unroll
                for (int k = 0; k < NF; ++k) fac[i][k] = 0.f;
            }
        }
        // element of scan step i: x -> J^T x + J^T g
        Aff<S> e = Aff<S>::ident();
#pragma unroll
        for (int i = 0; i < L; ++i) {
            float Mt[S * S], d[S];
#pragma unroll
            for (int r = 0; r < S; ++r)
#pragma unroll
                for (int k = 0; k < S; ++k) Mt[r * S + k] = Jm[i][k * S + r];
#pragma unroll
            for (int r = 0; r < S; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < S; ++k) acc = fmaf(Mt[r * S + k], gg[i][k], acc);
                d[r] = acc;
            }
            e = compose(e, make_aff<S>(Mt, d));
        }
        Aff<S> excl, total;
        cta_scan<S, C>(e, sm, excl, total);
        if (tid < 32) {
            float base[S];
#pragma unroll
            for (int k = 0; k < S; ++k) base[k] = 0.f;
            if (!look_back<S, C>(lb, sm, total, tile, chunk, nseq, A.epoch0 + 1u, base, A.ctl, A.sticky, A.dbg))
                if ((tid & 31) == 0) s_fail = 1;
        }
        __syncthreads();
        if (s_fail) return;
        float mu[S];
        excl.apply(sm.carry[c], mu);  // mu_{t+1} entering this thread's first step
        float gp[NP];
#pragma unroll
        for (int k = 0; k < NP; ++k) gp[k] = 0.f;
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = tbase + (L - 1 - i);
            float lam[S];
#pragma unroll
            for (int k = 0; k < S; ++k) lam[k] = gg[i][k] + mu[k];
            float gxv[3];
#pragma unroll
            for (int qg = 0; qg < 3; ++qg) {
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < S; ++k) acc = fmaf(dp[i][k * 3 + qg], lam[k], acc);
                gxv[qg] = acc;
            }
            if (S == 1) {
                gp[0] = fmaf(gxv[0], fac[i][0], gp[0]);
                gp[1] = fmaf(gxv[1], fac[i][0], gp[1]);
                gp[2] = fmaf(gxv[2], fac[i][1 % NF], gp[2]);
            } else {
                gp[0] = fmaf(gxv[0], fac[i][0], gp[0]);
                gp[1] = fmaf(gxv[1], fac[i][0], gp[1]);
                gp[2] = fmaf(gxv[2], fac[i][0], gp[2]);
                gp[3 % NP] = fmaf(gxv[0], fac[i][1 % NF], gp[3 % NP]);
                gp[4 % NP] = fmaf(gxv[2], fac[i][2 % NF], gp[4 % NP]);
            }
#pragma unroll
            for (int r = 0; r < S; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < S; ++k) acc = fmaf(Jm[i][k * S + r], lam[k], acc);
                mu[r] = acc;
            }
            if (cv && t < A.T) {
                float *o = A.gx + ((size_t)b * A.T + t) * 3 * A.H + hh;
                o[0] = gxv[0];
                o[A.H] = gxv[1];
                o[2 * A.H] = gxv[2];
                if (t == 0 && A.gh0) {
#pragma unroll
                    for (int k = 0; k < S; ++k) A.gh0[((size_t)b * A.H + hh) * S + k] = mu[k];
                }
            }
        }
#pragma unroll
        for (int k = 0; k < NP; ++k) s_gp[tid][k] = gp[k];
        __syncthreads();
        if (tid < C && cv) {
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                float acc = 0.f;
                for (int j = tid; j < kThreads; j += C) acc += s_gp[j][k];
                atomicAdd(A.gp + (size_t)k * A.H + hh, acc);
            }
        }
        __syncthreads();
    }
}

namespace {
int pick_C(int H) {
    if (H >= 32) return 32;
    int c = 1;
    while (c < H) c <<= 1;
    return c;
}
template <class Cell, int L> const void *adj_kernel_by_C(int C) {
    switch (C) {
        case 1: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 1, L>);
        case 2: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 2, L>);
        case 4: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 4, L>);
        case 8: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 8, L>);
        case 16: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 16, L>);
        default: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 32, L>);
    }
}
}  // namespace

int adjoint_plan(const AdjointReq &r, int num_sms, Plan *plan) {
    const int S = r.cell == 1 ? 2 : 1;
    const int L = S == 1 ? 8 : 4;
    const int C = pick_C(r.H);
    const int TCH = (kThreads / C) * L;
    const long nseq = (long)r.B * ((r.H + C - 1) / C);
    plan->ntiles = nseq * ((r.T + TCH - 1) / TCH);
    plan->kernel = S == 1 ? adj_kernel_by_C<GruCell, 8>(C) : adj_kernel_by_C<LstmCell, 4>(C);
    plan->variant = C;
    plan->C = C;
    plan->agg_words = (size_t)plan->ntiles * C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * C * S;
    plan->side_bytes = 0;
    plan->epochs = 2;
    plan->grid = occupancy_grid(plan->kernel, kThreads, 0, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t adjoint_launch(const AdjointReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                           cudaStream_t st) {
    AdjArgs A;
    A.B = r.B;
    A.T = r.T;
    A.H = r.H;
    A.xproj = r.xproj;
    A.a = r.a;
    A.peep = r.peep;
    A.h0 = r.h0;
    A.h = r.h;
    A.g = r.g;
    A.gx = r.grad_xproj;
    A.gp = r.grad_params;
    A.gh0 = r.grad_h0;
    A.ctl = w.ctl;
    A.sticky = w.sticky;
    A.agg = w.agg;
    A.inc = w.inc;
    A.epoch0 = w.epoch0;
    A.dbg.wait_ns = dbg.wait_ns;
    A.dbg.skip_tile = dbg.skip_tile;
    A.dbg.delta_log = nullptr;
    A.dbg.delta_log_cap = 0;
    A.dbg.no_halo = 1;
    void *args[] = {&A};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(kThreads), args, 0, st);
}

}  // namespace prn
