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
#include "staged_tiles.cuh"

namespace prn {

struct AdjArgs {
    int B, T, H;
    const float *xproj, *a, *peep, *h0, *h, *g;
    float *gx, *gp, *gh0;
    float *gws;  // per-CTA parameter-gradient partials [grid][NPAR][H] (table variant)
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

// TAB: the recurrent-parameter gradients accumulate in a shared-memory table of the
// CTA (all H units, shared atomics, no barrier per tile), written once to a per-CTA
// slab and summed over CTAs after a grid barrier (deterministic).  Otherwise each tile
// reduces its sub-chunks in shared memory and adds one value per unit to grad_params.
template <class Cell, int C, int L, bool TAB>
__global__ void __launch_bounds__(kThreads, 2) adjoint_kernel(const AdjArgs A) {
    constexpr int S = Cell::S;
    constexpr int NF = S == 1 ? 2 : 3;   // parameter factors per step
    constexpr int NP = Cell::NPAR;
    constexpr int SUB = kThreads / C;
    constexpr int TCH = SUB * L;
    __shared__ ScanSmem<S, C> sm;
    __shared__ float s_gp[TAB ? 1 : kThreads][NP];
    __shared__ int s_fail;
    extern __shared__ float gp_tab[];  // TAB: [NP][H]
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = (A.H + C - 1) / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    LookBack<S> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;
    if (TAB) {
        for (int e = tid; e < NP * A.H; e += kThreads) gp_tab[e] = 0.f;
        __syncthreads();
    }
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
        if (TAB) {
            if (cv) {
#pragma unroll
                for (int k = 0; k < NP; ++k) atomicAdd(gp_tab + k * A.H + hh, gp[k]);
            }
        } else {
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
    if (TAB) {
        const int nv = NP * A.H;
        __syncthreads();
        float *mine = A.gws + (size_t)blockIdx.x * nv;
        for (int e = tid; e < nv; e += kThreads) mine[e] = gp_tab[e];
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        for (int e = blockIdx.x * kThreads + tid; e < nv; e += gridDim.x * kThreads) {
            float acc = 0.f;
            for (int g = 0; g < (int)gridDim.x; ++g) acc += A.gws[(size_t)g * nv + e];
            A.gp[e] = acc;
        }
    }
}

// ------------------------------------------------------------------ staged (H % 32 == 0)
// The same reverse scan for tiles of 32 units x TCH steps whose inputs (xproj, the
// states before each step, g) are copied into shared memory with cp.async; the next
// tile's copies are issued as soon as the current tile's inputs are in registers, so
// they overlap its scan, look-back and gradient stores.
template <class Cell, int L> struct AdjStage {
    static constexpr int S = Cell::S, C = 32, SUB = kThreads / C, TCH = SUB * L;
    static constexpr int ROWP = 3 * C, ROWS = C * S;
    static constexpr int OFFH = TCH * ROWP;                 // states: TCH + 1 rows (row 0: before the tile)
    static constexpr int OFFG = OFFH + (TCH + 1) * ROWS;    // g: TCH rows
    static constexpr int FLOATS = OFFG + TCH * ROWS;
};

template <class Cell, int L>
__device__ __forceinline__ void adj_issue(const AdjArgs &A, float *st, int b, int ct, int t_lo) {
    using G = AdjStage<Cell, L>;
    constexpr int S = Cell::S, TCH = G::TCH, ROWS = G::ROWS;
    const size_t row = (size_t)b * A.T;
    for (int q = threadIdx.x; q < TCH * 3 * 8; q += kThreads) {
        const int r = q >> 3, part = q & 7, t = r / 3, g = r % 3;
        const bool v = t_lo + t < A.T;
        const float *gp = A.xproj + ((row + t_lo + (v ? t : 0)) * 3 + g) * A.H + ct * 32 + part * 4;
        cp_async16(st + r * 32 + part * 4, gp, v ? 16 : 0);
    }
    for (int q = threadIdx.x; q < (TCH + 1) * 8 * S; q += kThreads) {
        const int r = q / (8 * S), part = q % (8 * S), t = t_lo - 1 + r;  // state h_t (t = -1: h0)
        const float *gp;
        int bytes = 16;
        if (t < 0) {
            gp = A.h0 ? A.h0 + ((size_t)b * A.H + ct * 32) * S + part * 4 : A.h;
            if (!A.h0) bytes = 0;
        } else {
            const bool v = t < A.T;
            gp = A.h + ((row + (v ? t : 0)) * A.H + ct * 32) * S + part * 4;
            if (!v) bytes = 0;
        }
        cp_async16(st + G::OFFH + r * ROWS + part * 4, gp, bytes);
    }
    for (int q = threadIdx.x; q < TCH * 8 * S; q += kThreads) {
        const int r = q / (8 * S), part = q % (8 * S);
        const bool v = t_lo + r < A.T;
        const float *gp = A.g + ((row + t_lo + (v ? r : 0)) * A.H + ct * 32) * S + part * 4;
        cp_async16(st + G::OFFG + r * ROWS + part * 4, gp, v ? 16 : 0);
    }
    cp_async_commit();
}

template <class Cell, int L, bool TAB>
__global__ void __launch_bounds__(kThreads, 2) adjoint_staged_kernel(const AdjArgs A) {
    using G = AdjStage<Cell, L>;
    constexpr int S = Cell::S, C = 32, SUB = G::SUB, TCH = G::TCH;
    constexpr int NF = S == 1 ? 2 : 3;
    constexpr int NP = Cell::NPAR;
    extern __shared__ __align__(16) float smf[];
    float *const st = smf;                 // stage
    float *const gp_tab = smf + G::FLOATS;  // TAB: [NP][H]
    __shared__ ScanSmem<S, C> sm;
    __shared__ float s_gp[TAB ? 1 : kThreads][NP];
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = A.H / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    LookBack<S> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;
    if (TAB)
        for (int e = tid; e < NP * A.H; e += kThreads) gp_tab[e] = 0.f;
    TileWalk tw(nseq);
    if (blockIdx.x < ntiles) adj_issue<Cell, L>(A, st, tw.seq / nct, tw.seq % nct, (nchunk - 1 - tw.chunk) * TCH);
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
        const int chunk = tw.chunk, seq = tw.seq;  // scan order: from the end of time
        const int b = seq / nct, ct = seq % nct, h = ct * C + c;
        const int t_lo = (nchunk - 1 - chunk) * TCH;
        const int rbase = (SUB - 1 - s) * L;  // local row of the thread's earliest step
        cp_async_wait_all();
        __syncthreads();
        Cell cell;
        cell.load(A.a, A.peep, A.H, h);
        float Jm[L][S * S], gg[L][S], dp[L][3 * S], fac[L][NF];
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int lr = rbase + (L - 1 - i);  // scan step i is local row lr (descending time)
            const bool v = t_lo + lr < A.T;
            float p[3], hp[S], gv[S];
#pragma unroll
            for (int g = 0; g < 3; ++g) p[g] = st[lr * G::ROWP + g * 32 + c];
#pragma unroll
            for (int k = 0; k < S; ++k) {
                hp[k] = st[G::OFFH + lr * G::ROWS + c * S + k];  // row lr = state before step lr
                gv[k] = st[G::OFFG + lr * G::ROWS + c * S + k];
            }
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
        __syncthreads();  // the stage is consumed: copy the next tile
        {
            TileWalk nx = tw;
            nx.next();
            if (tile + gridDim.x < ntiles)
                adj_issue<Cell, L>(A, st, nx.seq / nct, nx.seq % nct, (nchunk - 1 - nx.chunk) * TCH);
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
        if (s_fail) {
            cp_async_wait_all();
            return;
        }
        float mu[S];
        excl.apply(sm.carry[c], mu);
        float gp[NP];
#pragma unroll
        for (int k = 0; k < NP; ++k) gp[k] = 0.f;
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = t_lo + rbase + (L - 1 - i);
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
            if (t < A.T) {
                float *o = A.gx + ((size_t)b * A.T + t) * 3 * A.H + h;
                o[0] = gxv[0];
                o[A.H] = gxv[1];
                o[2 * A.H] = gxv[2];
                if (t == 0 && A.gh0) {
#pragma unroll
                    for (int k = 0; k < S; ++k) A.gh0[((size_t)b * A.H + h) * S + k] = mu[k];
                }
            }
        }
        if (TAB) {
#pragma unroll
            for (int k = 0; k < NP; ++k) atomicAdd(gp_tab + k * A.H + h, gp[k]);
        } else {
#pragma unroll
            for (int k = 0; k < NP; ++k) s_gp[tid][k] = gp[k];
            __syncthreads();
            if (tid < C) {
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    float acc = 0.f;
                    for (int j = tid; j < kThreads; j += C) acc += s_gp[j][k];
                    atomicAdd(A.gp + (size_t)k * A.H + h, acc);
                }
            }
        }
    }
    cp_async_wait_all();
    if (TAB) {
        const int nv = NP * A.H;
        __syncthreads();
        float *mine = A.gws + (size_t)blockIdx.x * nv;
        for (int e = tid; e < nv; e += kThreads) mine[e] = gp_tab[e];
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        for (int e = blockIdx.x * kThreads + tid; e < nv; e += gridDim.x * kThreads) {
            float acc = 0.f;
            for (int g = 0; g < (int)gridDim.x; ++g) acc += A.gws[(size_t)g * nv + e];
            A.gp[e] = acc;
        }
    }
}

namespace {
int pick_C(int H) {
    if (H >= 32) return 32;
    int c = 1;
    while (c < H) c <<= 1;
    return c;
}
template <class Cell, int L, bool TAB> const void *adj_kernel_by_C(int C) {
    switch (C) {
        case 1: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 1, L, TAB>);
        case 2: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 2, L, TAB>);
        case 4: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 4, L, TAB>);
        case 8: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 8, L, TAB>);
        case 16: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 16, L, TAB>);
        default: return reinterpret_cast<const void *>(&adjoint_kernel<Cell, 32, L, TAB>);
    }
}
constexpr int kTabMaxFloats = 12288;  // shared-memory table limit (48 KB)
}  // namespace

int adjoint_plan(const AdjointReq &r, int num_sms, Plan *plan) {
    const int wide = adjoint_wide_plan(r, num_sms, plan);  // TMA-fed tiles for H % 32 == 0
    if (wide <= 0) return wide;
    const int S = r.cell == 1 ? 2 : 1;
    const int L = S == 1 ? 8 : 4;
    const int C = pick_C(r.H);
    const int TCH = (kThreads / C) * L;
    const long nseq = (long)r.B * ((r.H + C - 1) / C);
    plan->ntiles = nseq * ((r.T + TCH - 1) / TCH);
    const int np = S == 1 ? GruCell::NPAR : LstmCell::NPAR;
    const bool tab = (long)np * r.H <= kTabMaxFloats;
    const bool staged = r.H % 32 == 0;  // whole 128-byte rows of 32 units
    plan->dyn_smem = tab ? np * r.H * (int)sizeof(float) : 0;
    if (staged) {
        plan->kernel = S == 1 ? (tab ? reinterpret_cast<const void *>(&adjoint_staged_kernel<GruCell, 8, true>)
                                     : reinterpret_cast<const void *>(&adjoint_staged_kernel<GruCell, 8, false>))
                              : (tab ? reinterpret_cast<const void *>(&adjoint_staged_kernel<LstmCell, 4, true>)
                                     : reinterpret_cast<const void *>(&adjoint_staged_kernel<LstmCell, 4, false>));
        plan->dyn_smem += (S == 1 ? AdjStage<GruCell, 8>::FLOATS : AdjStage<LstmCell, 4>::FLOATS) * (int)sizeof(float);
    } else {
        plan->kernel = S == 1 ? (tab ? adj_kernel_by_C<GruCell, 8, true>(C) : adj_kernel_by_C<GruCell, 8, false>(C))
                              : (tab ? adj_kernel_by_C<LstmCell, 4, true>(C) : adj_kernel_by_C<LstmCell, 4, false>(C));
    }
    if (cudaFuncSetAttribute(plan->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, plan->dyn_smem) !=
        cudaSuccess)
        return -1;
    plan->variant = C;
    plan->C = C;
    plan->agg_words = (size_t)plan->ntiles * C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * C * S;
    plan->epochs = 2;
    plan->grid = occupancy_grid(plan->kernel, kThreads, plan->dyn_smem, num_sms, plan->ntiles);
    plan->side_bytes = tab ? (size_t)plan->grid * np * r.H * sizeof(float) : 0;  // per-CTA partials
    plan->tab = tab ? 1 : 0;
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t adjoint_launch(const AdjointReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                           cudaStream_t st) {
    if (plan.staged == 2) return adjoint_wide_launch(r, plan, w, dbg, st);
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
    A.gws = plan.tab ? w.side : nullptr;
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
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(kThreads), args, plan.dyn_smem, st);
}

}  // namespace prn
