// newton_common.cuh -- pieces shared by the Newton kernels for diagonal and 2x2-block
// cells: kernel arguments, projected-input access, state access, residual pass.
#pragma once
#include <cuda.h>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"

namespace prn {

struct NewtonDiagArgs {
    int B, T, H, in;
    int jmode;  // linearisation (apply_jmode)
    const float *xproj, *x, *W, *bias, *a, *peep, *h0;
    float *h;
    int max_iters;
    float tol;
    int *iters_out;
    float *delta_out, *residual_out;
    Ctl *ctl;
    int *sticky;
    unsigned long long *agg, *inc;
    float *side;
    unsigned epoch0;
    Dbg dbg;
};

// Projected inputs p (3 gates) of unit h at (b, t).
// IN = 0: read xproj [B, T, 3, H].  IN > 0: recompute W x_t + bias with IN inputs.
// IN = -1: same with the runtime width (<= 8).
template <int IN> struct Proj {
    static constexpr int MAXIN = IN > 0 ? IN : 8;
    float w[3][MAXIN], bz[3];
    const float *x;
    int T, in;
    __device__ __forceinline__ void load(const NewtonDiagArgs &A, int h) {
        x = A.x;
        T = A.T;
        in = IN > 0 ? IN : A.in;
#pragma unroll
        for (int g = 0; g < 3; ++g) {
            bz[g] = A.bias ? __ldg(A.bias + g * A.H + h) : 0.f;
#pragma unroll
            for (int i = 0; i < MAXIN; ++i)
                w[g][i] = (i < in) ? __ldg(A.W + (size_t)(g * A.H + h) * in + i) : 0.f;
        }
    }
    __device__ __forceinline__ void get(int b, int t, int, float p[3]) const {
        const float *xr = x + ((size_t)b * T + t) * in;
        float xv[MAXIN];
        if (IN == 2) {
            float2 v = *reinterpret_cast<const float2 *>(xr);
            xv[0] = v.x;
            xv[1 % MAXIN] = v.y;
        } else if (IN == 4) {
            float4 v = *reinterpret_cast<const float4 *>(xr);
            xv[0] = v.x;
            xv[1 % MAXIN] = v.y;
            xv[2 % MAXIN] = v.z;
            xv[3 % MAXIN] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < MAXIN; ++i) xv[i] = (i < in) ? xr[i] : 0.f;
        }
#pragma unroll
        for (int g = 0; g < 3; ++g) {
            float acc = bz[g];
#pragma unroll
            for (int i = 0; i < MAXIN; ++i) acc = fmaf(w[g][i], xv[i], acc);
            p[g] = acc;
        }
    }
};
template <> struct Proj<0> {
    const float *xp;
    int T, H;
    __device__ __forceinline__ void load(const NewtonDiagArgs &A, int) {
        xp = A.xproj;
        T = A.T;
        H = A.H;
    }
    __device__ __forceinline__ void get(int b, int t, int h, float p[3]) const {
        const float *q = xp + ((size_t)b * T + t) * 3 * H + h;
        p[0] = q[0];
        p[1] = q[H];
        p[2] = q[2 * H];
    }
};

template <int S>
__device__ __forceinline__ void load_state(const float *hbuf, size_t idx, float *v) {
    if (S == 1) {
        v[0] = hbuf[idx];
    } else {
        float2 u = *reinterpret_cast<const float2 *>(hbuf + idx * 2);
        v[0] = u.x;
        v[S - 1] = u.y;
    }
}
template <int S>
__device__ __forceinline__ void store_state(float *hbuf, size_t idx, const float *v) {
    if (S == 1) {
        hbuf[idx] = v[0];
    } else {
        *reinterpret_cast<float2 *>(hbuf + idx * 2) = make_float2(v[0], v[S - 1]);
    }
}

// Tensor maps handed to the staged kernels (unused by the layouts without TMA).
struct StagedMaps {
    CUtensorMap x, h;
};

// Launch of a staged plan (newton_staged.cu).
cudaError_t newton_staged_launch(const NewtonDiagArgs &A, const Plan &plan, cudaStream_t st);
// Wide layers, H % 32 == 0 with projected inputs (newton_wide.cu): plan (1 = shape not
// covered) and launch.
int newton_wide_plan(const NewtonDiagReq &r, int num_sms, Plan *plan);
cudaError_t newton_wide_launch(const NewtonDiagArgs &A, const Plan &plan, cudaStream_t st);

// Final residual r = max over every state element of |h_t - f(h_{t-1}, x_t)| at the
// returned iterate (one read of the states and inputs), reduced over the grid.
// Tiles are [TCH = (NT / C) * L steps] x [C channels], as in the solver kernels.
template <class Cell, int C, int L, int IN, int NT = kThreads>
__device__ bool residual_pass(const NewtonDiagArgs &A, unsigned *s_red) {
    constexpr int S = Cell::S;
    constexpr int TCH = (NT / C) * L;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = (A.H + C - 1) / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    float my_res = 0.f;
    TileWalk tw(nseq);
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
        const int chunk = tw.chunk;
        const int seq = tw.seq;
        const int b = seq / nct;
        const int h = (seq % nct) * C + c;
        if (h >= A.H) continue;
        const int t0 = chunk * TCH + s * L;
        Cell cell;
        cell.load(A.a, A.peep, A.H, h);
        Proj<IN> pj;
        pj.load(A, h);
        float hp[S];
#pragma unroll
        for (int q = 0; q < S; ++q) hp[q] = 0.f;
        if (t0 == 0) {
            if (A.h0) load_state<S>(A.h0, (size_t)b * A.H + h, hp);
        } else if (t0 - 1 < A.T) {
            load_state<S>(A.h, ((size_t)b * A.T + (t0 - 1)) * A.H + h, hp);
        }
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = t0 + i;
            if (t >= A.T) break;
            float p[3], cur[S], f[S], J[S * S];
            pj.get(b, t, h, p);
            load_state<S>(A.h, ((size_t)b * A.T + t) * A.H + h, cur);
            cell.eval(p, hp, f, J);
#pragma unroll
            for (int q = 0; q < S; ++q) {
                const float ad = fabsf(cur[q] - f[q]);
                my_res = (ad > my_res || isnan(ad)) ? ad : my_res;
                hp[q] = cur[q];
            }
        }
    }
    const unsigned bits = block_max_bits<NT>(my_res, s_red);
    if (tid == 0) atomicMax(&A.ctl->res_bits, bits);
    if (!grid_sync(A.ctl, A.sticky, A.dbg)) return false;
    if (blockIdx.x == 0 && tid == 0) {
        const unsigned rb = ld_acquire(&A.ctl->res_bits);
        *A.residual_out = __uint_as_float(rb);
        if (rb >= 0x7f800000u) atomicOr(A.sticky, kStNonfinite);
    }
    return true;
}

}  // namespace prn
