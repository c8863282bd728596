// scan.cu -- standalone linear recurrences by a chunked parallel scan, diagonal and
// 2x2-block ("Para-Seq" README, Main features: dense, diagonal and 2x2 block
// associative scans, plus reverse adjoint scans).
//
//   forward:  out_t = J_t out_{t-1} + b_t,        out_{-1} = h0 (or 0)
//   reverse:  out_t = b_t + J_{t+1}^T out_{t+1},  out_{T-1} = b_{T-1} + h0 (or 0)
//
// One pass over HBM: each thread composes its L steps in registers, the CTA combines
// its sub-chunks through warp shuffles and shared memory, and T-chunks are chained by
// decoupled look-back.  Reverse mode runs the same scan with T-chunks, sub-chunks
// and steps taken from the end.
#include "common.cuh"
#include "internal.h"

namespace prn {

struct ScanArgs {
    int B, T, N, reverse;
    const float *J, *b, *h0;
    float *out;
    Ctl *ctl;
    int *sticky;
    unsigned long long *agg, *inc;
    unsigned epoch0;
    Dbg dbg;
};

// Element of step t in scan order: forward (J_t, b_t); reverse (J_{t+1}^T, b_t), the
// last step's matrix being the identity.
template <int S>
__device__ __forceinline__ void load_elem(const ScanArgs &A, int b, int t, int n, float *M, float *d) {
    const size_t row = (size_t)b * A.T;
    if (!A.reverse) {
        const float *Jp = A.J + ((row + t) * A.N + n) * (S * S);
#pragma unroll
        for (int q = 0; q < S * S; ++q) M[q] = Jp[q];
    } else if (t + 1 < A.T) {
        const float *Jp = A.J + ((row + t + 1) * A.N + n) * (S * S);
        if (S == 1) {
            M[0] = Jp[0];
        } else {
            M[0] = Jp[0];
            M[1 % (S * S)] = Jp[2 % (S * S)];
            M[2 % (S * S)] = Jp[1 % (S * S)];
            M[3 % (S * S)] = Jp[3 % (S * S)];
        }
    } else {
#pragma unroll
        for (int q = 0; q < S * S; ++q) M[q] = (q % (S + 1)) == 0 ? 1.f : 0.f;
    }
    const float *bp = A.b + ((row + t) * A.N + n) * S;
#pragma unroll
    for (int q = 0; q < S; ++q) d[q] = bp[q];
}

template <int S, int C, int L>
__global__ void __launch_bounds__(kThreads, 2) scan_kernel(const ScanArgs A) {
    constexpr int SUB = kThreads / C;
    constexpr int TCH = SUB * L;
    __shared__ ScanSmem<S, C> sm;
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = (A.N + C - 1) / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    LookBack<S> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;
    TileWalk tw(nseq);
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
        const int chunk = tw.chunk;  // position in scan order
        const int seq = tw.seq;
        const int b = seq / nct;
        const int n = (seq % nct) * C + c;
        const bool cv = n < A.N;
        const int nn = cv ? n : 0;
        // time of this thread's first step in scan order, and the direction
        const int tchunk = A.reverse ? nchunk - 1 - chunk : chunk;
        const int sub = A.reverse ? SUB - 1 - s : s;
        const int tbase = tchunk * TCH + sub * L;
        float M[L][S * S], d[L][S];
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = A.reverse ? tbase + (L - 1 - i) : tbase + i;
            if (cv && t < A.T) {
                load_elem<S>(A, b, t, nn, M[i], d[i]);
            } else {
#pragma unroll
                for (int q = 0; q < S * S; ++q) M[i][q] = (q % (S + 1)) == 0 ? 1.f : 0.f;
#pragma unroll
                for (int q = 0; q < S; ++q) d[i][q] = 0.f;
            }
        }
        Aff<S> e = Aff<S>::ident();
#pragma unroll
        for (int i = 0; i < L; ++i) e = compose(e, make_aff<S>(M[i], d[i]));
        Aff<S> excl, total;
        cta_scan<S, C>(e, sm, excl, total);
        if (tid < 32) {
            float base[S];
#pragma unroll
            for (int q = 0; q < S; ++q) base[q] = 0.f;
            if (A.h0 && cv) {
#pragma unroll
                for (int q = 0; q < S; ++q) base[q] = A.h0[((size_t)b * A.N + nn) * S + q];
            }
            if (!look_back<S, C>(lb, sm, total, tile, chunk, nseq, A.epoch0 + 1u, base, A.ctl, A.sticky, A.dbg))
                if ((tid & 31) == 0) s_fail = 1;
        }
        __syncthreads();
        if (s_fail) return;
        float x[S];
        excl.apply(sm.carry[c], x);
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = A.reverse ? tbase + (L - 1 - i) : tbase + i;
            float y[S];
            make_aff<S>(M[i], d[i]).apply(x, y);
#pragma unroll
            for (int q = 0; q < S; ++q) x[q] = y[q];
            if (cv && t < A.T) {
                float *op = A.out + (((size_t)b * A.T + t) * A.N + nn) * S;
#pragma unroll
                for (int q = 0; q < S; ++q) op[q] = y[q];
            }
        }
        __syncthreads();
    }
}

namespace {
int pick_C(int N) {
    if (N >= 32) return 32;
    int c = 1;
    while (c < N) c <<= 1;
    return c;
}
template <int S, int L> const void *scan_kernel_by_C(int C) {
    switch (C) {
        case 1: return reinterpret_cast<const void *>(&scan_kernel<S, 1, L>);
        case 2: return reinterpret_cast<const void *>(&scan_kernel<S, 2, L>);
        case 4: return reinterpret_cast<const void *>(&scan_kernel<S, 4, L>);
        case 8: return reinterpret_cast<const void *>(&scan_kernel<S, 8, L>);
        case 16: return reinterpret_cast<const void *>(&scan_kernel<S, 16, L>);
        default: return reinterpret_cast<const void *>(&scan_kernel<S, 32, L>);
    }
}
}  // namespace

int scan_diag_plan(const ScanReq &r, int num_sms, Plan *plan) {
    const int S = r.kind == 1 ? 2 : 1;
    const int L = S == 1 ? 16 : 8;
    const int C = pick_C(r.N);
    const int TCH = (kThreads / C) * L;
    const long nseq = (long)r.B * ((r.N + C - 1) / C);
    plan->ntiles = nseq * ((r.T + TCH - 1) / TCH);
    plan->kernel = S == 1 ? scan_kernel_by_C<1, 16>(C) : scan_kernel_by_C<2, 8>(C);
    plan->variant = C;
    plan->C = C;
    plan->agg_words = (size_t)plan->ntiles * C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * C * S;
    plan->side_bytes = 0;
    plan->epochs = 2;
    plan->grid = occupancy_grid(plan->kernel, kThreads, 0, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t scan_diag_launch(const ScanReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                             cudaStream_t st) {
    ScanArgs A;
    A.B = r.B;
    A.T = r.T;
    A.N = r.N;
    A.reverse = r.reverse;
    A.J = r.J;
    A.b = r.b;
    A.h0 = r.h0;
    A.out = r.out;
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
