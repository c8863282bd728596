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
#include "staged_tiles.cuh"

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

// ------------------------------------------------------------------ staged (N % 32 == 0)
// The same scan for tiles of 32 channels x TCH steps whose J and b rows are copied into
// shared memory with cp.async through a ring of NST stages: a CTA's next NST-1 tiles
// are in flight while it scans, looks back and stores the current one.
#ifndef PRN_SCAN_DIAG_L
#define PRN_SCAN_DIAG_L 16
#endif
#ifndef PRN_SCAN_DIAG_MINB
#define PRN_SCAN_DIAG_MINB 3
#endif
constexpr int kStagedL[3] = {0, PRN_SCAN_DIAG_L, 8};  // steps per thread, by block size
constexpr int kStagedMinB[3] = {0, PRN_SCAN_DIAG_MINB, 2};
template <int S, int L> struct ScanStage {
    static constexpr int C = 32, SUB = kThreads / C, TCH = SUB * L, NST = 2;
    static constexpr int ROWJ = C * S * S, ROWB = C * S;  // floats per step
    static constexpr int OFFB = TCH * ROWJ;
    static constexpr int STAGE = TCH * (ROWJ + ROWB);
    static constexpr int FLOATS = NST * STAGE;
};

template <int S, int L>
__device__ __forceinline__ void scan_issue(const ScanArgs &A, float *st, int b, int ct, int t_lo) {
    using G = ScanStage<S, L>;
    constexpr int TCH = G::TCH, CJ = G::ROWJ / 4, CB = G::ROWB / 4;  // 16-byte chunks per step
    const size_t row = (size_t)b * A.T;
    const int jt0 = A.reverse ? t_lo + 1 : t_lo;  // reverse steps use J_{t+1}
    for (int q = threadIdx.x; q < TCH * CJ; q += kThreads) {
        const int r = q / CJ, part = q % CJ, t = jt0 + r;
        const bool v = t < A.T;
        cp_async16(st + r * G::ROWJ + part * 4, A.J + ((row + (v ? t : 0)) * A.N + ct * 32) * (S * S) + part * 4,
                   v ? 16 : 0);
    }
    for (int q = threadIdx.x; q < TCH * CB; q += kThreads) {
        const int r = q / CB, part = q % CB, t = t_lo + r;
        const bool v = t < A.T;
        cp_async16(st + G::OFFB + r * G::ROWB + part * 4, A.b + ((row + (v ? t : 0)) * A.N + ct * 32) * S + part * 4,
                   v ? 16 : 0);
    }
}

template <int S, int L>
__global__ void __launch_bounds__(kThreads, kStagedMinB[S]) scan_staged_kernel(const ScanArgs A) {
    using G = ScanStage<S, L>;
    constexpr int C = 32, SUB = G::SUB, TCH = G::TCH;
    extern __shared__ __align__(16) float st[];
    __shared__ ScanSmem<S, C> sm;
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = A.N / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    LookBack<S> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;
    auto t_lo_of = [&](int chunk) { return (A.reverse ? nchunk - 1 - chunk : chunk) * TCH; };
    // One commit group per tile slot, empty past the CTA's last tile, so that waiting
    // for all but the NST-1 newest groups always completes the current tile's.
    TileWalk tw(nseq), ahead(nseq);
    long tile_ahead = blockIdx.x;
#pragma unroll
    for (int k = 0; k < G::NST - 1; ++k) {
        if (tile_ahead < ntiles)
            scan_issue<S, L>(A, st + k * G::STAGE, ahead.seq / nct, ahead.seq % nct, t_lo_of(ahead.chunk));
        cp_async_commit();
        tile_ahead += gridDim.x;
        ahead.next();
    }
    int slot = 0;
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
        const int chunk = tw.chunk, b = tw.seq / nct, n = (tw.seq % nct) * C + c;
        const int t_lo = t_lo_of(chunk);
        const int sub = A.reverse ? SUB - 1 - s : s;
        {  // refill the slot consumed last iteration with the tile NST-1 ahead
            const int fill = slot == 0 ? G::NST - 1 : slot - 1;
            if (tile_ahead < ntiles)
                scan_issue<S, L>(A, st + fill * G::STAGE, ahead.seq / nct, ahead.seq % nct, t_lo_of(ahead.chunk));
            cp_async_commit();
            tile_ahead += gridDim.x;
            ahead.next();
        }
        cp_async_wait_group<G::NST - 1>();
        __syncthreads();
        const float *sg = st + slot * G::STAGE;
        slot = slot + 1 == G::NST ? 0 : slot + 1;
        float M[L][S * S], d[L][S];
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int lr = sub * L + (A.reverse ? L - 1 - i : i);  // local row of scan step i
            const int t = t_lo + lr;
            if (t < A.T) {
                const float *jp = sg + lr * G::ROWJ + c * (S * S);
                if (!A.reverse) {
#pragma unroll
                    for (int q = 0; q < S * S; ++q) M[i][q] = jp[q];
                } else if (t + 1 < A.T) {  // J_{t+1}^T
                    M[i][0] = jp[0];
                    if (S == 2) {
                        M[i][1 % (S * S)] = jp[2 % (S * S)];
                        M[i][2 % (S * S)] = jp[1 % (S * S)];
                        M[i][3 % (S * S)] = jp[3 % (S * S)];
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < S * S; ++q) M[i][q] = (q % (S + 1)) == 0 ? 1.f : 0.f;
                }
#pragma unroll
                for (int q = 0; q < S; ++q) d[i][q] = sg[G::OFFB + lr * G::ROWB + c * S + q];
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
            for (int q = 0; q < S; ++q) base[q] = A.h0 ? A.h0[((size_t)b * A.N + n) * S + q] : 0.f;
            if (!look_back<S, C>(lb, sm, total, tile, chunk, nseq, A.epoch0 + 1u, base, A.ctl, A.sticky, A.dbg))
                if ((tid & 31) == 0) s_fail = 1;
        }
        __syncthreads();
        if (s_fail) {
            cp_async_wait_all();
            return;
        }
        float x[S];
        excl.apply(sm.carry[c], x);
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = t_lo + sub * L + (A.reverse ? L - 1 - i : i);
            float y[S];
            make_aff<S>(M[i], d[i]).apply(x, y);
#pragma unroll
            for (int q = 0; q < S; ++q) x[q] = y[q];
            if (t < A.T) {
                float *op = A.out + (((size_t)b * A.T + t) * A.N + n) * S;
                if (S == 1) {
                    op[0] = y[0];
                } else {
                    *reinterpret_cast<float2 *>(op) = make_float2(y[0], y[S - 1]);
                }
            }
        }
    }
    cp_async_wait_all();
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
    const bool staged = r.N % 32 == 0;  // 128-byte rows of 32 channels
    const int L = staged ? kStagedL[S] : S == 1 ? 16 : 8;
    const int C = pick_C(r.N);
    const int TCH = (kThreads / C) * L;
    const long nseq = (long)r.B * ((r.N + C - 1) / C);
    plan->ntiles = nseq * ((r.T + TCH - 1) / TCH);
    plan->kernel = S == 1 ? scan_kernel_by_C<1, 16>(C) : scan_kernel_by_C<2, 8>(C);
    plan->dyn_smem = 0;
    if (staged) {
        constexpr int L1 = kStagedL[1], L2 = kStagedL[2];
        plan->kernel = S == 1 ? reinterpret_cast<const void *>(&scan_staged_kernel<1, L1>)
                              : reinterpret_cast<const void *>(&scan_staged_kernel<2, L2>);
        plan->dyn_smem = (S == 1 ? ScanStage<1, L1>::FLOATS : ScanStage<2, L2>::FLOATS) * (int)sizeof(float);
        if (cudaFuncSetAttribute(plan->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, plan->dyn_smem) !=
            cudaSuccess)
            return -1;
    }
    plan->variant = C;
    plan->C = C;
    plan->agg_words = (size_t)plan->ntiles * C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * C * S;
    plan->side_bytes = 0;
    plan->epochs = 2;
    plan->grid = occupancy_grid(plan->kernel, kThreads, plan->dyn_smem, num_sms, plan->ntiles);
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
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(kThreads), args, plan.dyn_smem, st);
}

}  // namespace prn
