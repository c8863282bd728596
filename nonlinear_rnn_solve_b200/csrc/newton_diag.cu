// newton_diag.cu -- fused Newton (DEER) forward for cells whose Jacobian is diagonal
// (ParaGRU) or 2x2 block diagonal (ParaLSTM).
//
// "Parallelizing non-linear sequential models over the sequence length", Approach:
// each Newton iteration linearises the recurrence with its Jacobians and solves the
// linear recurrence with an associative prefix scan.  Here one persistent cooperative
// kernel runs every iteration:
//
//   for k = 0, 1, ...:                                    (device-side loop)
//     for each tile [T-chunk x C channels] of this CTA:
//       read h^(k) and the projected inputs once; evaluate f, J and the residual
//       r_t = f(h^(k)_{t-1}) - h^(k)_t in registers (J and r never reach HBM);
//       scan the update delta_t = J_t delta_{t-1} + r_t, delta_{-1} = 0: thread-serial
//       over L steps, warp shuffles, shared memory, then decoupled look-back across
//       T-chunks;  write h^(k+1) = h^(k) + delta in place;
//     max |delta| -> grid barrier -> every CTA takes the same stop decision.
//
// The update in delta form is the b-form step h^(k+1)_t = J_t h^(k+1)_{t-1} + b_t,
// b_t = f_t - J_t h^(k)_{t-1}, minus h^(k)_t on both sides; it is equal in exact
// arithmetic and keeps fp32 rounding proportional to the (vanishing) update.
//
// In-place update without a second state buffer: a tile reads its own steps of h^(k)
// plus h^(k)_{t0-1} of the tile before it; the latter is read from a small side
// buffer written in the previous iteration, so no tile ever reads a step another
// tile may already have overwritten.
#include <algorithm>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"
#include "newton_common.cuh"

namespace prn {

template <class Cell, int C, int L, int IN>
__global__ void __launch_bounds__(kThreads, 2) newton_diag_kernel(const NewtonDiagArgs A) {
    constexpr int S = Cell::S;
    constexpr int SUB = kThreads / C;
    constexpr int TCH = SUB * L;
    __shared__ ScanSmem<S, C> sm;
    __shared__ unsigned s_red[kThreads / 32];
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = (A.H + C - 1) / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    const size_t side_stride = (size_t)ntiles * C * S;
    LookBack<S> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;

    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epoch = A.epoch0 + (unsigned)k + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        const float *side_in = A.side + (size_t)(k & 1) * side_stride;
        float *side_out = A.side + (size_t)((k + 1) & 1) * side_stride;
        float my_max = 0.f;
        TileWalk tw(nseq);
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
            const int chunk = tw.chunk;
            const int seq = tw.seq;
            const int b = seq / nct;
            const int h = (seq % nct) * C + c;
            const bool cv = h < A.H;
            const int hh = cv ? h : 0;
            const int t0 = chunk * TCH + s * L;
            Cell cell;
            cell.load(A.a, A.peep, A.H, hh);
            Proj<IN> pj;
            pj.load(A, hh);

            // state entering step t0 (iterate k)
            float hp[S];
#pragma unroll
            for (int q = 0; q < S; ++q) hp[q] = 0.f;
            if (t0 == 0) {
                if (A.h0) load_state<S>(A.h0, (size_t)b * A.H + hh, hp);
            } else if (k > 0) {
                if (s == 0) {
#pragma unroll
                    for (int q = 0; q < S; ++q) hp[q] = side_in[((tile - nseq) * C + c) * S + q];
                } else if (t0 - 1 < A.T) {
                    load_state<S>(A.h, ((size_t)b * A.T + (t0 - 1)) * A.H + hh, hp);
                }
            }
            float Jr[L][S * S], rr[L][S], hc[L][S];
#pragma unroll
            for (int i = 0; i < L; ++i) {
                const int t = t0 + i;
                const bool v = cv && t < A.T;
                float p[3];
                pj.get(b, v ? t : 0, hh, p);
                float cur[S];
#pragma unroll
                for (int q = 0; q < S; ++q) cur[q] = 0.f;
                if (k > 0 && v) load_state<S>(A.h, ((size_t)b * A.T + t) * A.H + hh, cur);
                float f[S], J[S * S];
                cell.eval(p, hp, f, J);
                apply_jmode<S>(A.jmode, J);
#pragma unroll
                for (int q = 0; q < S; ++q) {
                    rr[i][q] = v ? f[q] - cur[q] : 0.f;
                    hc[i][q] = cur[q];
                    hp[q] = cur[q];
                }
#pragma unroll
                for (int q = 0; q < S * S; ++q) Jr[i][q] = v ? J[q] : ((q % (S + 1)) == 0 ? 1.f : 0.f);
            }
            Aff<S> e = Aff<S>::ident();
#pragma unroll
            for (int i = 0; i < L; ++i) e = compose(e, make_aff<S>(Jr[i], rr[i]));
            Aff<S> excl, total;
            cta_scan<S, C>(e, sm, excl, total);
            if (tid < 32) {
                float base[S];
#pragma unroll
                for (int q = 0; q < S; ++q) base[q] = 0.f;  // delta entering t = 0 is 0
                if (!look_back<S, C>(lb, sm, total, tile, chunk, nseq, epoch, base, A.ctl, A.sticky, A.dbg))
                    if ((tid & 31) == 0) s_fail = 1;
            }
            __syncthreads();
            if (s_fail) return;  // a bounded wait ran out; the status says so
            float d[S];
            excl.apply(sm.carry[c], d);
#pragma unroll
            for (int i = 0; i < L; ++i) {
                const int t = t0 + i;
                float nd[S];
                const Aff<S> el = make_aff<S>(Jr[i], rr[i]);
                el.apply(d, nd);
                float hn[S];
#pragma unroll
                for (int q = 0; q < S; ++q) {
                    d[q] = nd[q];
                    hn[q] = hc[i][q] + nd[q];
                    const float ad = fabsf(nd[q]);
                    my_max = (ad > my_max || isnan(nd[q])) ? ad : my_max;
                }
                if (cv && t < A.T) store_state<S>(A.h, ((size_t)b * A.T + t) * A.H + hh, hn);
                if (i == L - 1 && s == SUB - 1 && cv && chunk < nchunk - 1) {
#pragma unroll
                    for (int q = 0; q < S; ++q) side_out[(tile * C + c) * S + q] = hn[q];
                }
            }
            __syncthreads();
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

    // Final residual max |h_t - f(h_{t-1})| at the returned iterate.
    if (A.residual_out && !stop_all)
        if (!residual_pass<Cell, C, L, IN>(A, s_red)) return;
    if (blockIdx.x == 0 && tid == 0) {
        *A.iters_out = iters;
        if (A.delta_out) *A.delta_out = last_delta;
        if (!stop_all && A.tol > 0.f && iters == A.max_iters && !(last_delta < A.tol))
            atomicOr(A.sticky, kStNotConverged);
    }
}

// ------------------------------------------------------------------ host dispatch
namespace {

int pick_C(int H) {
    if (H >= 32) return 32;
    int c = 1;
    while (c < H) c <<= 1;
    return c;
}

template <class Cell, int C, int IN> const void *kernel_for() {
    constexpr int L = Cell::S == 1 ? 16 : 8;
    return reinterpret_cast<const void *>(&newton_diag_kernel<Cell, C, L, IN>);
}

template <class Cell, int IN> const void *kernel_by_C(int C) {
    switch (C) {
        case 1: return kernel_for<Cell, 1, IN>();
        case 2: return kernel_for<Cell, 2, IN>();
        case 4: return kernel_for<Cell, 4, IN>();
        case 8: return kernel_for<Cell, 8, IN>();
        case 16: return kernel_for<Cell, 16, IN>();
        default: return kernel_for<Cell, 32, IN>();
    }
}

template <class Cell> const void *kernel_by_in(int C, bool fused, int in) {
    if (!fused) return kernel_by_C<Cell, 0>(C);
    if (in == 2) return kernel_by_C<Cell, 2>(C);
    if (in == 4) return kernel_by_C<Cell, 4>(C);
    return kernel_by_C<Cell, -1>(C);
}

}  // namespace

int newton_diag_plan(const NewtonDiagReq &r, int num_sms, Plan *plan) {
    const int staged = newton_staged_plan(r, num_sms, plan);
    if (staged <= 0) return staged;
    const int S = r.cell == 1 ? 2 : 1;
    const int L = S == 1 ? 16 : 8;
    const int C = pick_C(r.H);
    const int TCH = (kThreads / C) * L;
    const long nct = (r.H + C - 1) / C;
    const long nseq = (long)r.B * nct;
    const long nchunk = (r.T + TCH - 1) / TCH;
    plan->ntiles = nseq * nchunk;
    const bool fused = r.xproj == nullptr;
    plan->kernel = r.cell == 1 ? kernel_by_in<LstmCell>(C, fused, r.in) : kernel_by_in<GruCell>(C, fused, r.in);
    plan->variant = C;
    plan->C = C;
    plan->dyn_smem = 0;
    plan->agg_words = (size_t)plan->ntiles * C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * C * S;
    plan->side_bytes = 2 * (size_t)plan->ntiles * C * S * sizeof(float);
    plan->epochs = (unsigned)r.max_iters + 1u;
    plan->grid = occupancy_grid(plan->kernel, kThreads, 0, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t newton_diag_launch(const NewtonDiagReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                               cudaStream_t st) {
    NewtonDiagArgs A;
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
    A.side = w.side;
    A.epoch0 = w.epoch0;
    A.dbg.wait_ns = dbg.wait_ns;
    A.dbg.skip_tile = dbg.skip_tile;
    A.dbg.delta_log = dbg.delta_log;
    A.dbg.delta_log_cap = dbg.delta_log_cap;
    // a withheld publication (failure-detection test) must be met by the look-back
    A.dbg.no_halo = dbg.no_halo || dbg.skip_tile >= 0;
    if (plan.staged == 2) return newton_wide_launch(A, plan, st);
    if (plan.staged) return newton_staged_launch(A, plan, st);
    void *args[] = {&A};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(kThreads), args, plan.dyn_smem, st);
}

int occupancy_grid(const void *kernel, int threads, size_t smem, int num_sms, long ntiles) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess) return -1;
    if (per_sm <= 0) return -1;
    long g = (long)per_sm * num_sms;
    if (ntiles < g) g = ntiles;
    return (int)std::max<long>(g, 1);
}

}  // namespace prn
