// newton_staged.cu -- Newton (DEER) forward for ParaGRU / ParaLSTM with the tile's
// inputs staged in shared memory by asynchronous copies (cp.async), so that the HBM
// reads of the next tile overlap the scan, look-back and stores of the current one.
//
// Same method as newton_diag.cu ("Parallelizing non-linear sequential models over
// the sequence length", Approach: linearise, then solve the linear recurrence with a
// parallel prefix scan), specialised for the two shapes that carry the traffic:
//   long  (H == 1): a tile is 256 threads x L consecutive steps of one sequence; each
//         thread's segment sits in shared memory with a 16-byte pad so that its
//         128-bit reads are free of bank conflicts;
//   wide  (H % 32 == 0, projected inputs given): a tile is 32 channels x 8 sub-chunks
//         of L steps; every step is a 128-byte row per gate and per state, read by a
//         warp as one conflict-free row.
// Copies are issued as soon as the previous tile's slab has been read into registers
// (single stage, released early); the first tile of the next Newton iteration is
// prefetched right after this CTA's last stores, before the grid barrier.
#include <algorithm>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"
#include "newton_common.cuh"

#ifndef PRN_STAGED_MINB
#define PRN_STAGED_MINB 2  // resident CTAs per SM the register budget is sized for
#endif

namespace prn {

__device__ __forceinline__ void cp_async16(float *dst, const float *src, int src_bytes) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Copy n floats (n % 4 == 0) from a 16-byte aligned global address into consecutive
// segments of `seg` floats placed `str` floats apart; bytes at or beyond `end` are
// zero-filled.  Consecutive threads copy consecutive 16-byte chunks (coalesced).
__device__ __forceinline__ void copy_segments(float *dst, int seg, int str, const float *src, int n,
                                              const float *end) {
    for (int f = 4 * threadIdx.x; f < n; f += 4 * kThreads) {
        const float *gp = src + f;
        const long rem = end - gp;
        const int bytes = rem >= 4 ? 16 : (rem > 0 ? (int)rem * 4 : 0);
        cp_async16(dst + (f / seg) * str + (f % seg), bytes ? gp : src, bytes);
    }
}

// ---------------------------------------------------------------- long layout, H == 1
template <class Cell, int IN> struct LongLayout {
    static constexpr int S = Cell::S, C = 1, L = S == 1 ? 16 : 8, SUB = kThreads, TCH = SUB * L;
    static constexpr int PW = IN == 0 ? 3 : IN;     // input floats per step
    static constexpr int SEGP = L * PW, STRP = SEGP + 4;
    static constexpr int SEGH = L * S, STRH = SEGH + 4;
    static constexpr int OFFH = SUB * STRP;
    static constexpr int SMEM_FLOATS = SUB * (STRP + STRH);
    static_assert(SEGP % 4 == 0 && SEGH % 4 == 0, "segments are whole 16-byte chunks");
    static_assert(((SEGP / 4 + 1) & 1) && ((SEGH / 4 + 1) & 1), "odd chunk stride: conflict-free float4 reads");

    __device__ static void issue(const NewtonDiagArgs &A, float *sm, int b, int, int tch0, bool with_h) {
        const size_t row = (size_t)b * A.T;
        const float *pin = IN == 0 ? A.xproj : A.x;
        copy_segments(sm, SEGP, STRP, pin + (row + tch0) * PW, TCH * PW, pin + (row + A.T) * PW);
        if (with_h) copy_segments(sm + OFFH, SEGH, STRH, A.h + (row + tch0) * S, TCH * S, A.h + (row + A.T) * S);
    }
    // four consecutive steps (grp) of thread (s, c): inputs and states from shared memory
    __device__ static void load_group(const float *sm, int s, int, int grp, float pv[4][PW], float hv[4][S],
                                      bool with_h) {
        const float4 *pp = reinterpret_cast<const float4 *>(sm + s * STRP + grp * 4 * PW);
        float tmp[4 * PW];
#pragma unroll
        for (int q = 0; q < PW; ++q) {
            const float4 v = pp[q];
            tmp[4 * q] = v.x;
            tmp[4 * q + 1] = v.y;
            tmp[4 * q + 2] = v.z;
            tmp[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int q = 0; q < PW; ++q) pv[j][q] = tmp[j * PW + q];
        if (with_h) {
            const float4 *hp = reinterpret_cast<const float4 *>(sm + OFFH + s * STRH + grp * 4 * S);
            float th[4 * S];
#pragma unroll
            for (int q = 0; q < S; ++q) {
                const float4 v = hp[q];
                th[4 * q] = v.x;
                th[4 * q + 1] = v.y;
                th[4 * q + 2] = v.z;
                th[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int q = 0; q < S; ++q) hv[j][q] = th[j * S + q];
        }
    }
    // state at the step before thread s's first step (s > 0): last step of thread s - 1
    __device__ static void h_prev(const float *sm, int s, int, float *hp) {
#pragma unroll
        for (int q = 0; q < S; ++q) hp[q] = sm[OFFH + (s - 1) * STRH + SEGH - S + q];
    }
};

// ---------------------------------------------------------------- wide layout, H % 32 == 0
template <class Cell> struct WideLayout {
    static constexpr int S = Cell::S, C = 32, L = S == 1 ? 16 : 8, SUB = kThreads / C, TCH = SUB * L;
    static constexpr int PW = 3;
    static constexpr int ROWP = 3 * 32, ROWH = 32 * S;
    static constexpr int OFFH = TCH * ROWP;
    static constexpr int SMEM_FLOATS = TCH * (ROWP + ROWH);

    __device__ static void issue(const NewtonDiagArgs &A, float *sm, int b, int ct, int tch0, bool with_h) {
        const size_t row = (size_t)b * A.T;
        // inputs: TCH x 3 rows of 32 floats (8 chunks each)
        for (int q = threadIdx.x; q < TCH * 3 * 8; q += kThreads) {
            const int r = q >> 3, part = q & 7, t = r / 3, g = r % 3;
            const bool v = tch0 + t < A.T;
            const float *gp = A.xproj + ((row + tch0 + (v ? t : 0)) * 3 + g) * A.H + ct * 32 + part * 4;
            cp_async16(sm + r * 32 + part * 4, gp, v ? 16 : 0);
        }
        if (with_h) {
            for (int q = threadIdx.x; q < TCH * 8 * S; q += kThreads) {
                const int t = q / (8 * S), part = q % (8 * S);
                const bool v = tch0 + t < A.T;
                const float *gp = A.h + ((row + tch0 + (v ? t : 0)) * A.H + ct * 32) * S + part * 4;
                cp_async16(sm + OFFH + t * ROWH + part * 4, gp, v ? 16 : 0);
            }
        }
    }
    __device__ static void load_group(const float *sm, int s, int c, int grp, float pv[4][PW], float hv[4][S],
                                      bool with_h) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = s * L + grp * 4 + j;
#pragma unroll
            for (int g = 0; g < 3; ++g) pv[j][g] = sm[t * ROWP + g * 32 + c];
            if (with_h) {
                if (S == 1) {
                    hv[j][0] = sm[OFFH + t * ROWH + c];
                } else {
                    const float2 v = *reinterpret_cast<const float2 *>(sm + OFFH + t * ROWH + c * S);
                    hv[j][0] = v.x;
                    hv[j][S - 1] = v.y;
                }
            }
        }
    }
    __device__ static void h_prev(const float *sm, int s, int c, float *hp) {
#pragma unroll
        for (int q = 0; q < S; ++q) hp[q] = sm[OFFH + (s * L - 1) * ROWH + c * S + q];
    }
};

template <class Cell, class Lay, int IN>
__global__ void __launch_bounds__(kThreads, PRN_STAGED_MINB) newton_staged_kernel(const NewtonDiagArgs A) {
    constexpr int S = Cell::S, C = Lay::C, L = Lay::L, SUB = Lay::SUB, TCH = Lay::TCH, PW = Lay::PW;
    static_assert(L % 4 == 0, "steps are read in groups of four");
    extern __shared__ __align__(16) float smem[];
    __shared__ ScanSmem<S, C> sm;
    __shared__ unsigned s_red[kThreads / 32];
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = A.H / C;
    const long nseq = (long)A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = nseq * nchunk;
    const size_t side_stride = (size_t)ntiles * C * S;
    LookBack<S> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;

    // fused projection weights (long layout with raw inputs): p_g = bias_g + sum_q W[g][q] x_q
    float wz[3][IN > 0 ? IN : 1], bz[3];
#pragma unroll
    for (int g = 0; g < 3; ++g) {
        bz[g] = 0.f;
#pragma unroll
        for (int q = 0; q < (IN > 0 ? IN : 1); ++q) wz[g][q] = 0.f;
        if (IN > 0) {
            bz[g] = A.bias ? __ldg(A.bias + g * A.H) : 0.f;
#pragma unroll
            for (int q = 0; q < (IN > 0 ? IN : 1); ++q) wz[g][q] = __ldg(A.W + (size_t)g * A.H * IN + q);
        }
    }

    {
        const int chunk = (int)(blockIdx.x / nseq);
        const long seq = blockIdx.x - (long)chunk * nseq;
        Lay::issue(A, smem, (int)(seq / nct), (int)(seq % nct), chunk * TCH, false);
        cp_async_commit();
    }

    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epoch = A.epoch0 + (unsigned)k + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        const float *side_in = A.side + (size_t)(k & 1) * side_stride;
        float *side_out = A.side + (size_t)((k + 1) & 1) * side_stride;
        float my_max = 0.f;
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const int chunk = (int)(tile / nseq);
            const long seq = tile - (long)chunk * nseq;
            const int b = (int)(seq / nct);
            const int h = (int)(seq % nct) * C + c;
            const int t0 = chunk * TCH + s * L;
            cp_async_wait_all();
            __syncthreads();
            Cell cell;
            cell.load(A.a, A.peep, A.H, h);
            float hp[S];
#pragma unroll
            for (int q = 0; q < S; ++q) hp[q] = 0.f;
            if (t0 == 0) {
                if (A.h0) load_state<S>(A.h0, (size_t)b * A.H + h, hp);
            } else if (k > 0) {
                if (s == 0) {
#pragma unroll
                    for (int q = 0; q < S; ++q) hp[q] = side_in[((tile - nseq) * C + c) * S + q];
                } else {
                    Lay::h_prev(smem, s, c, hp);
                }
            }
            float Jr[L][S * S], rr[L][S], hc[L][S];
#pragma unroll
            for (int grp = 0; grp < L / 4; ++grp) {
                float pv[4][PW], hv[4][S];
                Lay::load_group(smem, s, c, grp, pv, hv, k > 0);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = grp * 4 + j;
                    const bool v = t0 + i < A.T;
                    float p[3];
#pragma unroll
                    for (int g = 0; g < 3; ++g) {
                        if (IN == 0) {
                            p[g] = pv[j][g];
                        } else {
                            float acc = bz[g];
#pragma unroll
                            for (int q = 0; q < (IN > 0 ? IN : 1); ++q) acc = fmaf(wz[g][q], pv[j][q % PW], acc);
                            p[g] = acc;
                        }
                    }
                    float cur[S], f[S], J[S * S];
#pragma unroll
                    for (int q = 0; q < S; ++q) cur[q] = k > 0 ? hv[j][q] : 0.f;
                    cell.eval(p, hp, f, J);
#pragma unroll
                    for (int q = 0; q < S; ++q) {
                        rr[i][q] = v ? f[q] - cur[q] : 0.f;
                        hc[i][q] = cur[q];
                        hp[q] = cur[q];
                    }
#pragma unroll
                    for (int q = 0; q < S * S; ++q) Jr[i][q] = v ? J[q] : ((q % (S + 1)) == 0 ? 1.f : 0.f);
                }
            }
            __syncthreads();  // the stage is consumed: refill it with the next tile
            const long next = tile + gridDim.x;
            if (next < ntiles) {
                const int nch = (int)(next / nseq);
                const long nsq = next - (long)nch * nseq;
                Lay::issue(A, smem, (int)(nsq / nct), (int)(nsq % nct), nch * TCH, k > 0);
                cp_async_commit();
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
            if (s_fail) {
                cp_async_wait_all();
                return;  // a bounded wait ran out; the status says so
            }
            float d[S];
            excl.apply(sm.carry[c], d);
#pragma unroll
            for (int i = 0; i < L; ++i) {
                const int t = t0 + i;
                float nd[S], hn[S];
                make_aff<S>(Jr[i], rr[i]).apply(d, nd);
#pragma unroll
                for (int q = 0; q < S; ++q) {
                    d[q] = nd[q];
                    hn[q] = hc[i][q] + nd[q];
                    const float ad = fabsf(nd[q]);
                    my_max = (ad > my_max || isnan(nd[q])) ? ad : my_max;
                }
                if (t < A.T) store_state<S>(A.h, ((size_t)b * A.T + t) * A.H + h, hn);
                if (i == L - 1 && s == SUB - 1 && chunk < nchunk - 1) {
#pragma unroll
                    for (int q = 0; q < S; ++q) side_out[(tile * C + c) * S + q] = hn[q];
                }
            }
            if (next >= ntiles) {
                // last tile of this iteration: prefetch this CTA's first tile for the next one
                __syncthreads();
                const int nch = (int)(blockIdx.x / nseq);
                const long nsq = blockIdx.x - (long)nch * nseq;
                Lay::issue(A, smem, (int)(nsq / nct), (int)(nsq % nct), nch * TCH, true);
                cp_async_commit();
            }
        }
        const unsigned bits = block_max_bits(my_max, s_red);
        if (tid == 0) atomicMax(&A.ctl->delta_bits[k % 3], bits);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) {
            cp_async_wait_all();
            return;
        }
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
    cp_async_wait_all();  // a speculative prefetch may still be in flight

    if (A.residual_out && !stop_all)
        if (!residual_pass<Cell, C, L, IN>(A, s_red)) return;
    if (blockIdx.x == 0 && tid == 0) {
        *A.iters_out = iters;
        if (A.delta_out) *A.delta_out = last_delta;
        if (!stop_all && A.tol > 0.f && iters == A.max_iters && !(last_delta < A.tol))
            atomicOr(A.sticky, kStNotConverged);
    }
}

// ------------------------------------------------------------------ host side
namespace {

template <class K> int prepare_kernel(K *kern, int smem_bytes) {
    if (cudaFuncSetAttribute(reinterpret_cast<const void *>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes) != cudaSuccess)
        return -1;
    return 0;
}

template <class Cell, class Lay, int IN> int choose(Plan *plan, int num_sms) {
    auto kern = &newton_staged_kernel<Cell, Lay, IN>;
    const int smem = Lay::SMEM_FLOATS * (int)sizeof(float);
    if (prepare_kernel(kern, smem)) return -1;
    plan->kernel = reinterpret_cast<const void *>(kern);
    plan->dyn_smem = smem;
    plan->grid = occupancy_grid(plan->kernel, kThreads, smem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

}  // namespace

// Staged kernels apply to H == 1 (long) or H % 32 == 0 with projected inputs (wide),
// with 16-byte aligned per-sequence slabs.  Returns 1 when the shape is not covered.
int newton_staged_plan(const NewtonDiagReq &r, int num_sms, Plan *plan) {
    const int S = r.cell == 1 ? 2 : 1;
    const int L = S == 1 ? 16 : 8;
    const bool fused = r.xproj == nullptr;
    if (r.H == 1) {
        const int PW = fused ? r.in : 3;
        if (fused && r.in != 1 && r.in != 2 && r.in != 4) return 1;
        if (((long)r.T * PW) % 4 || ((long)r.T * S) % 4) return 1;
        const int TCH = kThreads * L;
        plan->ntiles = (long)r.B * ((r.T + TCH - 1) / TCH);
        plan->variant = 101;
        int rc;
        if (S == 1) {
            rc = !fused ? choose<GruCell, LongLayout<GruCell, 0>, 0>(plan, num_sms)
                 : r.in == 1 ? choose<GruCell, LongLayout<GruCell, 1>, 1>(plan, num_sms)
                 : r.in == 2 ? choose<GruCell, LongLayout<GruCell, 2>, 2>(plan, num_sms)
                             : choose<GruCell, LongLayout<GruCell, 4>, 4>(plan, num_sms);
        } else {
            rc = !fused ? choose<LstmCell, LongLayout<LstmCell, 0>, 0>(plan, num_sms)
                 : r.in == 1 ? choose<LstmCell, LongLayout<LstmCell, 1>, 1>(plan, num_sms)
                 : r.in == 2 ? choose<LstmCell, LongLayout<LstmCell, 2>, 2>(plan, num_sms)
                             : choose<LstmCell, LongLayout<LstmCell, 4>, 4>(plan, num_sms);
        }
        if (rc) return -1;
        plan->C = 1;
    } else if (r.H % 32 == 0 && !fused) {
        const int TCH = (kThreads / 32) * L;
        plan->ntiles = (long)r.B * (r.H / 32) * ((r.T + TCH - 1) / TCH);
        plan->variant = 132;
        int rc = S == 1 ? choose<GruCell, WideLayout<GruCell>, 0>(plan, num_sms)
                        : choose<LstmCell, WideLayout<LstmCell>, 0>(plan, num_sms);
        if (rc) return -1;
        plan->C = 32;
    } else {
        return 1;
    }
    plan->agg_words = (size_t)plan->ntiles * plan->C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * plan->C * S;
    plan->side_bytes = 2 * (size_t)plan->ntiles * plan->C * S * sizeof(float);
    plan->epochs = (unsigned)r.max_iters + 1u;
    return 0;
}

}  // namespace prn
