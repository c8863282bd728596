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

// Padded stride (floats) for a per-thread segment of `seg` floats read as float4: the
// stride in 16-byte chunks must be odd so that a quarter-warp's 128-bit reads hit
// distinct bank groups.
constexpr int pad_stride(int seg) { return ((seg / 4) % 2 == 0) ? seg + 4 : seg + 8; }

// Shared memory the staged kernel uses beyond the input stage: per step and thread,
// the local prefix product Q (S*S floats), the local update D (S) and h^(k) (S),
// stored transposed ([component][step][thread]) so every access is conflict-free.
template <int S, int L> constexpr int park_floats() { return (S * S + 2 * S) * L * kThreads; }

// ---------------------------------------------------------------- long layout, H == 1
template <class Cell, int IN, int LL> struct LongLayout {
    static constexpr int S = Cell::S, C = 1, L = LL, SUB = kThreads, TCH = SUB * L;
    static constexpr int PW = IN == 0 ? 3 : IN;     // input floats per step
    static constexpr int SEGP = L * PW, STRP = pad_stride(SEGP);
    static constexpr int SEGH = L * S, STRH = pad_stride(SEGH);
    static constexpr int OFFH = SUB * STRP;
    static constexpr int SMEM_FLOATS = SUB * (STRP + STRH);
    static_assert(SEGP % 4 == 0 && SEGH % 4 == 0, "segments are whole 16-byte chunks");

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
    // Coalesced store of a finished tile: out[q][i][thread] (parked) -> h[b, tch0 .. +TCH).
    __device__ static void store_tile(const NewtonDiagArgs &A, const float *out, int b, int, int tch0) {
        const size_t row = (size_t)b * A.T;
        const int valid = min(TCH, A.T - tch0) * S;  // floats of this tile inside the sequence
        float *g = A.h + (row + tch0) * S;
        for (int f = 4 * threadIdx.x; f < valid; f += 4 * kThreads) {
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int fe = f + e, t = fe / S, q = fe % S;
                v[e] = out[(q * L + t % L) * kThreads + t / L];
            }
            if (f + 4 <= valid) {
                *reinterpret_cast<float4 *>(g + f) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
                for (int e = 0; f + e < valid; ++e) g[f + e] = v[e];
            }
        }
    }
};

// ---------------------------------------------------------------- wide layout, H % 32 == 0
template <class Cell, int LL> struct WideLayout {
    static constexpr int S = Cell::S, C = 32, L = LL, SUB = kThreads / C, TCH = SUB * L;
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
    // Coalesced store: each step is a 32 * S float row of the tile's channels.
    __device__ static void store_tile(const NewtonDiagArgs &A, const float *out, int b, int ct, int tch0) {
        const size_t row = (size_t)b * A.T;
        const int steps = min(TCH, A.T - tch0);
        for (int q = threadIdx.x; q < steps * 8 * S; q += kThreads) {
            const int t = q / (8 * S), part = q % (8 * S);
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int f = part * 4 + e, c = f / S, k = f % S;
                v[e] = out[(k * L + t % L) * kThreads + (t / L) * 32 + c];
            }
            *reinterpret_cast<float4 *>(A.h + ((row + tch0 + t) * A.H + ct * 32) * S + part * 4) =
                make_float4(v[0], v[1], v[2], v[3]);
        }
    }
};

template <class Cell, class Lay, int IN>
__global__ void __launch_bounds__(kThreads, PRN_STAGED_MINB) newton_staged_kernel(const NewtonDiagArgs A) {
    constexpr int S = Cell::S, C = Lay::C, L = Lay::L, SUB = Lay::SUB, TCH = Lay::TCH, PW = Lay::PW;
    constexpr int SS = S * S;
    static_assert(L % 4 == 0, "steps are read in groups of four");
    extern __shared__ __align__(16) float smem[];
    float *const park = smem + Lay::SMEM_FLOATS;  // [SS + 2S][L][kThreads]
    float *const parkQ = park, *const parkD = park + SS * L * kThreads, *const parkH = park + (SS + S) * L * kThreads;
    __shared__ ScanSmem<S, C> sm;
    __shared__ float s_carry[C][S];
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

        // the tile whose carry is still pending (its per-step values are parked)
        long ptile = -1;
        int pb = 0, pct = 0, pchunk = 0;
        Aff<S> pexcl = Aff<S>::ident(), ptotal = Aff<S>::ident();

        // Resolve the pending tile's carry (look-back), publish its inclusive value,
        // finish its states from the parked values and store them coalesced.
        auto finish_pending = [&]() -> bool {
            if (tid < 32) {
                float base[S], carry[S];
#pragma unroll
                for (int q = 0; q < S; ++q) base[q] = 0.f;  // delta entering t = 0 is 0
                if (!resolve_carry<S, C>(lb, ptile, pchunk, nseq, epoch, base, carry, A.ctl, A.sticky, A.dbg)) {
                    if (tid == 0) s_fail = 1;
                } else {
                    publish_inc<S, C>(lb, ptotal, carry, ptile, epoch, A.dbg);
                    if (tid < C) {
#pragma unroll
                        for (int q = 0; q < S; ++q) s_carry[tid][q] = carry[q];
                    }
                }
            }
            __syncthreads();
            if (s_fail) return false;
            float din[S];
            pexcl.apply(s_carry[c], din);
            const int t0 = pchunk * TCH + s * L;
#pragma unroll
            for (int i = 0; i < L; ++i) {
                float qm[SS], dv[S], hv[S];
#pragma unroll
                for (int q = 0; q < SS; ++q) qm[q] = parkQ[(q * L + i) * kThreads + tid];
#pragma unroll
                for (int q = 0; q < S; ++q) {
                    dv[q] = parkD[(q * L + i) * kThreads + tid];
                    hv[q] = parkH[(q * L + i) * kThreads + tid];
                }
                float out[S];
#pragma unroll
                for (int r = 0; r < S; ++r) {
                    float d = dv[r];
#pragma unroll
                    for (int q = 0; q < S; ++q) d = fmaf(qm[r * S + q], din[q], d);
                    out[r] = hv[r] + d;
                    if (t0 + i < A.T) {
                        const float ad = fabsf(d);
                        my_max = (ad > my_max || isnan(d)) ? ad : my_max;
                    }
                    parkH[(r * L + i) * kThreads + tid] = out[r];
                }
                if (i == L - 1 && s == SUB - 1 && pchunk < nchunk - 1) {
#pragma unroll
                    for (int q = 0; q < S; ++q) side_out[(ptile * C + c) * S + q] = out[q];
                }
            }
            __syncthreads();
            Lay::store_tile(A, parkH, pb, pct, pchunk * TCH);
            __syncthreads();
            return true;
        };

        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const int chunk = (int)(tile / nseq);
            const long seq = tile - (long)chunk * nseq;
            const int b = (int)(seq / nct);
            const int ct = (int)(seq % nct);
            const int h = ct * C + c;
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
            // local walk with zero carry: Q_i = J_i..J_0, D_i = local update after step i
            float Qv[L][SS], Dv[L][S], Hv[L][S];
            float Qc[SS], Dc[S];
#pragma unroll
            for (int q = 0; q < SS; ++q) Qc[q] = (q % (S + 1)) == 0 ? 1.f : 0.f;
#pragma unroll
            for (int q = 0; q < S; ++q) Dc[q] = 0.f;
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
                    float cur[S], f[S], J[SS];
#pragma unroll
                    for (int q = 0; q < S; ++q) cur[q] = k > 0 ? hv[j][q] : 0.f;
                    cell.eval(p, hp, f, J);
                    if (v) {
                        float nQ[SS], nD[S];
#pragma unroll
                        for (int r = 0; r < S; ++r) {
                            float dd = f[r] - cur[r];
#pragma unroll
                            for (int q = 0; q < S; ++q) dd = fmaf(J[r * S + q], Dc[q], dd);
                            nD[r] = dd;
#pragma unroll
                            for (int q2 = 0; q2 < S; ++q2) {
                                float acc = 0.f;
#pragma unroll
                                for (int q = 0; q < S; ++q) acc = fmaf(J[r * S + q], Qc[q * S + q2], acc);
                                nQ[r * S + q2] = acc;
                            }
                        }
#pragma unroll
                        for (int q = 0; q < SS; ++q) Qc[q] = nQ[q];
#pragma unroll
                        for (int q = 0; q < S; ++q) Dc[q] = nD[q];
                    }
#pragma unroll
                    for (int q = 0; q < SS; ++q) Qv[i][q] = Qc[q];
#pragma unroll
                    for (int q = 0; q < S; ++q) {
                        Dv[i][q] = Dc[q];
                        Hv[i][q] = cur[q];
                        hp[q] = cur[q];
                    }
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
            Aff<S> e = make_aff<S>(Qc, Dc);
            Aff<S> excl, total;
            cta_scan<S, C>(e, sm, excl, total);
            if (tid < 32) publish_agg<S, C>(lb, total, tile, chunk, epoch, A.dbg);
            // the previous tile's look-back has had a whole tile of time to become ready
            if (ptile >= 0 && !finish_pending()) {
                cp_async_wait_all();
                return;
            }
            // park this tile's per-step values
#pragma unroll
            for (int i = 0; i < L; ++i) {
#pragma unroll
                for (int q = 0; q < SS; ++q) parkQ[(q * L + i) * kThreads + tid] = Qv[i][q];
#pragma unroll
                for (int q = 0; q < S; ++q) {
                    parkD[(q * L + i) * kThreads + tid] = Dv[i][q];
                    parkH[(q * L + i) * kThreads + tid] = Hv[i][q];
                }
            }
            ptile = tile;
            pb = b;
            pct = ct;
            pchunk = chunk;
            pexcl = excl;
            ptotal = total;
            if (next >= ntiles) {
                // last tile of this iteration: finish it now, then prefetch this CTA's
                // first tile for the next iteration
                __syncthreads();
                if (!finish_pending()) {
                    cp_async_wait_all();
                    return;
                }
                ptile = -1;
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

template <class Cell, class Lay, int IN> int choose(Plan *plan, int num_sms, long B, long T, long H) {
    auto kern = &newton_staged_kernel<Cell, Lay, IN>;
    const int smem = (Lay::SMEM_FLOATS + park_floats<Lay::S, Lay::L>()) * (int)sizeof(float);
    if (prepare_kernel(kern, smem)) return -1;
    plan->kernel = reinterpret_cast<const void *>(kern);
    plan->dyn_smem = smem;
    plan->C = Lay::C;
    plan->ntiles = B * (H / Lay::C) * ((T + Lay::TCH - 1) / Lay::TCH);
    plan->grid = occupancy_grid(plan->kernel, kThreads, smem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

}  // namespace

// Staged kernels apply to H == 1 (long) or H % 32 == 0 with projected inputs (wide),
// with 16-byte aligned per-sequence slabs.  Returns 1 when the shape is not covered.
// Steps per thread (L) are chosen so that the input stage and the parked values of
// two CTAs fit one SM's shared memory.
int newton_staged_plan(const NewtonDiagReq &r, int num_sms, Plan *plan) {
    const int S = r.cell == 1 ? 2 : 1;
    const bool fused = r.xproj == nullptr;
    int rc;
    if (r.H == 1) {
        const int PW = fused ? r.in : 3;
        if (fused && r.in != 1 && r.in != 2 && r.in != 4) return 1;
        if (((long)r.T * PW) % 4 || ((long)r.T * S) % 4) return 1;
        plan->variant = 101;
        if (S == 1) {
            rc = !fused ? choose<GruCell, LongLayout<GruCell, 0, 8>, 0>(plan, num_sms, r.B, r.T, r.H)
                 : r.in == 1 ? choose<GruCell, LongLayout<GruCell, 1, 16>, 1>(plan, num_sms, r.B, r.T, r.H)
                 : r.in == 2 ? choose<GruCell, LongLayout<GruCell, 2, 16>, 2>(plan, num_sms, r.B, r.T, r.H)
                             : choose<GruCell, LongLayout<GruCell, 4, 8>, 4>(plan, num_sms, r.B, r.T, r.H);
        } else {
            rc = !fused ? choose<LstmCell, LongLayout<LstmCell, 0, 4>, 0>(plan, num_sms, r.B, r.T, r.H)
                 : r.in == 1 ? choose<LstmCell, LongLayout<LstmCell, 1, 8>, 1>(plan, num_sms, r.B, r.T, r.H)
                 : r.in == 2 ? choose<LstmCell, LongLayout<LstmCell, 2, 8>, 2>(plan, num_sms, r.B, r.T, r.H)
                             : choose<LstmCell, LongLayout<LstmCell, 4, 4>, 4>(plan, num_sms, r.B, r.T, r.H);
        }
    } else if (r.H % 32 == 0 && !fused) {
        plan->variant = 132;
        rc = S == 1 ? choose<GruCell, WideLayout<GruCell, 12>, 0>(plan, num_sms, r.B, r.T, r.H)
                    : choose<LstmCell, WideLayout<LstmCell, 8>, 0>(plan, num_sms, r.B, r.T, r.H);
    } else {
        return 1;
    }
    if (rc) return -1;
    plan->agg_words = (size_t)plan->ntiles * plan->C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * plan->C * S;
    plan->side_bytes = 2 * (size_t)plan->ntiles * plan->C * S * sizeof(float);
    plan->epochs = (unsigned)r.max_iters + 1u;
    return 0;
}

}  // namespace prn
