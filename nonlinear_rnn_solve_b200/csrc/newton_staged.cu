// newton_staged.cu -- Newton (DEER) forward for ParaGRU / ParaLSTM with each tile's
// inputs staged in shared memory ahead of use, so that the HBM reads of the next tile
// overlap the scan, look-back and stores of the current one.
//
// Same method as newton_diag.cu ("Parallelizing non-linear sequential models over
// the sequence length", Approach: linearise, then solve the linear recurrence with a
// parallel prefix scan), specialised for the shapes that carry the traffic:
//   TmaLong (H == 1, raw inputs of width <= 4): one thread streams the tile's inputs
//         and states with 2-D TMA copies into 128-byte-swizzled shared memory; every
//         thread reads its L consecutive steps as conflict-free 128-bit loads; results
//         go through a swizzled staging tile and leave as coalesced 16-byte stores;
//   CpLong (other H == 1 shapes): cp.async copies into padded per-thread segments;
//   Wide  (H % 32 == 0, projected inputs given): a tile is 32 channels x 8 sub-chunks
//         of L steps; every step is a 128-byte row per gate and per state.
// A tile whose steps all lie inside the sequence takes a path without per-step guards.
#include <cuda.h>
#include <string.h>

#include <algorithm>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"
#include "newton_common.cuh"
#include "staged_tiles.cuh"

#ifndef PRN_STAGED_MINB
#define PRN_STAGED_MINB 2  // resident CTAs per SM the register budget is sized for
#endif
#ifndef PRN_LONG_GRU_L
#define PRN_LONG_GRU_L 16  // steps per thread of the TMA-fed H = 1 ParaGRU tiles
#endif
#ifndef PRN_LONG_NT
#define PRN_LONG_NT 256  // threads per CTA of the TMA-fed H = 1 ParaGRU tiles
#endif
#ifndef PRN_LONG_MINB
#define PRN_LONG_MINB PRN_STAGED_MINB  // resident CTAs per SM for those tiles
#endif
#ifndef PRN_LONG_HALO
#define PRN_LONG_HALO 64  // steps before each H = 1 ParaGRU tile that the tile evaluates itself
#endif

// A halo's composed map delta -> a delta + d is taken as the constant d (the carry) when
// every entry of a is at most 2^-40 in magnitude: the dropped a delta is at most 2^-40
// times the delta entering the halo, far below the fp32 resolution of the states it
// updates (with a = 0 exactly, d is the value the scan would carry in, up to rounding
// order).  On the contractive ParaGRU inputs 63 steps bring a below 2^-64.
constexpr float kHaloConstTol = 0x1p-40f;

namespace prn {

// ---------------------------------------------------------------- cp.async long layout, H == 1
template <class Cell, int IN, int LL, int NT> struct CpLong {
    static constexpr int S = Cell::S, C = 1, L = LL, SUB = NT, TCH = SUB * L;
    static constexpr int PW = IN == 0 ? 3 : IN;  // input floats per step
    static constexpr int SEGP = L * PW, STRP = pad_stride(SEGP);
    static constexpr int SEGH = L * S, STRH = pad_stride(SEGH);
    static constexpr int OFFH = SUB * STRP;
    static constexpr int SMEM_FLOATS = SUB * (STRP + STRH);
    static constexpr int OUT_STRIDE = 0;
    static constexpr bool kTma = false;
    __device__ static void prefetch(const NewtonDiagArgs &, const StagedMaps &, int, int, bool) {}
    static constexpr int HALO = 0;
    static_assert(SEGP % 4 == 0 && SEGH % 4 == 0, "segments are whole 16-byte chunks");

    __device__ static void issue(const NewtonDiagArgs &A, const StagedMaps &, float *sm, unsigned long long *, int b,
                                 int, int tch0, bool with_h) {
        const size_t row = (size_t)b * A.T;
        const float *pin = IN == 0 ? A.xproj : A.x;
        copy_segments<NT>(sm, SEGP, STRP, pin + (row + tch0) * PW, TCH * PW, pin + (row + A.T) * PW);
        if (with_h)
            copy_segments<NT>(sm + OFFH, SEGH, STRH, A.h + (row + tch0) * S, TCH * S, A.h + (row + A.T) * S);
        cp_async_commit();
    }
    __device__ static void load_group(float *sm, int s, int, int grp, float pv[4][PW], float hv[4][S], bool with_h) {
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
    __device__ static void h_prev(float *sm, int s, int, float *hp) {
#pragma unroll
        for (int q = 0; q < S; ++q) hp[q] = sm[OFFH + (s - 1) * STRH + SEGH - S + q];
    }
    __device__ static void put_group(const NewtonDiagArgs &A, float *, int, int, int, const float hn[4][S], int b,
                                     int t, int) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (t + j < A.T) store_state<S>(A.h, (size_t)b * A.T + t + j, hn[j]);
    }
    __device__ static void flush(const NewtonDiagArgs &, float *, int, int, int) {}
};

// ---------------------------------------------------------------- wide layout, H % 32 == 0
template <class Cell, int LL, int NT> struct Wide {
    static constexpr int S = Cell::S, C = 32, L = LL, SUB = NT / C, TCH = SUB * L;
    static constexpr int PW = 3;
    static constexpr int ROWP = 3 * 32, ROWH = 32 * S;
    static constexpr int OFFH = TCH * ROWP;
    static constexpr int SMEM_FLOATS = TCH * (ROWP + ROWH);
    static constexpr int OUT_STRIDE = 0;
    static constexpr bool kTma = false;
    __device__ static void prefetch(const NewtonDiagArgs &, const StagedMaps &, int, int, bool) {}
    static constexpr int HALO = 0;

    __device__ static void issue(const NewtonDiagArgs &A, const StagedMaps &, float *sm, unsigned long long *, int b,
                                 int ct, int tch0, bool with_h) {
        const size_t row = (size_t)b * A.T;
        for (int q = threadIdx.x; q < TCH * 3 * 8; q += NT) {
            const int r = q >> 3, part = q & 7, t = r / 3, g = r % 3;
            const bool v = tch0 + t < A.T;
            const float *gp = A.xproj + ((row + tch0 + (v ? t : 0)) * 3 + g) * A.H + ct * 32 + part * 4;
            cp_async16(sm + r * 32 + part * 4, gp, v ? 16 : 0);
        }
        if (with_h) {
            for (int q = threadIdx.x; q < TCH * 8 * S; q += NT) {
                const int t = q / (8 * S), part = q % (8 * S);
                const bool v = tch0 + t < A.T;
                const float *gp = A.h + ((row + tch0 + (v ? t : 0)) * A.H + ct * 32) * S + part * 4;
                cp_async16(sm + OFFH + t * ROWH + part * 4, gp, v ? 16 : 0);
            }
        }
        cp_async_commit();
    }
    __device__ static void load_group(float *sm, int s, int c, int grp, float pv[4][PW], float hv[4][S], bool with_h) {
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
    __device__ static void h_prev(float *sm, int s, int c, float *hp) {
#pragma unroll
        for (int q = 0; q < S; ++q) hp[q] = sm[OFFH + (s * L - 1) * ROWH + c * S + q];
    }
    // a warp writes 32 consecutive channels of one step: already coalesced
    __device__ static void put_group(const NewtonDiagArgs &A, float *, int, int, int, const float hn[4][S], int b,
                                     int t, int h) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (t + j < A.T) store_state<S>(A.h, ((size_t)b * A.T + t + j) * A.H + h, hn[j]);
    }
    __device__ static void flush(const NewtonDiagArgs &, float *, int, int, int) {}
};

// One tile's compute phase: f, J and the residual for the thread's L steps, read from
// the staged slab.  FULL: every step lies inside the sequence (no guards).
template <class Cell, class Lay, int IN, bool FULL, bool JM>
__device__ __forceinline__ void tile_compute(const NewtonDiagArgs &A, float *smem, const Cell &cell, int s, int c,
                                             int t0, int k, float *hp, const float (&wz)[3][IN > 0 ? IN : 1],
                                             const float (&bz)[3], float (&Jr)[Lay::L][Cell::S * Cell::S],
                                             float (&rr)[Lay::L][Cell::S], float (&hc)[Lay::L][Cell::S]) {
    constexpr int S = Cell::S, L = Lay::L, PW = Lay::PW;
#pragma unroll
    for (int grp = 0; grp < L / 4; ++grp) {
        float pv[4][PW], hv[4][S];
        Lay::load_group(smem, s, c, grp, pv, hv, k > 0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = grp * 4 + j;
            const bool v = FULL || t0 + i < A.T;
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
            if (IN > 0)
                cell.eval_pre(p, hp, f, J);  // p was formed with the prescaled weights
            else
                cell.eval(p, hp, f, J);
            if (JM) apply_jmode<S>(A.jmode, J);  // JM: a linearisation other than the Jacobian
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
}

template <class Cell, class Lay, int IN, int NT, int MINB>
__global__ void __launch_bounds__(NT, MINB)
    newton_staged_kernel(const NewtonDiagArgs A, const __grid_constant__ StagedMaps M) {
    constexpr int S = Cell::S, C = Lay::C, L = Lay::L, SUB = Lay::SUB, TCH = Lay::TCH;
    constexpr int HALO = Lay::HALO, HW = HALO > 0 ? HALO : 1;
    static_assert(L % 4 == 0, "steps are handled in groups of four");
    static_assert(HALO == 0 || (HALO % 32 == 0 && HALO <= NT && HALO % L == 0 && IN > 0 && C == 1),
                  "a halo is one step per thread of whole warps, covers whole segments, raw inputs, H = 1");
    extern __shared__ __align__(1024) unsigned char smraw[];
    float *const smem = reinterpret_cast<float *>(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    // scan exchange and halo totals alternate between two copies by tile parity: a
    // warp may start the next tile while others still read this tile's copy (the tile
    // loop has one CTA barrier per tile on the common path)
    __shared__ ScanSmem<S, C, NT> sm2[2];
    __shared__ unsigned s_red[NT / 32];
    __shared__ int s_fail;
    __shared__ __align__(8) unsigned long long s_bar;
    __shared__ Aff<S> s_halo[2][HALO > 0 ? HALO / 32 : 1];
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = A.H / C;
    const int nseq = A.B * nct;  // the plan keeps tile counts below 2^31
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = (long)nseq * nchunk;
    // tile = chunk * nseq + seq advances by gridDim.x: (chunk, seq) are stepped without
    // dividing in the loop
    const int step_ch = (int)(gridDim.x / (unsigned)nseq), step_sq = (int)(gridDim.x % (unsigned)nseq);
    const int first_ch = (int)(blockIdx.x / (unsigned)nseq), first_sq = (int)(blockIdx.x % (unsigned)nseq);
    auto advance = [&](int &ch, int &sq) {
        ch += step_ch;
        sq += step_sq;
        if (sq >= nseq) {
            sq -= nseq;
            ++ch;
        }
    };
    // side buffers (two parities): the last HW states that every tile but a sequence's
    // last wrote in the previous iteration.  They are the current iterate for the
    // successor (its halo and first step), which must not read them from h: the
    // tile may already be overwriting them there.
    const size_t side_stride = (size_t)ntiles * C * HW * S;
    LookBack<S> lb{A.agg, A.inc};
    unsigned bar_phase = 0;
    if (tid == 0) {
        s_fail = 0;
        if (Lay::kTma) {
            mbar_init(&s_bar, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
    }
    __syncthreads();

    // fused projection weights (raw inputs, H == 1): p_g = bias_g + sum_q W[g][q] x_q
    float wz[3][IN > 0 ? IN : 1], bz[3];
#pragma unroll
    for (int g = 0; g < 3; ++g) {
        bz[g] = 0.f;
#pragma unroll
        for (int q = 0; q < (IN > 0 ? IN : 1); ++q) wz[g][q] = 0.f;
        if (IN > 0) {
            // folded into the cell's exponent scale (Cell::pre): the cell takes q = pre * p
            bz[g] = A.bias ? Cell::pre(g) * __ldg(A.bias + g * A.H) : 0.f;
#pragma unroll
            for (int q = 0; q < (IN > 0 ? IN : 1); ++q) wz[g][q] = Cell::pre(g) * __ldg(A.W + (size_t)g * A.H * IN + q);
        }
    }

    // Issue a tile's copies.  Data this CTA wrote with ordinary stores is made visible
    // to the TMA (async proxy) with proxy fences after the preceding barrier.
    auto issue = [&](int ch, int sq, bool with_h) {
        const int ib = Lay::C == 1 ? sq : sq / nct, ict = Lay::C == 1 ? 0 : sq % nct;  // C == 1: H == 1
        if (Lay::kTma) {
            if (tid == 0) {
                asm volatile("fence.proxy.async.global;" ::: "memory");
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                Lay::issue(A, M, smem, &s_bar, ib, ict, ch * TCH, with_h);
            }
        } else {
            Lay::issue(A, M, smem, &s_bar, ib, ict, ch * TCH, with_h);
        }
    };
    // Wait for the staged tile (bounded).  TMA: every thread waits on the mbarrier
    // itself (no CTA barrier); false when the wait gave up, which the caller turns
    // into a CTA-wide stop at the next barrier.  cp.async: each thread's copies serve
    // other threads, so a CTA barrier follows.
    auto wait_stage = [&]() -> bool {
        if (Lay::kTma) {
            bool ok = mbar_try(&s_bar, bar_phase);
            if (!ok) {
                const unsigned long long t0 = gtimer();
                while (!(ok = mbar_try(&s_bar, bar_phase))) {
                    if (ld_relaxed_int(&A.ctl->abort)) break;
                    if (gtimer() - t0 > A.dbg.wait_ns) {
                        raise_status(A.sticky, A.ctl, kStTimeout, true);
                        break;
                    }
                }
            }
            if (ok) bar_phase ^= 1u;  // on failure drain() waits for the pending phase
            return ok;
        }
        cp_async_wait_all();
        __syncthreads();
        return true;
    };
    // On an abort, let a TMA copy that is still in flight land before the CTA exits
    // (bounded like every wait).
    auto drain = [&]() {
        if (Lay::kTma) {
            const unsigned long long t0 = gtimer();
            while (!mbar_try(&s_bar, bar_phase) && gtimer() - t0 < A.dbg.wait_ns) {
            }
        } else {
            cp_async_wait_all();
        }
    };
    issue(first_ch, first_sq, false);
    Cell cell;
    if (C == 1) cell.load(A.a, A.peep, A.H, 0);  // C == 1 layouts are H == 1: one unit

    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epoch = A.epoch0 + (unsigned)k + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        const float *side_in = A.side + (size_t)(k & 1) * side_stride;
        float *side_out = A.side + (size_t)((k + 1) & 1) * side_stride;
        float my_max = 0.f;
        bool my_bad = false;
        int chunk = first_ch, seq = first_sq;
        int par = 0;                    // tile parity within the iteration
        int fl_b = -1, fl_ct = 0, fl_t = 0;  // staged results still to be written (previous tile)
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, advance(chunk, seq), par ^= 1) {
            ScanSmem<S, C, NT> &sm = sm2[Lay::kTma ? par : 0];  // cp.async layouts keep a barrier after the scan
            const int b = C == 1 ? seq : seq / nct;
            const int ct = C == 1 ? 0 : seq % nct;
            const int h = ct * C + c;
            const int tch0 = chunk * TCH;
            const int t0 = tch0 + s * L;
            // halo: thread tid < HALO evaluates step tch0 - HALO + tid (the first only
            // supplies the state before the second); loads start before the stage wait
            const bool use_halo = HALO > 0 && chunk > 0 && !A.dbg.no_halo;
            float hx[IN > 0 ? IN : 1], hcur[S], hprv[S];
            if (HALO > 0 && use_halo && tid < HALO) {
                const float *xr = A.x + ((size_t)b * A.T + (tch0 - HALO + tid)) * (IN > 0 ? IN : 1);
                if (IN == 2) {
                    const float2 v = *reinterpret_cast<const float2 *>(xr);
                    hx[0] = v.x;
                    hx[1 % (IN > 0 ? IN : 1)] = v.y;
                } else if (IN == 4) {
                    const float4 v = *reinterpret_cast<const float4 *>(xr);
                    hx[0] = v.x;
                    hx[1 % (IN > 0 ? IN : 1)] = v.y;
                    hx[2 % (IN > 0 ? IN : 1)] = v.z;
                    hx[3 % (IN > 0 ? IN : 1)] = v.w;
                } else {
#pragma unroll
                    for (int q = 0; q < (IN > 0 ? IN : 1); ++q) hx[q] = xr[q];
                }
                const float *sp = side_in + (size_t)(tile - nseq) * HW * S;
#pragma unroll
                for (int q = 0; q < S; ++q) {
                    hcur[q] = k > 0 ? sp[tid * S + q] : 0.f;
                    hprv[q] = (k > 0 && tid > 0) ? sp[(tid - 1) * S + q] : 0.f;
                }
            }
            if (!wait_stage()) s_fail = 1;  // acted on after the scan's barrier
            if (Lay::kTma && tid == 32) {
                // L2 prefetch of the tile whose load issue() starts after this tile's scan
                int nch = chunk, nsq = seq;
                bool wh = k > 0;
                if (tile + gridDim.x < ntiles) {
                    advance(nch, nsq);
                } else {
                    nch = first_ch;
                    nsq = first_sq;
                    wh = true;
                }
                Lay::prefetch(A, M, C == 1 ? nsq : nsq / nct, nch * TCH, wh);
            }
            if (C != 1) cell.load(A.a, A.peep, A.H, h);
            if (HALO > 0 && use_halo && tid < HALO) {
                Aff<S> he = Aff<S>::ident();
                if (tid > 0) {
                    float p[3], f[S], J[S * S], r[S];
#pragma unroll
                    for (int g = 0; g < 3; ++g) {
                        float acc = bz[g];
#pragma unroll
                        for (int q = 0; q < (IN > 0 ? IN : 1); ++q) acc = fmaf(wz[g][q], hx[q], acc);
                        p[g] = acc;
                    }
                    cell.eval_pre(p, hprv, f, J);
                    apply_jmode<S>(A.jmode, J);  // the halo linearises like the tile
#pragma unroll
                    for (int q = 0; q < S; ++q) r[q] = f[q] - hcur[q];
                    he = make_aff<S>(J, r);
                }
                // ordered composition of the warp's 32 steps, into lane 0
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const Aff<S> o = he.shfl_down(off);
                    if ((tid & 31) + off < 32) he = compose(he, o);
                }
                if ((tid & 31) == 0) s_halo[par][tid >> 5] = he;  // read after the scan's barrier
            }
            float hp[S];
#pragma unroll
            for (int q = 0; q < S; ++q) hp[q] = 0.f;
            if (t0 == 0) {
                if (A.h0) load_state<S>(A.h0, (size_t)b * A.H + h, hp);
            } else if (k > 0) {
                if (s == 0) {
#pragma unroll
                    for (int q = 0; q < S; ++q) hp[q] = side_in[(((tile - nseq) * C + c) * HW + HW - 1) * S + q];
                } else {
                    Lay::h_prev(smem, s, c, hp);
                }
            }
            float Jr[L][S * S], rr[L][S], hc[L][S];
            // the tile-uniform choices (whole tile inside the sequence, linearisation)
            // select code paths here, not per step
            const bool full = tch0 + TCH <= A.T;
            if (A.jmode == 0) {
                if (full)
                    tile_compute<Cell, Lay, IN, true, false>(A, smem, cell, s, c, t0, k, hp, wz, bz, Jr, rr, hc);
                else
                    tile_compute<Cell, Lay, IN, false, false>(A, smem, cell, s, c, t0, k, hp, wz, bz, Jr, rr, hc);
            } else {
                if (full)
                    tile_compute<Cell, Lay, IN, true, true>(A, smem, cell, s, c, t0, k, hp, wz, bz, Jr, rr, hc);
                else
                    tile_compute<Cell, Lay, IN, false, true>(A, smem, cell, s, c, t0, k, hp, wz, bz, Jr, rr, hc);
            }
            const long next = tile + gridDim.x;
            auto refill = [&]() {
                if (next < ntiles) {
                    int nch = chunk, nsq = seq;
                    advance(nch, nsq);
                    issue(nch, nsq, k > 0);
                }
            };
            Aff<S> e = Aff<S>::ident();
#pragma unroll
            for (int i = 0; i < L; ++i) e = compose(e, make_aff<S>(Jr[i], rr[i]));
            Aff<S> excl, total;
            cta_scan<S, C, NT>(e, sm, excl, total);  // the one CTA barrier of the TMA path
            if (s_fail) {
                drain();
                return;  // a bounded wait ran out; the status says so
            }
            // past the barrier every thread is done reading the stage: refill it
            refill();
            // the previous tile's staged results (written before the barrier) leave now
            if (fl_b >= 0) Lay::flush(A, smem + (par ^ 1) * Lay::OUT_STRIDE, fl_b, fl_ct, fl_t);
            // carry entering the tile: from the halo when its composed map is a constant up
            // to 2^-40 (every thread composes the same totals, so the branch is CTA-uniform),
            // else from the look-back by warp 0 and a second barrier
            float carry[S];
#pragma unroll
            for (int q = 0; q < S; ++q) carry[q] = 0.f;  // a sequence's first tile: delta entering t = 0 is 0
            bool known = chunk == 0;
            if (HALO > 0 && use_halo) {
                Aff<S> hall = s_halo[par][0];
#pragma unroll
                for (int w = 1; w < HW / 32; ++w) hall = compose(hall, s_halo[par][w]);
                float hv[Aff<S>::kFloats];
                hall.to_floats(hv);
                known = true;
#pragma unroll
                for (int q = 0; q < S * S; ++q) known = known && fabsf(hv[q]) <= kHaloConstTol;
#pragma unroll
                for (int q = 0; q < S; ++q) carry[q] = hv[S * S + q];
            }
            if (known) {
                if (tid < 32) {  // keep the look-back words complete for tiles that need them
                    publish_agg<S, C>(lb, total, tile, chunk, epoch, A.dbg);
                    publish_inc<S, C>(lb, total, carry, tile, epoch, A.dbg);
                }
            } else {
                if (tid < 32) {
                    float base[S];
#pragma unroll
                    for (int q = 0; q < S; ++q) base[q] = 0.f;  // delta entering t = 0 is 0
                    if (!look_back<S, C, NT>(lb, sm, total, tile, chunk, nseq, epoch, base, A.ctl, A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();
                if (s_fail) {
                    drain();
                    return;  // a bounded wait ran out; the status says so
                }
#pragma unroll
                for (int q = 0; q < S; ++q) carry[q] = sm.carry[c][q];
            }
            float d[S];
            excl.apply(carry, d);
#pragma unroll
            for (int grp = 0; grp < L / 4; ++grp) {
                float hn[4][S];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = grp * 4 + j;
                    float nd[S];
                    make_aff<S>(Jr[i], rr[i]).apply(d, nd);
#pragma unroll
                    for (int q = 0; q < S; ++q) {
                        d[q] = nd[q];
                        hn[j][q] = hc[i][q] + nd[q];
                        my_max = fmaxf(my_max, fabsf(nd[q]));
                    }
                }
                Lay::put_group(A, smem + par * Lay::OUT_STRIDE, s, c, grp, hn, b, t0 + grp * 4, h);
                if (HALO > 0) {
                    constexpr int FIRST = SUB - HALO / L;  // first thread whose steps the successor's halo covers
                    if (s >= FIRST && chunk < nchunk - 1) {
                        float4 *so = reinterpret_cast<float4 *>(side_out + ((size_t)tile * HW + (s - FIRST) * L + grp * 4) * S);
#pragma unroll
                        for (int u = 0; u < S; ++u)
                            so[u] = make_float4(hn[(4 * u) / S][(4 * u) % S], hn[(4 * u + 1) / S][(4 * u + 1) % S],
                                                hn[(4 * u + 2) / S][(4 * u + 2) % S], hn[(4 * u + 3) / S][(4 * u + 3) % S]);
                    }
                } else if (grp == L / 4 - 1 && s == SUB - 1 && chunk < nchunk - 1) {
#pragma unroll
                    for (int q = 0; q < S; ++q) side_out[(tile * C + c) * S + q] = hn[3][q];
                }
            }
            // a NaN or Inf anywhere in the segment reaches its last update (each update
            // feeds the next through J), where it is caught
#pragma unroll
            for (int q = 0; q < S; ++q) my_bad |= !finitef(d[q]);
            fl_b = b;
            fl_ct = ct;
            fl_t = tch0;
            if (!Lay::kTma && next >= ntiles) {
                // cp.async layouts: prefetch this CTA's first tile for the next iteration
                // (their stores went straight to h; the barrier orders them before the copies)
                __syncthreads();
                issue(first_ch, first_sq, true);
            }
        }
        // the last tile's staged results
        __syncthreads();
        if (fl_b >= 0) Lay::flush(A, smem + (par ^ 1) * Lay::OUT_STRIDE, fl_b, fl_ct, fl_t);
        const unsigned bits = block_max_bits<NT>(my_bad ? __int_as_float(0x7fc00000) : my_max, s_red);
        if (tid == 0) atomicMax(&A.ctl->delta_bits[k % 3], bits);
        // prefetch this CTA's first tile for the next iteration: past the barriers of the
        // block max, all of this CTA's stores to it are done (no other CTA writes it)
        if (Lay::kTma) issue(first_ch, first_sq, true);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) {
            drain();
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
    // a speculative prefetch may still be in flight
    if (Lay::kTma) {
        if (!wait_stage()) return;
    } else {
        cp_async_wait_all();
    }

    if (A.residual_out && !stop_all)
        if (!residual_pass<Cell, C, L, IN, NT>(A, s_red)) return;
    if (blockIdx.x == 0 && tid == 0) {
        *A.iters_out = iters;
        if (A.delta_out) *A.delta_out = last_delta;
        if (!stop_all && A.tol > 0.f && iters == A.max_iters && !(last_delta < A.tol))
            atomicOr(A.sticky, kStNotConverged);
    }
}

// ------------------------------------------------------------------ host side
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// fp32 tensor of `floats` elements viewed as rows of 32 floats; boxes of box_rows rows.
bool map_rows(CUtensorMap *map, const float *ptr, long floats, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || floats % 32) return false;
    cuuint64_t dims[2] = {32, (cuuint64_t)(floats / 32)};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class K> int prepare_kernel(K *kern, int smem_bytes) {
    const void *f = reinterpret_cast<const void *>(kern);
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess ||
        cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return -1;
    return 0;
}

template <class Cell, class Lay, int IN, int NT = kThreads, int MINB = PRN_STAGED_MINB>
int choose(Plan *plan, int num_sms, long B, long T, long H) {
    auto kern = &newton_staged_kernel<Cell, Lay, IN, NT, MINB>;
    const int smem = Lay::SMEM_FLOATS * (int)sizeof(float) + 1024;
    if (prepare_kernel(kern, smem)) return -1;
    plan->kernel = reinterpret_cast<const void *>(kern);
    plan->dyn_smem = smem;
    plan->C = Lay::C;
    plan->tch = Lay::TCH;
    plan->ntiles = B * (H / Lay::C) * ((T + Lay::TCH - 1) / Lay::TCH);
    plan->threads = NT;
    plan->halo_w = Lay::HALO > 0 ? Lay::HALO : 1;
    plan->grid = occupancy_grid(plan->kernel, NT, smem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

}  // namespace

// Staged kernels apply to H == 1 (long) or H % 32 == 0 with projected inputs (wide),
// with 16-byte aligned per-sequence slabs.  Returns 1 when the shape is not covered.
int newton_staged_plan(const NewtonDiagReq &r, int num_sms, Plan *plan) {
    const int S = r.cell == 1 ? 2 : 1;
    const bool fused = r.xproj == nullptr;
    int rc;
    plan->staged_tma = 0;
    if (r.H == 1) {
        const int PW = fused ? r.in : 3;
        if (fused && r.in != 1 && r.in != 2 && r.in != 4) return 1;
        if (((long)r.T * PW) % 4 || ((long)r.T * S) % 4) return 1;
        plan->variant = 101;
        // TMA needs every sequence's input and state slabs to start on a 128-byte row
        const bool tma = fused && ((long)r.T * PW) % 32 == 0 && ((long)r.T * S) % 32 == 0;
        if (S == 1) {
            if (tma)
                rc = r.in == 1
                         ? choose<GruCell, TmaLong<GruCell, 1, 16, kThreads, PRN_LONG_HALO>, 1>(plan, num_sms, r.B, r.T, r.H)
                     : r.in == 2 ? choose<GruCell, TmaLong<GruCell, 2, PRN_LONG_GRU_L, PRN_LONG_NT, PRN_LONG_HALO>, 2,
                                          PRN_LONG_NT, PRN_LONG_MINB>(plan, num_sms, r.B, r.T, r.H)
                                 : choose<GruCell, TmaLong<GruCell, 4, 8, kThreads, PRN_LONG_HALO>, 4>(plan, num_sms, r.B,
                                                                                                      r.T, r.H);
            else
                rc = !fused ? choose<GruCell, CpLong<GruCell, 0, 16, kThreads>, 0>(plan, num_sms, r.B, r.T, r.H)
                     : r.in == 1 ? choose<GruCell, CpLong<GruCell, 1, 16, kThreads>, 1>(plan, num_sms, r.B, r.T, r.H)
                     : r.in == 2 ? choose<GruCell, CpLong<GruCell, 2, 16, kThreads>, 2>(plan, num_sms, r.B, r.T, r.H)
                                 : choose<GruCell, CpLong<GruCell, 4, 8, kThreads>, 4>(plan, num_sms, r.B, r.T, r.H);
        } else {
            if (tma)
                rc = r.in == 1 ? choose<LstmCell, TmaLong<LstmCell, 1, 8, kThreads>, 1>(plan, num_sms, r.B, r.T, r.H)
                     : r.in == 2 ? choose<LstmCell, TmaLong<LstmCell, 2, 8, kThreads>, 2>(plan, num_sms, r.B, r.T, r.H)
                                 : choose<LstmCell, TmaLong<LstmCell, 4, 8, kThreads>, 4>(plan, num_sms, r.B, r.T, r.H);
            else
                rc = !fused ? choose<LstmCell, CpLong<LstmCell, 0, 8, kThreads>, 0>(plan, num_sms, r.B, r.T, r.H)
                     : r.in == 1 ? choose<LstmCell, CpLong<LstmCell, 1, 8, kThreads>, 1>(plan, num_sms, r.B, r.T, r.H)
                     : r.in == 2 ? choose<LstmCell, CpLong<LstmCell, 2, 8, kThreads>, 2>(plan, num_sms, r.B, r.T, r.H)
                                 : choose<LstmCell, CpLong<LstmCell, 4, 8, kThreads>, 4>(plan, num_sms, r.B, r.T, r.H);
        }
        plan->staged_tma = tma ? 1 : 0;
    } else if (r.H % 32 == 0 && !fused) {
        const int wide = newton_wide_plan(r, num_sms, plan);
        if (wide <= 0) return wide;
        plan->variant = 132;
        rc = S == 1 ? choose<GruCell, Wide<GruCell, 16, kThreads>, 0>(plan, num_sms, r.B, r.T, r.H)
                    : choose<LstmCell, Wide<LstmCell, 8, kThreads>, 0>(plan, num_sms, r.B, r.T, r.H);
    } else {
        return 1;
    }
    if (rc) return -1;
    if (plan->ntiles > 0x7fffffffL) return 1;
    plan->S = S;
    plan->agg_words = (size_t)plan->ntiles * plan->C * (S == 1 ? 2 : 6);
    plan->inc_words = (size_t)plan->ntiles * plan->C * S;
    plan->side_bytes = 2 * (size_t)plan->ntiles * plan->C * plan->halo_w * S * sizeof(float);
    plan->epochs = (unsigned)r.max_iters + 1u;
    plan->staged = 1;
    return 0;
}

// Launch a staged plan: build the tensor maps (TMA layouts) and pass them with the args.
cudaError_t newton_staged_launch(const NewtonDiagArgs &A, const Plan &plan, cudaStream_t st) {
    StagedMaps M;
    memset(&M, 0, sizeof(M));
    if (plan.staged_tma) {
        const int S = plan.S;
        const int PW = A.in;
        const int tch = plan.tch;
        if (!map_rows(&M.x, A.x, (long)A.B * A.T * PW, tch * PW / 32) ||
            !map_rows(&M.h, A.h, (long)A.B * A.T * S, tch * S / 32))
            return cudaErrorInvalidValue;
    }
    void *args[] = {const_cast<NewtonDiagArgs *>(&A), &M};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(plan.threads), args, plan.dyn_smem, st);
}

}  // namespace prn
