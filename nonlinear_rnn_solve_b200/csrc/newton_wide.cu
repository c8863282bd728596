// newton_wide.cu -- Newton (DEER) forward for wide ParaGRU / ParaLSTM layers (H a
// multiple of 32, projected inputs given): the LLM-width layer shapes of "ParaRNN:
// Unlocking Parallel Training of Nonlinear RNNs for Large Language Models" (abstract).
//
// Method as in newton_staged.cu ("Parallelizing non-linear sequential models over the
// sequence length", Approach: linearise the cell at the current iterate, solve the linear
// recurrence with a parallel prefix scan, repeat).  One persistent cooperative launch
// runs every iteration.  A tile is 32 channels x SUB sub-chunks of L steps:
//   - the tile's projected inputs (a [TCH x 3 x 32] box of xproj [B*T, 3, H]) and states
//     (a [TCH x 32*S] box of h) arrive in shared memory by two TMA copies (no multicast)
//     completing on the stage's mbarrier; NST stages form a ring, and the last warp to
//     finish with a stage refills it with the tile NST places ahead, so the copies of
//     the next tiles overlap the whole of the current one;
//   - every thread evaluates f, J and r = f - h^(k) for its L steps of one channel in
//     registers (J and r never reach memory), composes them, and the CTA scans the
//     sub-chunks (one barrier);
//   - the carry entering the tile is the predecessor tile's inclusive value (a chained
//     scan across tiles): warp 0 reads it before the compute phase, when the predecessor
//     normally finished a round earlier, and otherwise waits for it before the scan's
//     barrier while the other warps compute -- one CTA barrier per tile either way;
//   - h^(k+1) = h^(k) + delta is written in place (h^(k) re-read from the stage; each warp
//     stores 128 contiguous bytes per step); the tile's last state goes to a side buffer
//     for the successor's next iteration;
//   - on an iteration known to be the last (the cap), the residual
//     max |h_t - f(h_{t-1}, x_t)| at the result is formed in the same pass from the staged
//     inputs, instead of a separate pass over xproj and h.
#include <cuda.h>
#include <string.h>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"
#include "newton_common.cuh"
#include "staged_tiles.cuh"

namespace prn {

// A tile is CC channels x SUB = 256 / CC sub-chunks of L steps; a warp holds 32 / CC
// sub-chunks.  Shared-memory rows are dense (as the TMA writes them), so the sub-chunks
// of a warp must fall on different bank groups: for CC < 32 the row offset between
// them, L rows of 3 CC (inputs) or CC S (states) floats, must not be a multiple of 32
// banks (L = 7 serves CC = 16 and 8).
template <class Cell, int CC, int LL, int NS> struct WideCfg {
    static constexpr int S = Cell::S, C = CC, L = LL, SUB = kThreads / C, TCH = SUB * L, NST = NS;
    static constexpr int ROWP = 3 * C, ROWH = C * S;
    static constexpr int XF = TCH * ROWP, HF = TCH * ROWH;  // floats of the two boxes
    static constexpr int STAGE = XF + HF;                  // floats of one stage
    static constexpr int SMEM_FLOATS = NST * STAGE;
    static_assert(32 % C == 0 && TCH <= 256, "channels per tile divide a warp; TMA box height");
    static_assert((STAGE * 4) % 128 == 0 && (XF * 4) % 128 == 0, "stage alignment");
    static_assert(C == 32 || ((L * ROWP) % 32 != 0 && (L * ROWP * (32 / C / 2)) % 32 != 0),
                  "sub-chunks of a warp on distinct bank groups");
};

// Per-CTA state of the wide kernel: the staging ring and the tile schedule.
template <class Cell, int CC, int L, int NST> struct WideRun {
    using G = WideCfg<Cell, CC, L, NST>;
    static constexpr int S = Cell::S, C = G::C, SUB = G::SUB, TCH = G::TCH;
    const NewtonDiagArgs &A;
    const StagedMaps &M;
    float *smem;
    unsigned long long *bar;  // [NST] stage-full barriers
    unsigned *done;           // [NST] warps finished with the stage (shared counters)
    ScanSmem<S, C> *sm2;      // [2] by tile parity
    int *s_fail;
    int tid, c, s, nct, nseq, nchunk;
    long ntiles, ntile_cta;
    size_t side_stride;
    LookBack<S> lb;
    unsigned phase = 0;    // bit j: parity of stage j's next completion (every thread)
    unsigned pending = 0;  // bit j: stage j has a copy in flight not yet waited for
    // Coordinates (chunk, seq) of this CTA's current tile and of the tile NST places
    // ahead, stepped by gridDim.x tiles without dividing (tile = chunk * nseq + seq).
    struct Pos {
        int chunk, seq;
    };
    Pos cur, ahead;
    int step_ch, step_sq;
    __device__ __forceinline__ void step(Pos &p) const {
        p.chunk += step_ch;
        p.seq += step_sq;
        if (p.seq >= nseq) {
            p.seq -= nseq;
            ++p.chunk;
        }
    }
    // Reset the walkers to this CTA's first tile (start of an iteration).
    __device__ __forceinline__ void restart() {
        cur.chunk = (int)(blockIdx.x / (unsigned)nseq);
        cur.seq = (int)(blockIdx.x % (unsigned)nseq);
        ahead = cur;
        for (int q = 0; q < NST; ++q) step(ahead);
    }
    // Stage st <- tile (ch, sq); one thread calls it.  The proxy fences order this CTA's
    // earlier ordinary stores (h) and shared-memory reads before the TMA's accesses.
    __device__ __forceinline__ void issue(int st, int ch, int sq, bool with_h) const {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        const int b = sq / nct, ct = sq % nct;
        const int row = b * A.T + ch * TCH;
        float *dst = smem + st * G::STAGE;
        mbar_expect_tx(bar + st, (unsigned)(G::XF + (with_h ? G::HF : 0)) * 4u);
        tma_load_3d(dst, &M.x, ct * C, 0, row, bar + st);
        if (with_h) tma_load_2d(dst + G::XF, &M.h, ct * C * S, row, bar + st);
    }
    // L2 prefetch of a tile's boxes (only boxes wholly inside the tensors)
    __device__ __forceinline__ void prefetch(int ch, int sq, bool with_h) const {
        const int b = sq / nct, ct = sq % nct;
        const int row = b * A.T + ch * TCH;
        if ((long)row + TCH > (long)A.B * A.T) return;
        tma_prefetch_3d(&M.x, ct * C, 0, row);
        if (with_h) tma_prefetch_2d(&M.h, ct * C * S, row);
    }
    // Bounded wait for stage st (each thread on the mbarrier).
    __device__ __forceinline__ bool wait(int st) {
        const unsigned par = (phase >> st) & 1u;
        bool ok = mbar_try_sleep(bar + st, par, 20000u);
        if (!ok) {
            const unsigned long long t0 = gtimer();
            while (!(ok = mbar_try_sleep(bar + st, par, 20000u))) {
                if (ld_relaxed_int(&A.ctl->abort)) break;
                if (gtimer() - t0 > A.dbg.wait_ns) {
                    raise_status(A.sticky, A.ctl, kStTimeout, true);
                    break;
                }
            }
        }
        if (ok) {
            phase ^= 1u << st;
            pending &= ~(1u << st);
        }
        return ok;
    }
    // Let copies still in flight land before the CTA exits (bounded).
    __device__ void drain() {
        for (int st = 0; st < NST; ++st) {
            if (!((pending >> st) & 1u)) continue;
            const unsigned par = (phase >> st) & 1u;
            const unsigned long long t0 = gtimer();
            while (!mbar_try(bar + st, par) && gtimer() - t0 < A.dbg.wait_ns) {
            }
        }
    }
    // The first min(NST, tiles of this CTA) tiles of an iteration, into stages 0, 1, ..
    // (thread 0 issues; every thread records them).
    __device__ __forceinline__ void prologue(bool with_h) {
        restart();
        Pos w = cur;
        for (int j = 0; j < NST && j < ntile_cta; ++j, step(w)) {
            if (tid == 0) issue(j, w.chunk, w.seq, with_h);
            pending |= 1u << j;
        }
    }

    __device__ __forceinline__ void load_cur(const float *shh, int tr, int k, float *cur) const {
        if (k > 0) {
            if (S == 1) {
                cur[0] = shh[tr * G::ROWH + c];
            } else {
                const float2 u = *reinterpret_cast<const float2 *>(shh + tr * G::ROWH + c * S);
                cur[0] = u.x;
                cur[S - 1] = u.y;
            }
        } else {
#pragma unroll
            for (int q = 0; q < S; ++q) cur[q] = 0.f;
        }
    }

    // One tile (the j-th of this CTA in iteration k).  FULL: every step lies inside the
    // sequence (no guards); FUSE: the residual at the result is formed in this pass.
    // Returns false when the kernel must stop (a bounded wait ran out).
    template <bool FULL, bool FUSE>
    __device__ __forceinline__ bool tile(int k, long j, unsigned epoch, const float *side_in, float *side_out,
                                         float &my_max, float &my_res, bool &my_bad) {
        const int st = (int)(j % NST), par = (int)(j & 1);
        const float *sx = smem + st * G::STAGE;  // [TCH][3][32]
        const float *shh = sx + G::XF;           // [TCH][32 * S]
        ScanSmem<S, C> &sm = sm2[par];
        const long tile = blockIdx.x + j * (long)gridDim.x;
        const int chunk = cur.chunk, seq = cur.seq;
        const int b = seq / nct, ct = seq % nct;
        const int h = ct * C + c;
        const int t0 = chunk * TCH + s * L;
        // independent of the stage: issued before its wait
        Cell cell;
        cell.load(A.a, A.peep, A.H, h);
        float hp[S];
#pragma unroll
        for (int q = 0; q < S; ++q) hp[q] = 0.f;
        if (t0 == 0) {
            if (A.h0) load_state<S>(A.h0, (size_t)b * A.H + h, hp);
        } else if (k > 0 && s == 0) {
#pragma unroll
            for (int q = 0; q < S; ++q) hp[q] = side_in[((tile - nseq) * C + c) * S + q];
        }
        // first row of sub-chunks (lanes c < C of warp 0): the predecessor's inclusive
        // value, read early (epoch-tagged words)
        unsigned long long pw[S];
#pragma unroll
        for (int q = 0; q < S; ++q) pw[q] = 0ull;
        if (s == 0 && chunk > 0) {
#pragma unroll
            for (int q = 0; q < S; ++q) pw[q] = ld_relaxed_u64(lb.inc + ((tile - nseq) * C + c) * S + q);
        }
        if (!wait(st)) *s_fail = 1;  // acted on after the scan's barrier
        if (tid == 32 && j + NST < ntile_cta) prefetch(ahead.chunk, ahead.seq, k > 0);
        if (k > 0 && s > 0) {
#pragma unroll
            for (int q = 0; q < S; ++q) hp[q] = shh[(s * L - 1) * G::ROWH + c * S + q];
        }
        float hq[S];  // h^(k) before the thread's first step (where the residual starts)
#pragma unroll
        for (int q = 0; q < S; ++q) hq[q] = hp[q];
        float Jr[L][S * S], rr[L][S];
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int tr = s * L + i;
            float p[3], cur[S], f[S], J[S * S];
#pragma unroll
            for (int g = 0; g < 3; ++g) p[g] = sx[tr * G::ROWP + g * C + c];
            load_cur(shh, tr, k, cur);
            cell.eval(p, hp, f, J);
            if (A.jmode) apply_jmode<S>(A.jmode, J);
            const bool v = FULL || t0 + i < A.T;
#pragma unroll
            for (int q = 0; q < S; ++q) {
                rr[i][q] = v ? f[q] - cur[q] : 0.f;
                hp[q] = cur[q];
            }
#pragma unroll
            for (int q = 0; q < S * S; ++q) Jr[i][q] = v ? J[q] : ((q % (S + 1)) == 0 ? 1.f : 0.f);
        }
        Aff<S> e = Aff<S>::ident();
#pragma unroll
        for (int i = 0; i < L; ++i) e = compose(e, make_aff<S>(Jr[i], rr[i]));
        if (tid < 32) {
            // warp 0 (its lanes c >= C belong to later sub-chunks): the carry entering the
            // tile is the predecessor's inclusive value.  Read before the compute phase, it
            // is normally there already; otherwise warp 0 waits for it here, before the
            // scan's barrier, while the other warps still compute.  The predecessor has a
            // lower tile index, so it belongs to a resident CTA (or came earlier in this
            // one) and never waits on this tile.
            bool ok = true;
#pragma unroll
            for (int q = 0; q < S; ++q)
                if (s == 0 && chunk > 0) ok &= (unsigned)pw[q] == epoch;
            if (!__all_sync(0xffffffffu, ok)) {
                const unsigned long long *src = lb.inc + ((tile - nseq) * C + c) * S;
                unsigned long long t0 = 0;
                for (int polls = 0;; ++polls) {
                    ok = true;
                    if (s == 0) {
#pragma unroll
                        for (int q = 0; q < S; ++q) {
                            pw[q] = ld_relaxed_u64(src + q);
                            ok &= (unsigned)pw[q] == epoch;
                        }
                    }
                    if (__all_sync(0xffffffffu, ok)) break;
                    int bad = 0;
                    if (tid == 0) {
                        if (ld_relaxed_int(&A.ctl->abort)) bad = 1;
                        if (polls == 4) t0 = gtimer();
                        if (polls > 4 && gtimer() - t0 > A.dbg.wait_ns) {
                            raise_status(A.sticky, A.ctl, kStTimeout, true);
                            bad = 1;
                        }
                    }
                    if (__shfl_sync(0xffffffffu, bad, 0)) {
                        if (tid == 0) *s_fail = 1;
                        break;
                    }
                    if (polls > 4) __nanosleep(32);
                }
            }
            if (s == 0) {
#pragma unroll
                for (int q = 0; q < S; ++q) sm.carry[c][q] = chunk > 0 ? __uint_as_float((unsigned)(pw[q] >> 32)) : 0.f;
            }
        }
        Aff<S> excl, total;
        cta_scan<S, C>(e, sm, excl, total);  // the one CTA barrier of a tile
        if (*s_fail) {
            drain();
            return false;  // a bounded wait ran out; the status says so
        }
        if (tid < 32) publish_inc<S, C>(lb, total, sm.carry[c], tile, epoch, A.dbg);
        float d[S];
        excl.apply(sm.carry[c], d);
        if (FUSE && t0 > 0) {
#pragma unroll
            for (int q = 0; q < S; ++q) hq[q] += d[q];  // h^(k+1) = h^(k) + delta before the first step
        }
        float *hout = A.h + (((size_t)b * A.T + t0) * A.H + h) * S;
        const size_t hstep = (size_t)A.H * S;
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int tr = s * L + i;
            float nd[S], hn[S], cur[S];
            make_aff<S>(Jr[i], rr[i]).apply(d, nd);
            load_cur(shh, tr, k, cur);
#pragma unroll
            for (int q = 0; q < S; ++q) {
                d[q] = nd[q];
                hn[q] = cur[q] + nd[q];
                my_max = fmaxf(my_max, fabsf(nd[q]));
            }
            if (FULL || t0 + i < A.T) {
                if (S == 1)
                    hout[i * hstep] = hn[0];
                else
                    *reinterpret_cast<float2 *>(hout + i * hstep) = make_float2(hn[0], hn[S - 1]);
                if (FUSE) {
                    float p[3], f[S], J[S * S];
#pragma unroll
                    for (int g = 0; g < 3; ++g) p[g] = sx[tr * G::ROWP + g * C + c];
                    cell.eval(p, hq, f, J);
#pragma unroll
                    for (int q = 0; q < S; ++q) {
                        const float ad = fabsf(hn[q] - f[q]);
                        my_res = (ad > my_res || isnan(ad)) ? ad : my_res;
                        hq[q] = hn[q];
                    }
                }
            }
            if (i == L - 1 && s == SUB - 1 && chunk < nchunk - 1) {
#pragma unroll
                for (int q = 0; q < S; ++q) side_out[(tile * C + c) * S + q] = hn[q];
            }
        }
        // a NaN or Inf anywhere in the segment reaches its last update
#pragma unroll
        for (int q = 0; q < S; ++q) my_bad |= !finitef(d[q]);
        // This warp is done with the stage.  The last warp to finish refills it with the
        // tile NST places ahead: the acquire-release add on the counter orders every
        // warp's reads of the stage (and stores of h) before the copy.
        const bool more = j + NST < ntile_cta;
        if (more) pending |= 1u << st;
        __syncwarp();
        if ((tid & 31) == 0 && more) {
            unsigned cnt;
            asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                         : "=r"(cnt)
                         : "r"(smem_addr(done + st))
                         : "memory");
            if (cnt == kThreads / 32 - 1) {  // every warp of the CTA is done with it
                done[st] = 0;
                issue(st, ahead.chunk, ahead.seq, k > 0);
            }
        }
        step(cur);
        step(ahead);
        return true;
    }
};

// RES: a residual is asked for (the instantiation without it carries no residual code).
template <class Cell, int CC, int L, int NST, int MINB, bool RES>
__global__ void __launch_bounds__(kThreads, MINB)
    newton_wide_kernel(const NewtonDiagArgs A, const __grid_constant__ StagedMaps M) {
    using R = WideRun<Cell, CC, L, NST>;
    using G = typename R::G;
    constexpr int S = Cell::S, C = G::C, TCH = G::TCH;
    extern __shared__ __align__(1024) unsigned char smraw[];
    __shared__ ScanSmem<S, C> sm2[2];
    __shared__ unsigned s_red[kThreads / 32];
    __shared__ int s_fail;
    __shared__ unsigned s_done[NST];
    __shared__ __align__(8) unsigned long long s_bar[NST];
    R r{A, M};
    r.smem = reinterpret_cast<float *>(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    r.bar = s_bar;
    r.done = s_done;
    r.sm2 = sm2;
    r.s_fail = &s_fail;
    r.tid = threadIdx.x;
    r.c = threadIdx.x % C;
    r.s = threadIdx.x / C;
    r.nct = A.H / C;
    r.nseq = A.B * r.nct;
    r.step_ch = (int)(gridDim.x / (unsigned)r.nseq);
    r.step_sq = (int)(gridDim.x % (unsigned)r.nseq);
    r.nchunk = (A.T + TCH - 1) / TCH;
    r.ntiles = (long)r.nseq * r.nchunk;
    r.ntile_cta = blockIdx.x < r.ntiles ? (r.ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    r.side_stride = (size_t)r.ntiles * C * S;
    r.lb = LookBack<S>{A.agg, A.inc};
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_fail = 0;
        for (int st = 0; st < NST; ++st) {
            mbar_init(s_bar + st, 1);
            s_done[st] = 0;
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    r.prologue(false);

    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false, res_done = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epoch = A.epoch0 + (unsigned)k + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        const float *side_in = A.side + (size_t)(k & 1) * r.side_stride;
        float *side_out = A.side + (size_t)((k + 1) & 1) * r.side_stride;
        // the cap makes this iteration the last: the residual rides along
        const bool fuse_res = RES && A.residual_out != nullptr && k == A.max_iters - 1;
        float my_max = 0.f, my_res = 0.f;
        bool my_bad = false;
        for (long j = 0; j < r.ntile_cta; ++j) {
            const bool full = (r.cur.chunk + 1) * TCH <= A.T;
            bool ok;
            if (RES && fuse_res)
                ok = full ? r.template tile<true, RES>(k, j, epoch, side_in, side_out, my_max, my_res, my_bad)
                          : r.template tile<false, RES>(k, j, epoch, side_in, side_out, my_max, my_res, my_bad);
            else
                ok = full ? r.template tile<true, false>(k, j, epoch, side_in, side_out, my_max, my_res, my_bad)
                          : r.template tile<false, false>(k, j, epoch, side_in, side_out, my_max, my_res, my_bad);
            if (!ok) return;
        }
        const unsigned bits = block_max_bits(my_bad ? __int_as_float(0x7fc00000) : my_max, s_red);
        if (tid == 0) atomicMax(&A.ctl->delta_bits[k % 3], bits);
        if (RES && fuse_res) {
            const unsigned rb = block_max_bits(my_res, s_red);
            if (tid == 0) atomicMax(&A.ctl->res_bits, rb);
        }
        // this CTA's first tiles for the next iteration: past the barriers of the block
        // max every store of this CTA to them is done (no other CTA writes them)
        if (k + 1 < A.max_iters) r.prologue(true);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) {
            r.drain();
            return;
        }
        const unsigned dbits = ld_acquire(&A.ctl->delta_bits[k % 3]);
        last_delta = __uint_as_float(dbits);
        iters = k + 1;
        res_done = fuse_res;
        if (blockIdx.x == 0 && tid == 0 && A.dbg.delta_log && k < A.dbg.delta_log_cap) A.dbg.delta_log[k] = last_delta;
        if (dbits >= 0x7f800000u) {
            if (blockIdx.x == 0 && tid == 0) atomicOr(A.sticky, kStNonfinite);
            stop_all = true;
            break;
        }
        if (last_delta < A.tol) break;
    }
    // speculative copies may still be in flight
    for (int st = 0; st < NST; ++st)
        if (((r.pending >> st) & 1u) && !r.wait(st)) return;
    if (RES && A.residual_out && !stop_all) {
        if (res_done) {
            if (blockIdx.x == 0 && tid == 0) {
                const unsigned rb = ld_acquire(&A.ctl->res_bits);
                *A.residual_out = __uint_as_float(rb);
                if (rb >= 0x7f800000u) atomicOr(A.sticky, kStNonfinite);
            }
        } else if (!residual_pass<Cell, C, L, 0>(A, s_red)) {
            return;
        }
    }
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

template <class Cell, int CC, int L, int NST, int MINB>
int choose_wide(Plan *plan, int num_sms, long B, long T, long H, bool res) {
    using G = WideCfg<Cell, CC, L, NST>;
    if (H % CC) return 1;
    auto kern = res ? &newton_wide_kernel<Cell, CC, L, NST, MINB, true>
                    : &newton_wide_kernel<Cell, CC, L, NST, MINB, false>;
    const int smem = G::SMEM_FLOATS * (int)sizeof(float) + 1024;
    const void *f = reinterpret_cast<const void *>(kern);
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return -1;
    plan->kernel = f;
    plan->dyn_smem = smem;
    plan->C = G::C;
    plan->tch = G::TCH;
    plan->ntiles = B * (H / G::C) * ((T + G::TCH - 1) / G::TCH);
    plan->threads = kThreads;
    plan->halo_w = 1;
    plan->grid = occupancy_grid(plan->kernel, kThreads, smem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

}  // namespace

// Wide layers: H % 32 == 0 with projected inputs.  Returns 1 when the shape is not covered.
// Channels per tile: 32 (128-byte rows per gate and step); 16 and 8 are selectable for
// measurements and tests (debug knob 6) and measured slower on the layer shapes.
int newton_wide_plan(const NewtonDiagReq &r, int num_sms, Plan *plan) {
    if (r.H % 32 || r.xproj == nullptr || !encode_fn()) return 1;
    if ((long)r.B * r.T >= (1L << 31)) return 1;  // TMA row coordinates are 32-bit
    const int S = r.cell == 1 ? 2 : 1;
    const bool res = r.residual_out != nullptr;
    const int cc = r.variant ? r.variant : 32;
    int rc;
    if (S == 1) {
        rc = cc == 32   ? choose_wide<GruCell, 32, 12, 2, 2>(plan, num_sms, r.B, r.T, r.H, res)
             : cc == 16 ? choose_wide<GruCell, 16, 7, 2, 2>(plan, num_sms, r.B, r.T, r.H, res)
                        : choose_wide<GruCell, 8, 7, 2, 2>(plan, num_sms, r.B, r.T, r.H, res);
    } else {
        rc = cc == 32   ? choose_wide<LstmCell, 32, 8, 2, 2>(plan, num_sms, r.B, r.T, r.H, res)
             : cc == 16 ? choose_wide<LstmCell, 16, 7, 2, 2>(plan, num_sms, r.B, r.T, r.H, res)
                        : choose_wide<LstmCell, 8, 7, 2, 2>(plan, num_sms, r.B, r.T, r.H, res);
    }
    if (rc) return rc > 0 ? 1 : -1;
    if (plan->ntiles > 0x7fffffffL) return 1;
    plan->variant = 200 + plan->C;
    plan->S = S;
    plan->agg_words = 0;  // a chained scan: only inclusive values are published
    plan->inc_words = (size_t)plan->ntiles * plan->C * S;
    plan->side_bytes = 2 * (size_t)plan->ntiles * plan->C * S * sizeof(float);
    plan->epochs = (unsigned)r.max_iters + 1u;
    plan->staged = 2;
    plan->staged_tma = 1;
    return 0;
}

// Launch: the tensor maps of xproj [B*T, 3, H] (boxes C x 3 x TCH) and of the states
// [B*T, H*S] (boxes C*S x TCH), passed with the arguments.
cudaError_t newton_wide_launch(const NewtonDiagArgs &A, const Plan &plan, cudaStream_t st) {
    StagedMaps M;
    memset(&M, 0, sizeof(M));
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const int S = plan.S;
    {
        cuuint64_t dims[3] = {(cuuint64_t)A.H, 3, (cuuint64_t)A.B * A.T};
        cuuint64_t strides[2] = {(cuuint64_t)A.H * 4, (cuuint64_t)3 * A.H * 4};
        cuuint32_t box[3] = {(cuuint32_t)plan.C, 3, (cuuint32_t)plan.tch};
        cuuint32_t estr[3] = {1, 1, 1};
        if (fn(&M.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(A.xproj), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)A.H * S, (cuuint64_t)A.B * A.T};
        cuuint64_t strides[1] = {(cuuint64_t)A.H * S * 4};
        cuuint32_t box[2] = {(cuuint32_t)(plan.C * S), (cuuint32_t)plan.tch};
        cuuint32_t estr[2] = {1, 1};
        if (fn(&M.h, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, A.h, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    void *args[] = {const_cast<NewtonDiagArgs *>(&A), &M};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(plan.threads), args, plan.dyn_smem, st);
}

}  // namespace prn
