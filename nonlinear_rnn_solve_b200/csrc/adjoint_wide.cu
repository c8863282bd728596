// adjoint_wide.cu -- adjoint backward for wide ParaGRU / ParaLSTM layers (H a multiple of
// 32): the reverse scan of adjoint.cu ("Para-Seq" README, Main features: adjoint backward
// by reverse adjoint scans; DEER summary, Surprising findings: one linear solve, no
// backpropagation through the iterations), with the data movement of the wide-layer
// Newton kernel (newton_wide.cu):
//   - a tile is 32 units x 8 sub-chunks of L steps; its projected inputs (a box of
//     xproj [B*T, 3, H]), the states before each of its steps (a box of TCH + 1 rows of
//     h, from the row before the tile) and the upstream gradients (a box of g) arrive by
//     three TMA copies (no multicast) on the stage's mbarrier; two stages form a ring, the
//     last warp done with a stage refills it with the tile two places ahead;
//   - the scan runs from the end of time: the carry entering a tile is the inclusive value
//     of the tile after it in time (a chained scan), read by warp 0 before the compute
//     phase and, when it is not there yet, waited for before the scan's barrier;
//   - the epilogue forms grad_xproj (each warp stores 128 contiguous bytes per gate and
//     step) and accumulates the recurrent-parameter gradients in a shared table per CTA,
//     summed over CTAs in a fixed order after a grid barrier.
// For the backward pass of a whole layer (input projection included) a variant stores
// grad_xproj rounded to bf16, the operand type of the projection's tensor-core products,
// and adds its column sums (the bias gradient, from the fp32 values) with one global
// atomic per lane, gate and tile.
#include <cuda.h>
#include <cuda_bf16.h>
#include <string.h>

#include "cells.cuh"
#include "common.cuh"
#include "internal.h"
#include "staged_tiles.cuh"

namespace prn {

struct AdjWArgs {
    int B, T, H;
    const float *xproj, *a, *peep, *h0, *h, *g;
    float *gx, *gp, *gh0;
    unsigned short *gxb;   // bf16 grad_xproj (the BF variant)
    unsigned short *gxbt;  // its transpose [3 H][B T] (the BF variant, 8 steps per thread; may be null)
    float *gbias;          // bias gradient [3][H] (the BF variant; may be null)
    float *gws;  // per-CTA parameter-gradient partials [grid][NPAR][H]
    Ctl *ctl;
    int *sticky;
    unsigned long long *inc;
    unsigned epoch;
    Dbg dbg;
};

struct AdjWMaps {
    CUtensorMap x, h, g;
};

template <class Cell, int LL> struct AdjWCfg {
    static constexpr int S = Cell::S, C = 32, L = LL, SUB = kThreads / C, TCH = SUB * L, NST = 2;
    static constexpr int ROWP = 3 * C, ROWS = C * S;
    static constexpr int XF = TCH * ROWP;          // projected inputs, TCH rows
    static constexpr int HF = (TCH + 1) * ROWS;    // states t_lo - 1 .. t_lo + TCH - 1
    static constexpr int GF = TCH * ROWS;          // upstream gradients
    static constexpr int STAGE = XF + HF + GF;
    static_assert((XF * 4) % 128 == 0 && ((XF + HF) * 4) % 128 == 0 && (STAGE * 4) % 128 == 0, "TMA destinations");
    static_assert(TCH + 1 <= 256, "TMA box height");
};

template <class Cell, int L, bool BF>
__global__ void __launch_bounds__(kThreads, 2)
    adjoint_wide_kernel(const AdjWArgs A, const __grid_constant__ AdjWMaps M) {
    using G = AdjWCfg<Cell, L>;
    constexpr int S = Cell::S, C = G::C, SUB = G::SUB, TCH = G::TCH, NST = G::NST;
    constexpr int NF = S == 1 ? 2 : 3;  // parameter factors per step
    constexpr int NP = Cell::NPAR;
    extern __shared__ __align__(1024) unsigned char smraw[];
    float *const smem = reinterpret_cast<float *>(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    float *const gp_tab = smem + NST * G::STAGE;  // [NP][H]
    __shared__ ScanSmem<S, C> sm2[2];
    __shared__ int s_fail;
    __shared__ unsigned s_done[NST];
    __shared__ __align__(8) unsigned long long s_bar[NST];
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nct = A.H / C;
    const int nseq = A.B * nct;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long ntiles = (long)nseq * nchunk;
    const long ntile_cta = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int step_ch = (int)(gridDim.x / (unsigned)nseq), step_sq = (int)(gridDim.x % (unsigned)nseq);
    auto step = [&](int &ch, int &sq) {
        ch += step_ch;
        sq += step_sq;
        if (sq >= nseq) {
            sq -= nseq;
            ++ch;
        }
    };
    unsigned phase = 0, pending = 0;
    if (tid == 0) {
        s_fail = 0;
        for (int st = 0; st < NST; ++st) {
            mbar_init(s_bar + st, 1);
            s_done[st] = 0;
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int e = tid; e < NP * A.H; e += kThreads) gp_tab[e] = 0.f;
    __syncthreads();
    // stage st <- tile (chunk in scan order, sequence) (one thread)
    auto issue = [&](int st, int ch, int sq) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        const int b = sq / nct, ct = sq % nct;
        const int row = b * A.T + (nchunk - 1 - ch) * TCH;  // earliest step of the tile
        float *dst = smem + st * G::STAGE;
        mbar_expect_tx(s_bar + st, (unsigned)G::STAGE * 4u);
        tma_load_3d(dst, &M.x, ct * C, 0, row, s_bar + st);
        tma_load_2d(dst + G::XF, &M.h, ct * C * S, row - 1, s_bar + st);  // from the state before the tile
        tma_load_2d(dst + G::XF + G::HF, &M.g, ct * C * S, row, s_bar + st);
    };
    auto wait = [&](int st) -> bool {
        const unsigned par = (phase >> st) & 1u;
        bool ok = mbar_try_sleep(s_bar + st, par, 20000u);
        if (!ok) {
            const unsigned long long t0 = gtimer();
            while (!(ok = mbar_try_sleep(s_bar + st, par, 20000u))) {
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
    };
    auto drain = [&]() {
        for (int st = 0; st < NST; ++st) {
            if (!((pending >> st) & 1u)) continue;
            const unsigned par = (phase >> st) & 1u;
            const unsigned long long t0 = gtimer();
            while (!mbar_try(s_bar + st, par) && gtimer() - t0 < A.dbg.wait_ns) {
            }
        }
    };
    int ch = (int)(blockIdx.x / (unsigned)nseq), sq = (int)(blockIdx.x % (unsigned)nseq);
    int ach = ch, asq = sq;  // NST tiles ahead
    for (int j = 0; j < NST; ++j) {
        if (j < ntile_cta) {
            if (tid == 0) issue(j, ach, asq);
            pending |= 1u << j;
        }
        step(ach, asq);
    }
    for (long j = 0; j < ntile_cta; ++j) {
        const int st = (int)(j % NST), par = (int)(j & 1);
        const long tile = blockIdx.x + j * (long)gridDim.x;
        const int chunk = ch, seq = sq;  // chunk in scan order: from the end of time
        const int b = seq / nct, ct = seq % nct, h = ct * C + c;
        const int t_lo = (nchunk - 1 - chunk) * TCH;
        const int rbase = (SUB - 1 - s) * L;  // local row of the thread's earliest step
        ScanSmem<S, C> &sm = sm2[par];
        const float *sx = smem + st * G::STAGE, *shh = sx + G::XF, *sg = shh + G::HF;
        Cell cell;
        cell.load(A.a, A.peep, A.H, h);
        float h0v[S];  // the state before t = 0
#pragma unroll
        for (int k = 0; k < S; ++k) h0v[k] = 0.f;
        if (t_lo == 0 && rbase == 0 && A.h0) {
#pragma unroll
            for (int k = 0; k < S; ++k) h0v[k] = A.h0[((size_t)b * A.H + h) * S + k];
        }
        unsigned long long pw[S];
#pragma unroll
        for (int k = 0; k < S; ++k) pw[k] = 0ull;
        if (s == 0 && chunk > 0) {
#pragma unroll
            for (int k = 0; k < S; ++k) pw[k] = ld_relaxed_u64(A.inc + ((tile - nseq) * C + c) * S + k);
        }
        if (!wait(st)) s_fail = 1;  // acted on after the scan's barrier
        float Jm[L][S * S], gg[L][S], dp[L][3 * S], fac[L][NF];
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int lr = rbase + (L - 1 - i);  // scan step i is local row lr (descending time)
            const bool v = t_lo + lr < A.T;
            float p[3], hp[S], gv[S];
#pragma unroll
            for (int gq = 0; gq < 3; ++gq) p[gq] = sx[lr * G::ROWP + gq * C + c];
            if (S == 1) {
                hp[0] = shh[lr * G::ROWS + c];  // row lr = the state before step lr
                gv[0] = sg[lr * G::ROWS + c];
            } else {
                const float2 u = *reinterpret_cast<const float2 *>(shh + lr * G::ROWS + c * S);
                const float2 w = *reinterpret_cast<const float2 *>(sg + lr * G::ROWS + c * S);
                hp[0] = u.x;
                hp[S - 1] = u.y;
                gv[0] = w.x;
                gv[S - 1] = w.y;
            }
            if (t_lo + lr == 0) {
#pragma unroll
                for (int k = 0; k < S; ++k) hp[k] = h0v[k];
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
        if (tid < 32) {
            // warp 0: the carry (mu entering the tile from later times) is the inclusive
            // value of the tile before this one in scan order; wait for it here, before the
            // scan's barrier, when the early read did not find it
            bool ok = true;
#pragma unroll
            for (int k = 0; k < S; ++k)
                if (chunk > 0) ok &= (unsigned)pw[k] == A.epoch;
            if (!__all_sync(0xffffffffu, ok)) {
                const unsigned long long *src = A.inc + ((tile - nseq) * C + c) * S;
                unsigned long long t0 = 0;
                for (int polls = 0;; ++polls) {
                    ok = true;
#pragma unroll
                    for (int k = 0; k < S; ++k) {
                        pw[k] = ld_relaxed_u64(src + k);
                        ok &= (unsigned)pw[k] == A.epoch;
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
                        if (tid == 0) s_fail = 1;
                        break;
                    }
                    if (polls > 4) __nanosleep(32);
                }
            }
#pragma unroll
            for (int k = 0; k < S; ++k) sm.carry[c][k] = chunk > 0 ? __uint_as_float((unsigned)(pw[k] >> 32)) : 0.f;
        }
        Aff<S> excl, total;
        cta_scan<S, C>(e, sm, excl, total);  // the one CTA barrier of a tile
        if (s_fail) {
            drain();
            return;  // a bounded wait ran out; the status says so
        }
        if (tid < 32) publish_inc<S, C>(LookBack<S>{nullptr, A.inc}, total, sm.carry[c], tile, A.epoch, A.dbg);
        float mu[S];
        excl.apply(sm.carry[c], mu);
        float gpv[NP];
#pragma unroll
        for (int k = 0; k < NP; ++k) gpv[k] = 0.f;
        const size_t obase = ((size_t)b * A.T + t_lo + rbase + L - 1) * 3 * A.H + h;  // scan step 0
        const size_t ostep = (size_t)3 * A.H;
        float gbv[3] = {0.f, 0.f, 0.f};  // bias-gradient terms (BF)
        // the transposed copy (BF, 8 steps per thread): gate q's 8 values of this thread's
        // steps, in time order, packed two per word for one 16-byte store
        constexpr bool kT8 = BF && L == 8;
        unsigned pk[3][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
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
                gpv[0] = fmaf(gxv[0], fac[i][0], gpv[0]);
                gpv[1] = fmaf(gxv[1], fac[i][0], gpv[1]);
                gpv[2] = fmaf(gxv[2], fac[i][1 % NF], gpv[2]);
            } else {
                gpv[0] = fmaf(gxv[0], fac[i][0], gpv[0]);
                gpv[1] = fmaf(gxv[1], fac[i][0], gpv[1]);
                gpv[2] = fmaf(gxv[2], fac[i][0], gpv[2]);
                gpv[3 % NP] = fmaf(gxv[0], fac[i][1 % NF], gpv[3 % NP]);
                gpv[4 % NP] = fmaf(gxv[2], fac[i][2 % NF], gpv[4 % NP]);
            }
#pragma unroll
            for (int r = 0; r < S; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < S; ++k) acc = fmaf(Jm[i][k * S + r], lam[k], acc);
                mu[r] = acc;
            }
            if (t < A.T) {
                if (BF) {
                    unsigned short *oi = A.gxb + (obase - i * ostep);
#pragma unroll
                    for (int qg = 0; qg < 3; ++qg) {
                        const unsigned short bits = __bfloat16_as_ushort(__float2bfloat16_rn(gxv[qg]));
                        oi[qg * A.H] = bits;
                        if (kT8) pk[qg][(L - 1 - i) >> 1] |= (unsigned)bits << (16 * ((L - 1 - i) & 1));
                        gbv[qg] += gxv[qg];
                    }
                } else {
                    float *oi = A.gx + (obase - i * ostep);
                    oi[0] = gxv[0];
                    oi[A.H] = gxv[1];
                    oi[2 * A.H] = gxv[2];
                }
                if (t == 0 && A.gh0) {
#pragma unroll
                    for (int k = 0; k < S; ++k) A.gh0[((size_t)b * A.H + h) * S + k] = mu[k];
                }
            }
        }
#pragma unroll
        for (int k = 0; k < NP; ++k) atomicAdd(gp_tab + k * A.H + h, gpv[k]);
        if (BF && A.gbias) {
#pragma unroll
            for (int qg = 0; qg < 3; ++qg) atomicAdd(A.gbias + qg * A.H + h, gbv[qg]);
        }
        if (kT8 && A.gxbt && t_lo + rbase + L <= A.T) {
            // row q H + h of the transpose, columns b T + t_lo + rbase .. + 7: 16-byte aligned
            // (T is a multiple of 8, so an 8-step run lies wholly inside the sequence or
            // wholly past its end)
            const size_t M = (size_t)A.B * A.T, col = (size_t)b * A.T + t_lo + rbase;
#pragma unroll
            for (int qg = 0; qg < 3; ++qg)
                *reinterpret_cast<uint4 *>(A.gxbt + (size_t)(qg * A.H + h) * M + col) =
                    make_uint4(pk[qg][0], pk[qg][1], pk[qg][2], pk[qg][3]);
        }
        // this warp is done with the stage; the last warp to finish refills it with the
        // tile NST places ahead (acquire-release add on the counter)
        const bool more = j + NST < ntile_cta;
        if (more) pending |= 1u << st;
        __syncwarp();
        if ((tid & 31) == 0 && more) {
            unsigned cnt;
            asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                         : "=r"(cnt)
                         : "r"(smem_addr(s_done + st))
                         : "memory");
            if (cnt == kThreads / 32 - 1) {
                s_done[st] = 0;
                issue(st, ach, asq);
            }
        }
        step(ach, asq);
        step(ch, sq);
    }
    for (int st = 0; st < NST; ++st)
        if (((pending >> st) & 1u) && !wait(st)) return;
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

constexpr int kTabMax = 12288;  // shared-memory gradient table limit (floats)

template <class Cell, int L, bool BF> int choose(Plan *plan, int num_sms, long B, long T, long H) {
    using G = AdjWCfg<Cell, L>;
    const int np = Cell::NPAR;
    const int smem = (G::NST * G::STAGE + np * (int)H) * (int)sizeof(float) + 1024;
    const void *f = reinterpret_cast<const void *>(&adjoint_wide_kernel<Cell, L, BF>);
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return -1;
    plan->kernel = f;
    plan->dyn_smem = smem;
    plan->C = G::C;
    plan->tch = G::TCH;
    plan->ntiles = B * (H / G::C) * ((T + G::TCH - 1) / G::TCH);
    plan->threads = kThreads;
    plan->grid = occupancy_grid(plan->kernel, kThreads, smem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

}  // namespace

// The bf16 variant's transposed copy: ParaGRU (8 steps per thread), whole 8-step runs
// of every sequence 16-byte aligned in the transpose's rows (T % 8 == 0).
bool adjoint_wide_writes_transpose(const AdjointReq &r) { return r.cell == 0 && r.out_bf16 && r.T % 8 == 0; }

// H % 32 == 0 and a shared-memory gradient table that fits; 1: not covered.
int adjoint_wide_plan(const AdjointReq &r, int num_sms, Plan *plan) {
    const int S = r.cell == 1 ? 2 : 1;
    const int np = S == 1 ? GruCell::NPAR : LstmCell::NPAR;
    if (r.H % 32 || (long)np * r.H > kTabMax || !encode_fn()) return 1;
    if ((long)r.B * r.T >= (1L << 31)) return 1;
    const bool bf = r.out_bf16;
    const int rc = S == 1 ? (bf ? choose<GruCell, 8, true>(plan, num_sms, r.B, r.T, r.H)
                                : choose<GruCell, 8, false>(plan, num_sms, r.B, r.T, r.H))
                          : (bf ? choose<LstmCell, 5, true>(plan, num_sms, r.B, r.T, r.H)
                                : choose<LstmCell, 5, false>(plan, num_sms, r.B, r.T, r.H));
    if (rc) return -1;
    if (plan->ntiles > 0x7fffffffL) return 1;
    plan->variant = 300 + S;
    plan->S = S;
    plan->agg_words = 0;  // a chained scan: only inclusive values are published
    plan->inc_words = (size_t)plan->ntiles * plan->C * S;
    plan->epochs = 2;
    plan->side_bytes = (size_t)plan->grid * np * r.H * sizeof(float);  // per-CTA partials
    plan->tab = 1;
    plan->staged = 2;
    return 0;
}

cudaError_t adjoint_wide_launch(const AdjointReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                                cudaStream_t st) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const int S = plan.S;
    AdjWMaps M;
    memset(&M, 0, sizeof(M));
    {
        cuuint64_t dims[3] = {(cuuint64_t)r.H, 3, (cuuint64_t)r.B * r.T};
        cuuint64_t strides[2] = {(cuuint64_t)r.H * 4, (cuuint64_t)3 * r.H * 4};
        cuuint32_t box[3] = {32, 3, (cuuint32_t)plan.tch};
        cuuint32_t estr[3] = {1, 1, 1};
        if (fn(&M.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(r.xproj), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    for (int q = 0; q < 2; ++q) {  // states (TCH + 1 rows per box) and upstream gradients
        cuuint64_t dims[2] = {(cuuint64_t)r.H * S, (cuuint64_t)r.B * r.T};
        cuuint64_t strides[1] = {(cuuint64_t)r.H * S * 4};
        cuuint32_t box[2] = {(cuuint32_t)(32 * S), (cuuint32_t)(plan.tch + (q == 0 ? 1 : 0))};
        cuuint32_t estr[2] = {1, 1};
        if (fn(q == 0 ? &M.h : &M.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(q == 0 ? r.h : r.g), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    AdjWArgs A;
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
    A.gxb = r.grad_xproj_bf16;
    A.gxbt = r.grad_xproj_bf16_t;
    A.gbias = r.grad_bias;
    A.gp = r.grad_params;
    A.gh0 = r.grad_h0;
    A.gws = w.side;
    A.ctl = w.ctl;
    A.sticky = w.sticky;
    A.inc = w.inc;
    A.epoch = w.epoch0 + 1u;
    A.dbg.wait_ns = dbg.wait_ns;
    A.dbg.skip_tile = dbg.skip_tile;
    A.dbg.delta_log = nullptr;
    A.dbg.delta_log_cap = 0;
    A.dbg.no_halo = 1;
    void *args[] = {&A, &M};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(plan.threads), args, plan.dyn_smem, st);
}

}  // namespace prn
