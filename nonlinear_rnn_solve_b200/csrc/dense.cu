// dense.cu -- the vanilla tanh RNN h_t = tanh(A h_{t-1} + U x_t + b), solved with full
// DEER (dense n x n Jacobians) or quasi-DEER (their diagonal), and the standalone dense
// linear scan.
//
// "Para-Seq" README, Main features: ParaRNN is a vanilla tanh RNN with DEER modes;
// dense associative scans.  "Parallelizing non-linear sequential models over the
// sequence length", Surprising findings / Limitations: the explicit Jacobian products
// cost O(n^3) per step, memory O(n^2).  "Towards Scalable and Stable Parallelization
// of Nonlinear RNNs", Abstract: quasi-Newton keeps only the diagonal of the Jacobian.
//
// Full DEER: J_t = diag(1 - f_t^2) A.  A tile [T-chunk x all n units] of one sequence
// forms f, d_t = 1 - f_t^2 and the residual r_t = f_t - h^(k)_t for every step in
// parallel (the matvec A h^(k)_{t-1} reads the previous iterate staged in shared
// memory), then walks its steps once to build the chunk map
//   delta_out = P delta_in + D,   P = J_L ... J_1  (n^3 per step, the DEER cost),
// takes delta_in from the preceding tile's published value (an inclusive chain),
// publishes its own, and re-walks delta_t = J_t delta_{t-1} + r_t to write h^(k+1).
// Quasi-DEER: the Jacobian is diagonal, so the diagonal scan of the ParaGRU path is
// reused with the matvec in the cell evaluation.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace prn {

struct TanhArgs {
    int B, T, n, in;
    int jmode;  // quasi kernel: 0 the diagonal of the Jacobian, 2 zero (Jacobi), 3 identity (Picard)
    const float *xproj, *x, *W, *bias, *A, *h0;
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

// Spin until a 64-bit look-back word carries `epoch`; bounded like every wait.
__device__ __forceinline__ bool wait_word(const unsigned long long *p, unsigned epoch, float *v, Ctl *ctl,
                                          int *sticky, const Dbg &dbg) {
    unsigned long long t0 = 0;
    for (int polls = 0;; ++polls) {
        const unsigned long long w = ld_relaxed_u64(p);
        if ((unsigned)w == epoch) {
            *v = __uint_as_float((unsigned)(w >> 32));
            return true;
        }
        if (ld_relaxed_int(&ctl->abort)) return false;
        if (polls == 4) t0 = gtimer();
        if (polls > 4) {
            if (gtimer() - t0 > dbg.wait_ns) {
                raise_status(sticky, ctl, kStTimeout, true);
                return false;
            }
            __nanosleep(32);
        }
    }
}

// Shared-memory layout of a tanh tile (N = padded state size, TCH steps).
template <int N, int TCH> struct TanhSmem {
    static constexpr int AS = N + 4;  // padded row stride (keeps float4 alignment)
    float AT[N * AS];                 // AT[k][i] = A[i][k]
    float hs[(TCH + 1) * N];          // h^(k) for steps t0-1 .. t0+TCH-1 (row 0 = t0-1)
    float xin[TCH * 8];               // raw inputs of the tile (fused projection)
    float Wt[8 * N];                  // Wt[q][i] = W[i][q]
    float bz[N];
};

// Projected input and cell output of (step row tr, unit i) of the tile:
// u = A h_{t-1} + p_t, with p_t from xproj or from the staged raw inputs.
template <int N, int TCH>
__device__ __forceinline__ float tanh_preact(const TanhArgs &A, const TanhSmem<N, TCH> &sm, int b, int t, int tr,
                                             int i) {
    float u;
    if (A.xproj) {
        u = A.xproj[((size_t)b * A.T + t) * A.n + i];
    } else {
        u = sm.bz[i];
        for (int q = 0; q < A.in; ++q) u = fmaf(sm.Wt[q * N + i], sm.xin[tr * 8 + q], u);
    }
    const float *hp = sm.hs + tr * N;  // h^(k)_{t-1}
#pragma unroll 16
    for (int k = 0; k < N; ++k) u = fmaf(sm.AT[k * TanhSmem<N, TCH>::AS + i], hp[k], u);
    return u;
}

// Stage A^T, W^T, bias once per CTA (zero-padded to N).
template <int N, int TCH> __device__ void tanh_stage_params(const TanhArgs &A, TanhSmem<N, TCH> &sm) {
    constexpr int AS = TanhSmem<N, TCH>::AS;
    for (int e = threadIdx.x; e < N * N; e += kThreads) {
        const int i = e / N, k = e % N;  // A[i][k]
        sm.AT[k * AS + i] = (i < A.n && k < A.n) ? A.A[(size_t)i * A.n + k] : 0.f;
    }
    for (int e = threadIdx.x; e < 8 * N; e += kThreads) {
        const int q = e / N, i = e % N;
        sm.Wt[e] = (!A.xproj && q < A.in && i < A.n) ? A.W[(size_t)i * A.in + q] : 0.f;
    }
    for (int i = threadIdx.x; i < N; i += kThreads) sm.bz[i] = (!A.xproj && A.bias && i < A.n) ? A.bias[i] : 0.f;
}

// Stage the tile's inputs and states: hs rows 0..TCH (states t0-1 .. t0+TCH-1 of
// iterate k; h0 before t = 0; zeros for k = 0) and raw inputs.
template <int N, int TCH>
__device__ void tanh_stage_tile(const TanhArgs &A, TanhSmem<N, TCH> &sm, int b, int t0, int k, const float *prev_side,
                                bool residual_mode) {
    for (int e = threadIdx.x; e < (TCH + 1) * N; e += kThreads) {
        const int r = e / N, i = e % N, t = t0 + r - 1;  // state h_{t+1} in output indexing = index t
        float v = 0.f;
        if (i < A.n) {
            if (t < 0) {
                v = A.h0 ? A.h0[(size_t)b * A.n + i] : 0.f;
            } else if (t < A.T && (k > 0 || residual_mode)) {
                v = (r == 0 && prev_side) ? prev_side[i] : A.h[((size_t)b * A.T + t) * A.n + i];
            }
        }
        sm.hs[e] = v;
    }
    if (!A.xproj) {
        for (int e = threadIdx.x; e < TCH * 8; e += kThreads) {
            const int r = e / 8, q = e % 8, t = t0 + r;
            sm.xin[e] = (q < A.in && t < A.T) ? A.x[((size_t)b * A.T + t) * A.in + q] : 0.f;
        }
    }
}

// ------------------------------------------------------------------ full DEER
template <int N> struct DeerCfg {
    static constexpr int TCH = N >= 64 ? 64 : (N >= 32 ? 128 : 256);
    static constexpr int BR = N >= 16 ? N / 16 : 1;   // register block of the chain product
    static constexpr int TG = N / BR;                  // thread grid side (16, or 8 for N = 8)
};

template <int N> struct DeerExtra {
    static constexpr int TCH = DeerCfg<N>::TCH;
    float d[TCH * N];       // 1 - f^2
    float r[TCH * N];       // f - h^(k)
    float P[2][N * N];      // chain product, double buffered
    float D[2][N];          // chain offset
    float carry[N];
    float dl[2][N];         // re-walk delta, double buffered
};

template <int N>
__global__ void __launch_bounds__(kThreads, 1) tanh_deer_kernel(const TanhArgs A) {
    constexpr int TCH = DeerCfg<N>::TCH, BR = DeerCfg<N>::BR, TG = DeerCfg<N>::TG;
    constexpr int AS = TanhSmem<N, TCH>::AS;
    extern __shared__ __align__(16) unsigned char smraw[];
    TanhSmem<N, TCH> &sm = *reinterpret_cast<TanhSmem<N, TCH> *>(smraw);
    DeerExtra<N> &sx = *reinterpret_cast<DeerExtra<N> *>(smraw + ((sizeof(TanhSmem<N, TCH>) + 15) & ~size_t(15)));
    __shared__ unsigned s_red[kThreads / 32];
    __shared__ int s_fail;
    const int tid = threadIdx.x;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long nseq = A.B;
    const long ntiles = nseq * nchunk;
    if (tid == 0) s_fail = 0;
    tanh_stage_params<N, TCH>(A, sm);
    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epoch = A.epoch0 + (unsigned)k + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        const float *side_in = A.side + (size_t)(k & 1) * ntiles * N;
        float *side_out = A.side + (size_t)((k + 1) & 1) * ntiles * N;
        float my_max = 0.f;
        TileWalk tw(nseq);
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
            const int chunk = tw.chunk;
            const int b = tw.seq;
            const int t0 = chunk * TCH;
            const int steps = min(TCH, A.T - t0);
            __syncthreads();
            tanh_stage_tile<N, TCH>(A, sm, b, t0, k, (k > 0 && chunk > 0) ? side_in + (tile - nseq) * N : nullptr,
                                    false);
            __syncthreads();
            // d_t, r_t for every (step, unit)
            for (int e = tid; e < TCH * N; e += kThreads) {
                const int tr = e / N, i = e % N, t = t0 + tr;
                float dv = 0.f, rv = 0.f;
                if (tr < steps && i < A.n) {
                    const float f = tanh_(tanh_preact<N, TCH>(A, sm, b, t, tr, i));
                    dv = 1.f - f * f;
                    rv = f - sm.hs[(tr + 1) * N + i];
                }
                sx.d[e] = dv;
                sx.r[e] = rv;
            }
            // chain: P = I, D = 0, then P <- diag(d_t) A P, D <- diag(d_t) A D + r_t
            for (int e = tid; e < N * N; e += kThreads) sx.P[0][e] = (e / N == e % N) ? 1.f : 0.f;
            if (tid < N) sx.D[0][tid] = 0.f;
            __syncthreads();
            int cur = 0;
            for (int tr = 0; tr < steps; ++tr) {
                const float *Pi = sx.P[cur];
                float *Po = sx.P[cur ^ 1];
                const float *dv = sx.d + tr * N;
                if (tid < TG * TG) {
                    const int i0 = (tid / TG) * BR, j0 = (tid % TG) * BR;
                    float acc[BR][BR];
#pragma unroll
                    for (int a = 0; a < BR; ++a)
#pragma unroll
                        for (int c = 0; c < BR; ++c) acc[a][c] = 0.f;
#pragma unroll 8
                    for (int kk = 0; kk < N; ++kk) {
                        float av[BR], pv[BR];
#pragma unroll
                        for (int a = 0; a < BR; ++a) av[a] = sm.AT[kk * AS + i0 + a];
#pragma unroll
                        for (int c = 0; c < BR; ++c) pv[c] = Pi[kk * N + j0 + c];
#pragma unroll
                        for (int a = 0; a < BR; ++a)
#pragma unroll
                            for (int c = 0; c < BR; ++c) acc[a][c] = fmaf(av[a], pv[c], acc[a][c]);
                    }
#pragma unroll
                    for (int a = 0; a < BR; ++a)
#pragma unroll
                        for (int c = 0; c < BR; ++c) Po[(i0 + a) * N + j0 + c] = dv[i0 + a] * acc[a][c];
                }
                if (tid >= kThreads - N) {
                    const int i = tid - (kThreads - N);
                    float acc = 0.f;
                    for (int kk = 0; kk < N; ++kk) acc = fmaf(sm.AT[kk * AS + i], sx.D[cur][kk], acc);
                    sx.D[cur ^ 1][i] = fmaf(dv[i], acc, sx.r[tr * N + i]);
                }
                __syncthreads();
                cur ^= 1;
            }
            // inclusive chain across tiles: delta_in from the preceding tile
            if (tid < N) {
                float cv = 0.f;
                if (chunk > 0 && !wait_word(A.inc + (tile - nseq) * N + tid, epoch, &cv, A.ctl, A.sticky, A.dbg))
                    s_fail = 1;
                sx.carry[tid] = cv;
            }
            __syncthreads();
            if (s_fail) return;
            if (tid < N) {
                float acc = sx.D[cur][tid];
                for (int j = 0; j < N; ++j) acc = fmaf(sx.P[cur][tid * N + j], sx.carry[j], acc);
                if (A.dbg.skip_tile != tile) st_relaxed_u64(A.inc + tile * N + tid, pack_tag(acc, epoch));
                sx.dl[0][tid] = sx.carry[tid];
            }
            __syncthreads();
            // re-walk: delta_t = diag(d_t) A delta_{t-1} + r_t, h^(k+1) = h^(k) + delta
            int dc = 0;
            for (int tr = 0; tr < steps; ++tr) {
                if (tid < 4 * N) {
                    const int i = tid >> 2, q = tid & 3;
                    float acc = 0.f;
                    for (int kk = q; kk < N; kk += 4) acc = fmaf(sm.AT[kk * AS + i], sx.dl[dc][kk], acc);
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                    if (q == 0) {
                        const float nd = fmaf(sx.d[tr * N + i], acc, sx.r[tr * N + i]);
                        sx.dl[dc ^ 1][i] = nd;
                        if (i < A.n) {
                            const float hn = sm.hs[(tr + 1) * N + i] + nd;
                            const float ad = fabsf(nd);
                            my_max = (ad > my_max || isnan(nd)) ? ad : my_max;
                            A.h[((size_t)b * A.T + t0 + tr) * A.n + i] = hn;
                            if (tr == TCH - 1 && chunk < nchunk - 1) side_out[tile * N + i] = hn;
                        }
                    }
                }
                __syncthreads();
                dc ^= 1;
            }
        }
        const unsigned bits = block_max_bits(my_max, s_red);
        if (tid == 0) atomicMax(&A.ctl->delta_bits[k % 3], bits);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        const unsigned dbits = ld_acquire(&A.ctl->delta_bits[k % 3]);
        last_delta = __uint_as_float(dbits);
        iters = k + 1;
        if (blockIdx.x == 0 && tid == 0 && A.dbg.delta_log && k < A.dbg.delta_log_cap) A.dbg.delta_log[k] = last_delta;
        if (dbits >= 0x7f800000u) {
            if (blockIdx.x == 0 && tid == 0) atomicOr(A.sticky, kStNonfinite);
            stop_all = true;
            break;
        }
        if (last_delta < A.tol) break;
    }
    if (A.residual_out && !stop_all) {
        float my_res = 0.f;
        TileWalk tw(nseq);
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
            const int chunk = tw.chunk;
            const int b = tw.seq;
            const int t0 = chunk * TCH;
            const int steps = min(TCH, A.T - t0);
            __syncthreads();
            tanh_stage_tile<N, TCH>(A, sm, b, t0, 1, nullptr, true);
            __syncthreads();
            for (int e = tid; e < TCH * N; e += kThreads) {
                const int tr = e / N, i = e % N;
                if (tr < steps && i < A.n) {
                    const float f = tanh_(tanh_preact<N, TCH>(A, sm, b, t0 + tr, tr, i));
                    const float ad = fabsf(sm.hs[(tr + 1) * N + i] - f);
                    my_res = (ad > my_res || isnan(ad)) ? ad : my_res;
                }
            }
        }
        const unsigned bits = block_max_bits(my_res, s_red);
        if (tid == 0) atomicMax(&A.ctl->res_bits, bits);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        if (blockIdx.x == 0 && tid == 0) {
            const unsigned rb = ld_acquire(&A.ctl->res_bits);
            *A.residual_out = __uint_as_float(rb);
            if (rb >= 0x7f800000u) atomicOr(A.sticky, kStNonfinite);
        }
    }
    if (blockIdx.x == 0 && tid == 0) {
        *A.iters_out = iters;
        if (A.delta_out) *A.delta_out = last_delta;
        if (!stop_all && A.tol > 0.f && iters == A.max_iters && !(last_delta < A.tol))
            atomicOr(A.sticky, kStNotConverged);
    }
}

// ------------------------------------------------------------------ quasi-DEER
// CTA scan for C = 64 channels (two warps per sub-chunk row): tid = s * 64 + c.
struct Scan64Smem {
    Aff<1> w[kThreads / 64][64];
    ScanSmem<1, 32> half[2];
};

template <int N> struct QuasiCfg {
    static constexpr int C = N;                 // channels per tile = padded state size
    static constexpr int SUB = kThreads / C;
    static constexpr int L = 16;
    static constexpr int TCH = SUB * L;
};

// Shared memory of a quasi-DEER tile.  Phase A evaluates the cell for the whole tile as
// a small matrix product, U[tr][i] = sum_k A[i][k] h^(k)[tr-1][k] + p[tr][i], with each
// thread holding a 4-step x 4-unit block in registers (two 128-bit loads feed sixteen
// FMAs), and leaves J, r and h^(k) per (step, unit).  Phase B is the diagonal scan.
template <int N> struct QuasiSmem {
    static constexpr int TCH = QuasiCfg<N>::TCH;
    static constexpr int AS = N + 4;    // row stride of AT and Wt (float4-aligned)
    static constexpr int HS = TCH + 4;  // row stride of hT and xT (float4-aligned, >= TCH + 1)
    float AT[N * AS];                   // AT[k][i] = A[i][k]
    float Wt[8 * AS];                   // Wt[q][i] = W[i][q]
    float bz[N];
    float diag[N];                      // A_ii
    float hT[N * HS];                   // hT[k][r] = h^(k) of unit k at step t0 - 1 + r
    float hr[(TCH + 1) * N];            // the same states by row: hr[r][k] (conflict-free row reads)
    float xT[8 * HS];                   // xT[q][tr] = x of input q at step t0 + tr
    float Js[TCH * N], rs[TCH * N];     // per (step row, unit)
};

template <int N> __device__ void quasi_stage_params(const TanhArgs &A, QuasiSmem<N> &sm) {
    constexpr int AS = QuasiSmem<N>::AS;
    for (int e = threadIdx.x; e < N * N; e += kThreads) {
        const int i = e / N, k = e % N;  // A[i][k]
        sm.AT[k * AS + i] = (i < A.n && k < A.n) ? A.A[(size_t)i * A.n + k] : 0.f;
    }
    for (int e = threadIdx.x; e < 8 * N; e += kThreads) {
        const int q = e / N, i = e % N;
        sm.Wt[q * AS + i] = (!A.xproj && q < A.in && i < A.n) ? A.W[(size_t)i * A.in + q] : 0.f;
    }
    for (int i = threadIdx.x; i < N; i += kThreads) sm.bz[i] = (!A.xproj && A.bias && i < A.n) ? A.bias[i] : 0.f;
    for (int i = threadIdx.x; i < N; i += kThreads) sm.diag[i] = i < A.n ? A.A[(size_t)i * A.n + i] : 0.f;
}

// h^(k) of unit i at tile row r (the state before step t0 + r): h0 before the sequence,
// the side value for the preceding tile's last step, zeros on the first iteration.
__device__ __forceinline__ float quasi_state(const TanhArgs &A, int b, int t0, int r, int i, bool have_h,
                                             const float *prev_side) {
    const int t = t0 + r - 1;
    if (i >= A.n) return 0.f;
    if (t < 0) return A.h0 ? A.h0[(size_t)b * A.n + i] : 0.f;
    if (t < A.T && have_h) return (r == 0 && prev_side) ? prev_side[i] : A.h[((size_t)b * A.T + t) * A.n + i];
    return 0.f;
}

// A tile's states (rows 0 .. TCH: the states before steps t0 .. t0 + TCH) and raw inputs,
// loaded into registers -- the next tile's while the current one computes -- and then
// written to shared memory, transposed (hT: four consecutive steps of one unit are one
// 128-bit word) and by rows (hr).  A thread holds 4-row groups of one unit, so each
// transposed write is one 128-bit store: a quarter-warp writes eight units' groups at
// unit strides of HS floats (HS % 32 == 4), eight distinct 16-byte bank groups.
template <int N> struct QuasiPrefetch {
    static constexpr int TCH = QuasiSmem<N>::TCH, HS = QuasiSmem<N>::HS;
    static constexpr int G4 = TCH * N / 4 / kThreads;  // 4-row groups per thread
    static constexpr int XPT = TCH * 8 / kThreads;
    static_assert(G4 * 4 * kThreads == TCH * N, "whole 4-row groups per thread");
    static_assert(HS % 4 == 0 && HS % 32 == 4, "float4 rows, conflict-free transposed stores");
    float hv[G4][4], hx, xv[XPT];
    __device__ __forceinline__ void load(const TanhArgs &A, int b, int t0, bool have_h, const float *prev_side) {
#pragma unroll
        for (int j = 0; j < G4; ++j) {
            const int e4 = threadIdx.x + j * kThreads, g = e4 / N, i = e4 % N;
#pragma unroll
            for (int q = 0; q < 4; ++q) hv[j][q] = quasi_state(A, b, t0, 4 * g + q, i, have_h, prev_side);
        }
        hx = threadIdx.x < N ? quasi_state(A, b, t0, TCH, threadIdx.x, have_h, prev_side) : 0.f;
        if (!A.xproj) {
#pragma unroll
            for (int j = 0; j < XPT; ++j) {
                const int e = threadIdx.x + j * kThreads, r = e / 8, q = e % 8, t = t0 + r;
                xv[j] = (q < A.in && t < A.T) ? A.x[((size_t)b * A.T + t) * A.in + q] : 0.f;
            }
        }
    }
    __device__ __forceinline__ void store(const TanhArgs &A, QuasiSmem<N> &sm) const {
#pragma unroll
        for (int j = 0; j < G4; ++j) {
            const int e4 = threadIdx.x + j * kThreads, g = e4 / N, i = e4 % N;
            *reinterpret_cast<float4 *>(sm.hT + i * HS + 4 * g) = make_float4(hv[j][0], hv[j][1], hv[j][2], hv[j][3]);
#pragma unroll
            for (int q = 0; q < 4; ++q) sm.hr[(4 * g + q) * N + i] = hv[j][q];
        }
        if (threadIdx.x < N) {
            sm.hT[threadIdx.x * HS + TCH] = hx;
            sm.hr[TCH * N + threadIdx.x] = hx;
        }
        if (!A.xproj) {
#pragma unroll
            for (int j = 0; j < XPT; ++j) {
                const int e = threadIdx.x + j * kThreads;
                sm.xT[(e % 8) * HS + e / 8] = xv[j];
            }
        }
    }
};

// Stage a tile directly (the first tile of an iteration, the residual pass).
template <int N>
__device__ __forceinline__ void quasi_stage_tile(const TanhArgs &A, QuasiSmem<N> &sm, int b, int t0, bool have_h,
                                                 const float *prev_side) {
    QuasiPrefetch<N> p;
    p.load(A, b, t0, have_h, prev_side);
    p.store(A, sm);
}

// Phase A: f = tanh(A h_{t-1} + p_t) for the thread's 4 x 4 block; J = (1 - f^2) A_ii
// (identity outside the sequence), r = f - h^(k)_t; returns max |r| over valid entries.
template <int N>
__device__ float quasi_phase_a(const TanhArgs &A, QuasiSmem<N> &sm, int b, int t0) {
    constexpr int TCH = QuasiSmem<N>::TCH, AS = QuasiSmem<N>::AS, HS = QuasiSmem<N>::HS;
    constexpr int NUB = N / 4;
    const int ub = threadIdx.x % NUB, sb = threadIdx.x / NUB;
    const int i0 = 4 * ub, r0 = 4 * sb;
    float acc[4][4];
    if (A.xproj) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = t0 + r0 + j;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                acc[j][u] = (t < A.T && i0 + u < A.n) ? A.xproj[((size_t)b * A.T + t) * A.n + i0 + u] : 0.f;
        }
    } else {
        const float4 bz = *reinterpret_cast<const float4 *>(sm.bz + i0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[j][0] = bz.x;
            acc[j][1] = bz.y;
            acc[j][2] = bz.z;
            acc[j][3] = bz.w;
        }
        for (int q = 0; q < A.in; ++q) {
            const float4 w = *reinterpret_cast<const float4 *>(sm.Wt + q * AS + i0);
            const float4 x = *reinterpret_cast<const float4 *>(sm.xT + q * HS + r0);
            const float xv[4] = {x.x, x.y, x.z, x.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[j][u] = fmaf(wv[u], xv[j], acc[j][u]);
        }
    }
#pragma unroll 8
    for (int k = 0; k < N; ++k) {
        const float4 a = *reinterpret_cast<const float4 *>(sm.AT + k * AS + i0);
        const float4 h = *reinterpret_cast<const float4 *>(sm.hT + k * HS + r0);  // h_{t-1} of steps r0..r0+3
        const float av[4] = {a.x, a.y, a.z, a.w}, hv[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[j][u] = fmaf(av[u], hv[j], acc[j][u]);
    }
    float res = 0.f;
    const float4 dg4 = *reinterpret_cast<const float4 *>(sm.diag + i0);
    const float dg[4] = {dg4.x, dg4.y, dg4.z, dg4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int tr = r0 + j;
        const bool tv = t0 + tr < A.T;
        const float4 c4 = *reinterpret_cast<const float4 *>(sm.hr + (tr + 1) * N + i0);  // h^(k)_t
        const float cur[4] = {c4.x, c4.y, c4.z, c4.w};
        float Jv[4], rv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool v = tv && i0 + u < A.n;
            const float f = tanh_(acc[j][u]);
            Jv[u] = !v ? 1.f : A.jmode == 2 ? 0.f : A.jmode == 3 ? 1.f : (1.f - f * f) * dg[u];
            rv[u] = v ? f - cur[u] : 0.f;
            const float ad = fabsf(rv[u]);
            res = (ad > res || isnan(ad)) ? ad : res;
        }
        *reinterpret_cast<float4 *>(sm.Js + tr * N + i0) = make_float4(Jv[0], Jv[1], Jv[2], Jv[3]);
        *reinterpret_cast<float4 *>(sm.rs + tr * N + i0) = make_float4(rv[0], rv[1], rv[2], rv[3]);
    }
    return res;
}

template <int N>
__global__ void __launch_bounds__(kThreads, 2) tanh_quasi_kernel(const TanhArgs A) {
    constexpr int C = QuasiCfg<N>::C, SUB = QuasiCfg<N>::SUB, L = QuasiCfg<N>::L, TCH = QuasiCfg<N>::TCH;
    static_assert(N % 4 == 0 && (N / 4) * (TCH / 4) == kThreads, "one 4 x 4 block per thread");
    extern __shared__ __align__(16) unsigned char smraw[];
    QuasiSmem<N> &sm = *reinterpret_cast<QuasiSmem<N> *>(smraw);
    __shared__ ScanSmem<1, (C <= 32 ? C : 32)> ss;
    __shared__ Scan64Smem s64;
    __shared__ unsigned s_red[kThreads / 32];
    __shared__ int s_fail;
    const int tid = threadIdx.x, c = tid % C, s = tid / C;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long nseq = A.B;
    const long ntiles = nseq * nchunk;
    LookBack<1> lb{A.agg, A.inc};
    if (tid == 0) s_fail = 0;
    quasi_stage_params<N>(A, sm);
    QuasiPrefetch<N> pf;
    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epoch = A.epoch0 + (unsigned)k + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        const float *side_in = A.side + (size_t)(k & 1) * ntiles * C;
        float *side_out = A.side + (size_t)((k + 1) & 1) * ntiles * C;
        float my_max = 0.f;
        TileWalk tw(nseq);
        bool staged = false;  // pf holds this tile's data
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
            const int chunk = tw.chunk;
            const int b = tw.seq;
            const int t0 = chunk * TCH;
            __syncthreads();
            if (staged)
                pf.store(A, sm);
            else
                quasi_stage_tile<N>(A, sm, b, t0, k > 0, (k > 0 && chunk > 0) ? side_in + (tile - nseq) * C : nullptr);
            __syncthreads();
            // the next tile of this iteration (its states are the previous iteration's:
            // nothing this iteration writes) is loaded while this one computes
            staged = tile + gridDim.x < ntiles;
            if (staged) {
                int nch = chunk + tw.step_ch, nsq = b + tw.step_sq;
                if (nsq >= nseq) {
                    nsq -= (int)nseq;
                    ++nch;
                }
                const long nt = tile + gridDim.x;
                pf.load(A, nsq, nch * TCH, k > 0, (k > 0 && nch > 0) ? side_in + (nt - nseq) * C : nullptr);
            }
            quasi_phase_a<N>(A, sm, b, t0);
            __syncthreads();
            const bool cv = c < A.n;
            Aff<1> e = Aff<1>::ident();
#pragma unroll
            for (int i = 0; i < L; ++i) {
                const int tr = s * L + i;
                e = compose(e, Aff<1>{sm.Js[tr * N + c], sm.rs[tr * N + c]});
            }
            Aff<1> excl, total;
            const float zero[1] = {0.f};
            float carry_c;
            if (C <= 32) {
                cta_scan<1, (C <= 32 ? C : 32)>(e, ss, excl, total);
                if (tid < 32) {
                    if (!look_back<1, (C <= 32 ? C : 32)>(lb, ss, total, tile, chunk, nseq, epoch, zero, A.ctl,
                                                          A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();
                if (s_fail) return;
                carry_c = ss.carry[c % (C <= 32 ? C : 32)][0];
            } else {
                s64.w[s][c] = e;
                __syncthreads();
                Aff<1> pre = Aff<1>::ident();
                for (int w = 0; w < s; ++w) pre = compose(pre, s64.w[w][c]);
                excl = pre;
                if (tid < 64) {
                    Aff<1> t = Aff<1>::ident();
#pragma unroll
                    for (int w = 0; w < SUB; ++w) t = compose(t, s64.w[w][tid]);
                    const int half = tid >> 5;
                    if (!look_back<1, 32>(lb, s64.half[half], t, 2 * tile + half, chunk, 2 * nseq, epoch, zero, A.ctl,
                                          A.sticky, A.dbg))
                        if ((tid & 31) == 0) s_fail = 1;
                }
                __syncthreads();
                if (s_fail) return;
                carry_c = s64.half[c >> 5].carry[c & 31][0];
            }
            float d = fmaf(excl.a, carry_c, excl.d);
#pragma unroll
            for (int i = 0; i < L; ++i) {
                const int tr = s * L + i, t = t0 + tr;
                d = fmaf(sm.Js[tr * N + c], d, sm.rs[tr * N + c]);
                const float hn = sm.hr[(tr + 1) * N + c] + d;
                if (cv && t < A.T) {
                    const float ad = fabsf(d);
                    my_max = (ad > my_max || isnan(d)) ? ad : my_max;
                    A.h[((size_t)b * A.T + t) * A.n + c] = hn;
                    if (tr == TCH - 1 && chunk < nchunk - 1) side_out[tile * C + c] = hn;
                }
            }
        }
        const unsigned bits = block_max_bits(my_max, s_red);
        if (tid == 0) atomicMax(&A.ctl->delta_bits[k % 3], bits);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        const unsigned dbits = ld_acquire(&A.ctl->delta_bits[k % 3]);
        last_delta = __uint_as_float(dbits);
        iters = k + 1;
        if (blockIdx.x == 0 && tid == 0 && A.dbg.delta_log && k < A.dbg.delta_log_cap) A.dbg.delta_log[k] = last_delta;
        if (dbits >= 0x7f800000u) {
            if (blockIdx.x == 0 && tid == 0) atomicOr(A.sticky, kStNonfinite);
            stop_all = true;
            break;
        }
        if (last_delta < A.tol) break;
    }
    if (A.residual_out && !stop_all) {
        // max |h_t - f(h_{t-1}, x_t)| at the result: phase A's max |r| with the result
        // staged as the iterate
        float my_res = 0.f;
        TileWalk tw(nseq);
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
            const int b = tw.seq;
            const int t0 = tw.chunk * TCH;
            __syncthreads();
            quasi_stage_tile<N>(A, sm, b, t0, true, nullptr);
            __syncthreads();
            const float r = quasi_phase_a<N>(A, sm, b, t0);
            my_res = (r > my_res || isnan(r)) ? r : my_res;
        }
        const unsigned bits = block_max_bits(my_res, s_red);
        if (tid == 0) atomicMax(&A.ctl->res_bits, bits);
        if (!grid_sync(A.ctl, A.sticky, A.dbg)) return;
        if (blockIdx.x == 0 && tid == 0) {
            const unsigned rb = ld_acquire(&A.ctl->res_bits);
            *A.residual_out = __uint_as_float(rb);
            if (rb >= 0x7f800000u) atomicOr(A.sticky, kStNonfinite);
        }
    }
    if (blockIdx.x == 0 && tid == 0) {
        *A.iters_out = iters;
        if (A.delta_out) *A.delta_out = last_delta;
        if (!stop_all && A.tol > 0.f && iters == A.max_iters && !(last_delta < A.tol))
            atomicOr(A.sticky, kStNotConverged);
    }
}

// ------------------------------------------------------------------ dense linear scan
// out_t = M_t out_{t-1} + b_t along the scan order, M_t = J_t (forward) or J_{t+1}^T
// (reverse, identity at the last step).  Per tile: the chunk map (P, D) by one walk,
// the inclusive chain across tiles, then a re-walk writing out_t.
struct DScanArgs {
    int B, T, n, reverse;
    const float *J, *b, *h0;
    float *out;
    Ctl *ctl;
    int *sticky;
    unsigned long long *inc;
    unsigned epoch0;
    Dbg dbg;
};

template <int N> struct DScanSmem {
    static constexpr int MS = N + 4;
    // the matrix that defines scan step t, row-major with padded rows: J_t (forward:
    // M_t = J_t) or J_{t+1} (reverse: M_t = J_{t+1}^T); double buffered per step
    float Js[2][N * MS];
    float P[2][N * N];
    float D[2][N];
    float carry[N];
    float v[2][N];
};

// Stage the matrix of scan step t (time index) of sequence b into buffer js: with
// 16-byte cp.async copies when n % 4 == 0 (the padding rows and columns, zeroed once,
// are never written), else with plain loads that also write the padding; the identity
// after the last step of a reverse scan.  Copies are committed by the caller.
template <int N>
__device__ __forceinline__ void dscan_stage_M(const DScanArgs &A, float *js, int b, int t, bool vec) {
    constexpr int MS = DScanSmem<N>::MS;
    const int tt = A.reverse ? t + 1 : t;
    if (tt >= A.T) {  // reverse, last step: M = I
        for (int e = threadIdx.x; e < N * N; e += kThreads) {
            const int i = e / N, k = e % N;
            js[i * MS + k] = (i == k && i < A.n) ? 1.f : 0.f;
        }
        return;
    }
    const float *src = A.J + ((size_t)b * A.T + tt) * A.n * A.n;
    if (vec) {
        const int cpr = A.n >> 2;  // 16-byte chunks per row
        for (int e = threadIdx.x; e < A.n * cpr; e += kThreads) {
            const int i = e / cpr, c = e - i * cpr;
            cp_async16(js + i * MS + 4 * c, src + i * A.n + 4 * c, 16);
        }
    } else {
        for (int e = threadIdx.x; e < N * N; e += kThreads) {
            const int i = e / N, k = e % N;
            js[i * MS + k] = (i < A.n && k < A.n) ? src[i * A.n + k] : 0.f;
        }
    }
}

// One step of the chain map, P <- M_t P, for the thread's BR x BR block (rows i0.., columns
// j0..): forward M_t[i][k] = js[i][k], reverse M_t[i][k] = js[k][i].
template <int N, bool REV>
__device__ __forceinline__ void dscan_chain_step(const float *js, const float *P, float *Pn, int i0, int j0) {
    constexpr int MS = DScanSmem<N>::MS, BR = DeerCfg<N>::BR;
    float acc[BR][BR];
#pragma unroll
    for (int a = 0; a < BR; ++a)
#pragma unroll
        for (int c = 0; c < BR; ++c) acc[a][c] = 0.f;
    if constexpr (BR == 4) {
        if constexpr (REV) {
#pragma unroll 8
            for (int kk = 0; kk < N; ++kk) {
                const float4 m = *reinterpret_cast<const float4 *>(js + kk * MS + i0);  // M_t[i0 + a][kk]
                const float4 p = *reinterpret_cast<const float4 *>(P + kk * N + j0);
                const float mv[4] = {m.x, m.y, m.z, m.w}, pv[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(mv[a], pv[c], acc[a][c]);
            }
        } else {
#pragma unroll 2
            for (int k4 = 0; k4 < N; k4 += 4) {
                float mv[4][4], pv[4][4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {  // M_t[i0 + a][k4 .. k4 + 3]
                    const float4 m = *reinterpret_cast<const float4 *>(js + (i0 + a) * MS + k4);
                    mv[a][0] = m.x;
                    mv[a][1] = m.y;
                    mv[a][2] = m.z;
                    mv[a][3] = m.w;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // P[k4 + q][j0 .. j0 + 3]
                    const float4 v = *reinterpret_cast<const float4 *>(P + (k4 + q) * N + j0);
                    pv[q][0] = v.x;
                    pv[q][1] = v.y;
                    pv[q][2] = v.z;
                    pv[q][3] = v.w;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(mv[a][q], pv[q][c], acc[a][c]);
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
            *reinterpret_cast<float4 *>(Pn + (i0 + a) * N + j0) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    } else {
#pragma unroll 8
        for (int kk = 0; kk < N; ++kk) {
            float av[BR], pv[BR];
#pragma unroll
            for (int a = 0; a < BR; ++a) av[a] = REV ? js[kk * MS + i0 + a] : js[(i0 + a) * MS + kk];
#pragma unroll
            for (int c = 0; c < BR; ++c) pv[c] = P[kk * N + j0 + c];
#pragma unroll
            for (int a = 0; a < BR; ++a)
#pragma unroll
                for (int c = 0; c < BR; ++c) acc[a][c] = fmaf(av[a], pv[c], acc[a][c]);
        }
#pragma unroll
        for (int a = 0; a < BR; ++a)
#pragma unroll
            for (int c = 0; c < BR; ++c) Pn[(i0 + a) * N + j0 + c] = acc[a][c];
    }
}

// Row r of M_t times the vector x (N entries): forward reads row r of js (16-byte
// loads), reverse column r.
template <int N, bool REV> __device__ __forceinline__ float dscan_row_dot(const float *js, int r, const float *x) {
    constexpr int MS = DScanSmem<N>::MS;
    float acc = 0.f;
    if constexpr (REV) {
#pragma unroll 8
        for (int kk = 0; kk < N; ++kk) acc = fmaf(js[kk * MS + r], x[kk], acc);
    } else {
#pragma unroll 4
        for (int k4 = 0; k4 < N; k4 += 4) {
            const float4 m = *reinterpret_cast<const float4 *>(js + r * MS + k4);
            const float4 v = *reinterpret_cast<const float4 *>(x + k4);
            acc = fmaf(m.x, v.x, acc);
            acc = fmaf(m.y, v.y, acc);
            acc = fmaf(m.z, v.z, acc);
            acc = fmaf(m.w, v.w, acc);
        }
    }
    return acc;
}

// Two CTAs per SM: each step's matrix is copied into the other buffer while the current
// one is used (cp.async, waited for before the step's barrier), so the copies' latency
// overlaps the chain product.
template <int N, bool REV>
__device__ __forceinline__ void dense_scan_body(const DScanArgs &A, DScanSmem<N> &sm, int *s_fail, bool vec) {
    constexpr int TCH = DeerCfg<N>::TCH, BR = DeerCfg<N>::BR, TG = DeerCfg<N>::TG, MS = DScanSmem<N>::MS;
    const int tid = threadIdx.x;
    const int nchunk = (A.T + TCH - 1) / TCH;
    const long nseq = A.B;
    const long ntiles = nseq * nchunk;
    const unsigned epoch = A.epoch0 + 1u;
    TileWalk tw(nseq);
    for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next()) {
        const int chunk = tw.chunk;  // scan order
        const int b = tw.seq;
        const int tch = REV ? nchunk - 1 - chunk : chunk;
        const int tbeg = tch * TCH;
        const int steps = min(TCH, A.T - tbeg);
        auto time_of = [&](int i) { return REV ? tbeg + steps - 1 - i : tbeg + i; };
        for (int e = tid; e < N * N; e += kThreads) sm.P[0][e] = (e / N == e % N) ? 1.f : 0.f;
        if (tid < N) sm.D[0][tid] = 0.f;
        dscan_stage_M<N>(A, sm.Js[0], b, time_of(0), vec);
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        int cur = 0;
        for (int i = 0; i < steps; ++i) {
            const int t = time_of(i);
            if (i + 1 < steps) dscan_stage_M<N>(A, sm.Js[(i + 1) & 1], b, time_of(i + 1), vec);
            cp_async_commit();
            const float *js = sm.Js[i & 1];
            if (tid < TG * TG) dscan_chain_step<N, REV>(js, sm.P[cur], sm.P[cur ^ 1], (tid / TG) * BR, (tid % TG) * BR);
            if (tid >= kThreads - N) {
                const int r = tid - (kThreads - N);
                const float acc = dscan_row_dot<N, REV>(js, r, sm.D[cur]);
                sm.D[cur ^ 1][r] = (r < A.n) ? acc + A.b[((size_t)b * A.T + t) * A.n + r] : acc;
            }
            cp_async_wait_all();
            __syncthreads();
            cur ^= 1;
        }
        if (tid < N) {
            float cv = 0.f;
            if (chunk == 0) {
                cv = (A.h0 && tid < A.n) ? A.h0[(size_t)b * A.n + tid] : 0.f;
            } else if (!wait_word(A.inc + (tile - nseq) * N + tid, epoch, &cv, A.ctl, A.sticky, A.dbg)) {
                *s_fail = 1;
            }
            sm.carry[tid] = cv;
        }
        __syncthreads();
        if (*s_fail) return;
        if (tid < N) {
            float acc = sm.D[cur][tid];
            for (int j = 0; j < N; ++j) acc = fmaf(sm.P[cur][tid * N + j], sm.carry[j], acc);
            if (A.dbg.skip_tile != tile) st_relaxed_u64(A.inc + tile * N + tid, pack_tag(acc, epoch));
            sm.v[0][tid] = sm.carry[tid];
        }
        dscan_stage_M<N>(A, sm.Js[0], b, time_of(0), vec);
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        int vc = 0;
        for (int i = 0; i < steps; ++i) {
            const int t = time_of(i);
            if (i + 1 < steps) dscan_stage_M<N>(A, sm.Js[(i + 1) & 1], b, time_of(i + 1), vec);
            cp_async_commit();
            const float *js = sm.Js[i & 1];
            if (tid < 4 * N) {
                const int r = tid >> 2, q = tid & 3;
                float acc = 0.f;
                for (int kk = q; kk < N; kk += 4) acc = fmaf(REV ? js[kk * MS + r] : js[r * MS + kk], sm.v[vc][kk], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (q == 0) {
                    if (r < A.n) acc += A.b[((size_t)b * A.T + t) * A.n + r];
                    sm.v[vc ^ 1][r] = acc;
                    if (r < A.n) A.out[((size_t)b * A.T + t) * A.n + r] = acc;
                }
            }
            cp_async_wait_all();
            __syncthreads();
            vc ^= 1;
        }
    }
}

template <int N>
__global__ void __launch_bounds__(kThreads, 3) dense_scan_kernel(const DScanArgs A) {
    extern __shared__ __align__(16) unsigned char smraw[];
    DScanSmem<N> &sm = *reinterpret_cast<DScanSmem<N> *>(smraw);
    __shared__ int s_fail;
    const int tid = threadIdx.x;
    // 16-byte copies of whole rows: n % 4 == 0 (then every row start is 16-byte aligned)
    const bool vec = (A.n & 3) == 0 && ((uintptr_t)A.J & 15) == 0;
    if (tid == 0) s_fail = 0;
    // the padding of both staging buffers stays zero: the 16-byte copies never write it
    for (int e = tid; e < 2 * N * DScanSmem<N>::MS; e += kThreads) (&sm.Js[0][0])[e] = 0.f;
    __syncthreads();
    if (A.reverse)
        dense_scan_body<N, true>(A, sm, &s_fail, vec);
    else
        dense_scan_body<N, false>(A, sm, &s_fail, vec);
}

// Small states (n <= 8): one warp per tile, so the sequential walks synchronise with
// warp shuffles instead of CTA barriers.  Lane l holds P[r][c], P[r][c + 1] of the
// chunk map (r = l / 4, c = 2 (l % 4)) and D[r]; a step needs row r of M_t and the
// column entries P[k][c] from lane 4 k + l % 4.  The warp stages blocks of 32 steps
// of J and b in shared memory with cp.async, one block ahead of its walk.  Tiles are
// taken in increasing order by the warps of a cooperative grid, so a tile's
// predecessor is always resident or done; the carry chain across tiles is the
// inclusive chain of the kernel above.
constexpr int kDsw = 1024;            // steps per warp tile
constexpr int kDswBlk = 32;           // steps per staged block
constexpr int kDswWarps = 4;          // warps per CTA
constexpr int kDswBuf = kDswBlk * 72;  // floats per staging buffer: 32 (n^2 + n), n <= 8

// Stage J for times jt0 .. jt0 + 31 and b for times bt0 .. bt0 + 31 (zero beyond T).
__device__ __forceinline__ void dsw_stage(const DScanArgs &A, float *buf, int b, int jt0, int bt0) {
    const int lane = threadIdx.x & 31, n = A.n, nn = n * n;
    const size_t row = (size_t)b * A.T;
    for (int e = lane; e < kDswBlk * nn; e += 32) {
        const int tt = jt0 + e / nn;
        cp_async4(buf + e, A.J + (row + min(tt, A.T - 1)) * nn + e % nn, tt < A.T);
    }
    for (int e = lane; e < kDswBlk * n; e += 32) {
        const int tt = bt0 + e / n;
        cp_async4(buf + kDswBlk * nn + e, A.b + (row + min(tt, A.T - 1)) * n + e % n, tt < A.T);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(kDswWarps * 32) dense_scan_warp_kernel(const DScanArgs A) {
    extern __shared__ __align__(16) float dsw_smem[];
    const int lane = threadIdx.x & 31, r = lane >> 2, c = (lane & 3) * 2, n = A.n, nn = n * n;
    float *const buf0 = dsw_smem + (threadIdx.x >> 5) * 2 * kDswBuf;
    const long gw = (long)blockIdx.x * kDswWarps + (threadIdx.x >> 5);
    const long nwarps = (long)gridDim.x * kDswWarps;
    const int nchunk = (A.T + kDsw - 1) / kDsw;
    const long nseq = A.B;
    const long ntiles = nseq * nchunk;
    const unsigned epoch = A.epoch0 + 1u;
    for (long tile = gw; tile < ntiles; tile += nwarps) {
        const int chunk = (int)(tile / nseq), b = (int)(tile % nseq);  // scan order
        const int tch = A.reverse ? nchunk - 1 - chunk : chunk;
        const int tbeg = tch * kDsw;
        const int steps = min(kDsw, A.T - tbeg);
        const int nblk = (steps + kDswBlk - 1) / kDswBlk;
        // block j covers scan steps 32 j .. 32 j + 31; their times form one run
        auto blk_t0 = [&](int j) {  // smallest time of block j
            return A.reverse ? tbeg + steps - min(steps, kDswBlk * (j + 1)) : tbeg + kDswBlk * j;
        };
        auto stage = [&](int j) {
            const int t0 = blk_t0(j);
            dsw_stage(A, buf0 + (j & 1) * kDswBuf, b, A.reverse ? t0 + 1 : t0, t0);
        };
        // M_t row r (entries k < n) and b_t[r] of scan step i, from the staged block
        auto row_of = [&](int i, float *m, float &bt) {
            const int j = i / kDswBlk, t = A.reverse ? tbeg + steps - 1 - i : tbeg + i;
            const int t0 = blk_t0(j);
            const float *bf = buf0 + (j & 1) * kDswBuf;
#pragma unroll
            for (int k = 0; k < 8; ++k) m[k] = 0.f;
            bt = 0.f;
            if (r >= n) return;
            bt = bf[kDswBlk * nn + (t - t0) * n + r];
            if (!A.reverse) {
                const float *J = bf + (t - t0) * nn + r * n;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < n) m[k] = J[k];
            } else if (t + 1 < A.T) {  // row r of J_{t+1}^T
                const float *J = bf + (t + 1 - (t0 + 1)) * nn + r;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < n) m[k] = J[k * n];
            } else {
                m[r] = 1.f;
            }
        };
        // walk 1: the chunk map x -> P x + D
        float p0 = (r == c) ? 1.f : 0.f, p1 = (r == c + 1) ? 1.f : 0.f, d = 0.f;
        stage(0);
        for (int j = 0; j < nblk; ++j) {
            if (j + 1 < nblk) {
                stage(j + 1);
                asm volatile("cp.async.wait_group 1;" ::: "memory");
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
            __syncwarp();
            const int iend = min(steps, kDswBlk * (j + 1));
            for (int i = kDswBlk * j; i < iend; ++i) {
                float m[8], bt;
                row_of(i, m, bt);
                float q0 = 0.f, q1 = 0.f, qd = bt;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    q0 = fmaf(m[k], __shfl_sync(0xffffffffu, p0, 4 * k + (lane & 3)), q0);
                    q1 = fmaf(m[k], __shfl_sync(0xffffffffu, p1, 4 * k + (lane & 3)), q1);
                    qd = fmaf(m[k], __shfl_sync(0xffffffffu, d, 4 * k), qd);
                }
                p0 = q0;
                p1 = q1;
                d = qd;
            }
            __syncwarp();  // the buffer of block j is refilled by stage(j + 2)
        }
        // carry entering the tile, then publish this tile's inclusive value
        float cv = 0.f;
        int bad = 0;
        if (lane < 8) {
            if (chunk == 0) {
                cv = (A.h0 && lane < n) ? A.h0[(size_t)b * n + lane] : 0.f;
            } else if (!wait_word(A.inc + (tile - nseq) * 8 + lane, epoch, &cv, A.ctl, A.sticky, A.dbg)) {
                bad = 1;
            }
        }
        if (__any_sync(0xffffffffu, bad)) return;  // a bounded wait ran out; the status says so
        const float c0 = __shfl_sync(0xffffffffu, cv, c), c1 = __shfl_sync(0xffffffffu, cv, c + 1);
        float inc = fmaf(p0, c0, p1 * c1);
        inc += __shfl_xor_sync(0xffffffffu, inc, 1);
        inc += __shfl_xor_sync(0xffffffffu, inc, 2);
        inc += d;
        if ((lane & 3) == 0 && A.dbg.skip_tile != tile) st_relaxed_u64(A.inc + tile * 8 + r, pack_tag(inc, epoch));
        // walk 2: the outputs from the carry
        float v = __shfl_sync(0xffffffffu, cv, r);  // v[r], replicated over the row's lanes
        stage(0);
        for (int j = 0; j < nblk; ++j) {
            if (j + 1 < nblk) {
                stage(j + 1);
                asm volatile("cp.async.wait_group 1;" ::: "memory");
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
            __syncwarp();
            const int iend = min(steps, kDswBlk * (j + 1));
            for (int i = kDswBlk * j; i < iend; ++i) {
                const int t = A.reverse ? tbeg + steps - 1 - i : tbeg + i;
                float m[8], bt;
                row_of(i, m, bt);
                float q = bt;
#pragma unroll
                for (int k = 0; k < 8; ++k) q = fmaf(m[k], __shfl_sync(0xffffffffu, v, 4 * k), q);
                v = q;
                if ((lane & 3) == 0 && r < n) A.out[((size_t)b * A.T + t) * n + r] = v;
            }
            __syncwarp();
        }
    }
}

// ------------------------------------------------------------------ host side
namespace {

int pad_n(int n) {
    int N = 8;
    while (N < n) N <<= 1;
    return N;
}

template <class K> int set_smem(K kern, size_t bytes) {
    return cudaFuncSetAttribute(reinterpret_cast<const void *>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)bytes) == cudaSuccess
               ? 0
               : -1;
}

template <int N> size_t deer_smem() {
    return ((sizeof(TanhSmem<N, DeerCfg<N>::TCH>) + 15) & ~size_t(15)) + sizeof(DeerExtra<N>);
}
template <int N> size_t quasi_smem() { return sizeof(QuasiSmem<N>); }

template <int N> int tanh_plan_n(const NewtonTanhReq &r, int num_sms, Plan *plan) {
    if (r.quasi) {
        constexpr int TCH = QuasiCfg<N>::TCH;
        auto kern = &tanh_quasi_kernel<N>;
        const size_t sm = quasi_smem<N>();
        if (set_smem(kern, sm)) return -1;
        plan->kernel = reinterpret_cast<const void *>(kern);
        plan->dyn_smem = (int)sm;
        plan->ntiles = (long)r.B * ((r.T + TCH - 1) / TCH);
        plan->C = N;
        plan->agg_words = (size_t)plan->ntiles * N * 2 * (N > 32 ? 1 : 1);
        plan->inc_words = (size_t)plan->ntiles * N;
    } else {
        constexpr int TCH = DeerCfg<N>::TCH;
        auto kern = &tanh_deer_kernel<N>;
        const size_t sm = deer_smem<N>();
        if (set_smem(kern, sm)) return -1;
        plan->kernel = reinterpret_cast<const void *>(kern);
        plan->dyn_smem = (int)sm;
        plan->ntiles = (long)r.B * ((r.T + TCH - 1) / TCH);
        plan->C = N;
        plan->agg_words = 0;
        plan->inc_words = (size_t)plan->ntiles * N;
    }
    plan->side_bytes = 2 * (size_t)plan->ntiles * N * sizeof(float);
    plan->epochs = (unsigned)r.max_iters + 1u;
    plan->variant = N;
    plan->grid = occupancy_grid(plan->kernel, kThreads, plan->dyn_smem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

}  // namespace

int newton_tanh_plan(const NewtonTanhReq &r, int num_sms, Plan *plan) {
    if (r.n > 64) return 1;
    if (!r.xproj && (r.in < 1 || r.in > 8)) return 1;
    const int q8 = tanh_quasi8_plan(r, num_sms, plan);  // warp-per-unit kernel for n == 8
    if (q8 <= 0) return q8;
    const int tc = deer_tc_plan(r, num_sms, plan);  // tensor-core chain products for 32 < n <= 64
    if (tc <= 0) return tc;
    switch (pad_n(r.n)) {
        case 8: return tanh_plan_n<8>(r, num_sms, plan);
        case 16: return tanh_plan_n<16>(r, num_sms, plan);
        case 32: return tanh_plan_n<32>(r, num_sms, plan);
        default: return tanh_plan_n<64>(r, num_sms, plan);
    }
}

cudaError_t newton_tanh_launch(const NewtonTanhReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                               cudaStream_t st) {
    if (plan.variant == 1108) return tanh_quasi8_launch(r, plan, w, dbg, st);
    if (plan.variant == 1164) return deer_tc_launch(r, plan, w, dbg, st);
    TanhArgs A;
    A.B = r.B;
    A.T = r.T;
    A.n = r.n;
    A.jmode = r.jmode;
    A.in = r.in;
    A.xproj = r.xproj;
    A.x = r.x;
    A.W = r.W;
    A.bias = r.bias;
    A.A = r.A;
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
    A.dbg.no_halo = 1;
    void *args[] = {&A};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(kThreads), args, plan.dyn_smem, st);
}

int scan_dense_plan(const ScanReq &r, int num_sms, Plan *plan) {
    if (r.N > 64) return 1;
    const int N = pad_n(r.N);
    if (N == 8) {  // one warp per tile
        plan->kernel = reinterpret_cast<const void *>(&dense_scan_warp_kernel);
        plan->dyn_smem = kDswWarps * 2 * kDswBuf * (int)sizeof(float);
        if (cudaFuncSetAttribute(plan->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, plan->dyn_smem) !=
            cudaSuccess)
            return -1;
        plan->ntiles = (long)r.B * ((r.T + kDsw - 1) / kDsw);
        plan->C = N;
        plan->agg_words = 0;
        plan->inc_words = (size_t)plan->ntiles * 8;
        plan->side_bytes = 0;
        plan->epochs = 2;
        plan->variant = 1008;
        plan->threads = kDswWarps * 32;
        const long ctas = (plan->ntiles + kDswWarps - 1) / kDswWarps;
        plan->grid = occupancy_grid(plan->kernel, plan->threads, plan->dyn_smem, num_sms, ctas);
        return plan->grid > 0 ? 0 : -1;
    }
    size_t sm = 0;
    const void *kern = nullptr;
    int TCH = 0;
    switch (N) {
        case 8: kern = reinterpret_cast<const void *>(&dense_scan_kernel<8>); sm = sizeof(DScanSmem<8>); TCH = DeerCfg<8>::TCH; break;
        case 16: kern = reinterpret_cast<const void *>(&dense_scan_kernel<16>); sm = sizeof(DScanSmem<16>); TCH = DeerCfg<16>::TCH; break;
        case 32: kern = reinterpret_cast<const void *>(&dense_scan_kernel<32>); sm = sizeof(DScanSmem<32>); TCH = DeerCfg<32>::TCH; break;
        default: kern = reinterpret_cast<const void *>(&dense_scan_kernel<64>); sm = sizeof(DScanSmem<64>); TCH = DeerCfg<64>::TCH; break;
    }
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess) return -1;
    plan->kernel = kern;
    plan->dyn_smem = (int)sm;
    plan->ntiles = (long)r.B * ((r.T + TCH - 1) / TCH);
    plan->C = N;
    plan->agg_words = 0;
    plan->inc_words = (size_t)plan->ntiles * N;
    plan->side_bytes = 0;
    plan->epochs = 2;
    plan->variant = N;
    plan->grid = occupancy_grid(plan->kernel, kThreads, plan->dyn_smem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t scan_dense_launch(const ScanReq &r, const Plan &plan, const Work &w, const DbgHost &dbg, cudaStream_t st) {
    DScanArgs A;
    A.B = r.B;
    A.T = r.T;
    A.n = r.N;
    A.reverse = r.reverse;
    A.J = r.J;
    A.b = r.b;
    A.h0 = r.h0;
    A.out = r.out;
    A.ctl = w.ctl;
    A.sticky = w.sticky;
    A.inc = w.inc;
    A.epoch0 = w.epoch0;
    A.dbg.wait_ns = dbg.wait_ns;
    A.dbg.skip_tile = dbg.skip_tile;
    A.dbg.delta_log = nullptr;
    A.dbg.delta_log_cap = 0;
    A.dbg.no_halo = 1;
    void *args[] = {&A};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(plan.threads), args, plan.dyn_smem, st);
}

}  // namespace prn
