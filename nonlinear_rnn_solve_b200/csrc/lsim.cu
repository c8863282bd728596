// lsim.cu -- fixed-step simulation of a linear time-invariant system
//   dx/dt = A x + B u,  y = C x + D u
// by a chunked linear scan ("Para-Seq" README, Quick example `lsim(A, B, C, D, U, t)`,
// and the `src.ode_solvers` row of Main features: scan-based fixed-step linear
// simulation; Notes and limitations: fixed-step time grids only).
//
// One step of the ODE is exact for an input held over the step (zero-order hold) or
// varying linearly between samples (first-order hold):
//   x_0 = x0,   x_k = Ad x_{k-1} + G0 u_{k-1} + G1 u_k   (k >= 1),   y_k = C x_k + D u_k,
// with Ad = e^{A h} and G0, G1 from the exponential of one block upper-triangular
// matrix (Van Loan's construction), computed on the device in fp64 by scaling and
// squaring of a Taylor polynomial.
//
// The matrix of the recurrence is the same at every step, so the scan carries states
// only: a thread takes 32 consecutive steps and emits the chunk's end state from a
// zero state (a contraction of the chunk's inputs with 33 precomputed matrices, or the
// recurrence stepped); those end states form a sequence of the same kind with matrix
// Ad^32, chunked again until one chunk covers a level; a fix-up pass turns every
// level's end states into the states entering the next chunk, top down; the last pass
// re-runs each 32-step chunk from its entering state and writes y (and x).  Every pass
// is independent per thread: no CTA waits on another.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace prn {

namespace {

constexpr int kChunk = 32;     // steps per thread, every level
constexpr int kThreadsL = 128;  // threads per CTA of the input-level passes
constexpr int kThreadsLv = 32;  // of the upper-level passes (few threads: spread over the SMs)
constexpr int kDiscThreads = 1024;
constexpr int kTaylor = 10;  // degree; the scaled matrix has 1-norm <= 1/4

__host__ __device__ constexpr long up4(long x) { return (x + 3) & ~3L; }

// Offsets (floats) of the fp32 matrices the discretisation writes, padded to NP:
// AdT [NP][NP] (AdT[j][i] = Ad[i][j]), G0T, G1T [m][NP], Cp [p][NP], Dm [p][m], the
// chunk kernels KT [33][m][NP] (below), then the transposed chunk powers Ad^(32^l),
// l = 1 .. levels, [NP][NP] each at a stride of ps floats.  Every offset is a multiple
// of 4 floats (16-byte copies).
struct MatLayout {
    long ad, g0, g1, c, d, kk, pw, ps, total;
    __host__ __device__ MatLayout(int NP, int m, int p, int levels) {
        ps = up4((long)NP * NP);
        ad = 0;
        g0 = up4(ad + (long)NP * NP);
        g1 = up4(g0 + (long)m * NP);
        c = up4(g1 + (long)m * NP);
        d = up4(c + (long)p * NP);
        kk = up4(d + (long)p * m);
        pw = up4(kk + (long)(kChunk + 1) * m * NP);
        total = pw + levels * ps;
    }
};

// The end state of a 32-step chunk k0 .. k0 + 31 (k0 >= 1) run from a zero state is
// linear in its inputs u_{k0-1} .. u_{k0+31}:
//   x_{k0+31} = sum_{l=-1}^{31} K_l u_{k0+l},
//   K_l = Ad^(30-l) (G0 + Ad G1) (0 <= l <= 30),  K_31 = G1,  K_{-1} = Ad^31 G0,
// so the first pass contracts each chunk's inputs with these 33 n x m matrices (n m
// multiply-adds per step) instead of stepping the recurrence (n^2 + n m), where they
// fit in shared memory.
constexpr long kMaxChunkKernelFloats = 8192;
__host__ __device__ inline bool use_chunk_kernels(int NP, int m) {
    return (long)(kChunk + 1) * m * NP <= kMaxChunkKernelFloats;
}

// ------------------------------------------------------------------ discretisation (fp64)
// Z [n x m] = X [n x n] Y [n x m], row-major in shared memory, by the whole CTA.
__device__ void smem_matmul_rect(const double *X, const double *Y, double *Z, int n, int m) {
    for (int idx = threadIdx.x; idx < n * m; idx += blockDim.x) {
        const int i = idx / m, j = idx % m;
        double acc = 0.0;
        for (int k = 0; k < n; ++k) acc = fma(X[i * n + k], Y[k * m + j], acc);
        Z[idx] = acc;
    }
    __syncthreads();
}

// Product of q x q row-major matrices in shared memory, by the whole CTA: a 2 x 2
// block of Z per thread (one shared load per multiply-add).
__device__ void smem_matmul(const double *X, const double *Y, double *Z, int q) {
    const int qb = (q + 1) / 2;
    for (int idx = threadIdx.x; idx < qb * qb; idx += blockDim.x) {
        const int i0 = 2 * (idx / qb), j0 = 2 * (idx % qb);
        const int i1 = min(i0 + 1, q - 1), j1 = min(j0 + 1, q - 1);
        double a00 = 0.0, a01 = 0.0, a10 = 0.0, a11 = 0.0;
        for (int k = 0; k < q; ++k) {
            const double x0 = X[i0 * q + k], x1 = X[i1 * q + k], y0 = Y[k * q + j0], y1 = Y[k * q + j1];
            a00 = fma(x0, y0, a00);
            a01 = fma(x0, y1, a01);
            a10 = fma(x1, y0, a10);
            a11 = fma(x1, y1, a11);
        }
        Z[i0 * q + j0] = a00;
        if (j0 + 1 < q) Z[i0 * q + j0 + 1] = a01;
        if (i0 + 1 < q) {
            Z[(i0 + 1) * q + j0] = a10;
            if (j0 + 1 < q) Z[(i0 + 1) * q + j0 + 1] = a11;
        }
    }
    __syncthreads();
}

// One CTA: e^M for M = [[A h, B h, 0], [0, 0, I], [0, 0, 0]] (the last block row and
// column only with the linear hold), by scaling M to 1-norm <= 1/4, a degree-10
// Taylor polynomial in Horner form (truncation below 1e-14 relative), and squaring
// back (Moler and Van Loan, "Nineteen dubious ways to compute the exponential of a
// matrix", method 3).  Then the chunk powers Ad^(32^l) by five squarings per level.
__global__ void __launch_bounds__(kDiscThreads) lsim_discretize_kernel(const float *A, const float *Bm, const float *C,
                                                                      const float *D, int n, int m, int p, double h,
                                                                      int interp, int NP, int levels, float *mats) {
    extern __shared__ double dsm[];
    const int q = n + m * (interp ? 2 : 1);
    double *X = dsm, *E = dsm + q * q, *Tm = dsm + 2 * q * q;
    __shared__ double s_factor;
    __shared__ int s_squarings;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < q * q; idx += blockDim.x) {
        const int i = idx / q, j = idx % q;
        double v = 0.0;
        if (i < n && j < n) v = (double)A[i * n + j] * h;
        else if (i < n && j < n + m) v = (double)Bm[i * m + (j - n)] * h;
        else if (interp && i >= n && i < n + m && j >= n + m) v = (i - n == j - n - m) ? 1.0 : 0.0;
        X[idx] = v;
    }
    __syncthreads();
    if (tid == 0) {
        double nrm = 0.0;
        for (int j = 0; j < q; ++j) {
            double cs = 0.0;
            for (int i = 0; i < q; ++i) cs += fabs(X[i * q + j]);
            nrm = fmax(nrm, cs);
        }
        int s = 0;
        double scale = 1.0;
        while (!(nrm * scale <= 0.25) && s < 1100) {  // NaN stops at the bound
            scale *= 0.5;
            ++s;
        }
        s_factor = scale;
        s_squarings = s;
    }
    __syncthreads();
    const double scale = s_factor;
    const int sq = s_squarings;
    for (int idx = tid; idx < q * q; idx += blockDim.x) {
        X[idx] *= scale;
        E[idx] = (idx / q == idx % q) ? 1.0 : 0.0;
    }
    __syncthreads();
    // Horner: E <- I + X E / k for k = K .. 1 gives sum_{i <= K} X^i / i!
    for (int k = kTaylor; k >= 1; --k) {
        smem_matmul(X, E, Tm, q);
        const double inv = 1.0 / (double)k;
        for (int idx = tid; idx < q * q; idx += blockDim.x)
            E[idx] = ((idx / q == idx % q) ? 1.0 : 0.0) + Tm[idx] * inv;
        __syncthreads();
    }
    for (int s = 0; s < sq; ++s) {
        smem_matmul(E, E, Tm, q);
        double *t = E;
        E = Tm;
        Tm = t;
    }
    const MatLayout Lm(NP, m, p, levels);
    // Ad, G0, G1, C, D in the padded fp32 layouts (zero padding keeps extra state
    // components at zero)
    for (int idx = tid; idx < NP * NP; idx += blockDim.x) {
        const int j = idx / NP, i = idx % NP;
        mats[Lm.ad + idx] = (i < n && j < n) ? (float)E[i * q + j] : 0.f;
    }
    for (int idx = tid; idx < m * NP; idx += blockDim.x) {
        const int qq = idx / NP, i = idx % NP;
        float g0 = 0.f, g1 = 0.f;
        if (i < n) {
            const double p0 = E[i * q + n + qq];
            const double p1 = interp ? E[i * q + n + m + qq] : 0.0;
            g0 = (float)(p0 - p1);
            g1 = (float)p1;
        }
        mats[Lm.g0 + idx] = g0;
        mats[Lm.g1 + idx] = g1;
    }
    for (int idx = tid; idx < p * NP; idx += blockDim.x) {
        const int r = idx / NP, j = idx % NP;
        mats[Lm.c + idx] = j < n ? C[r * n + j] : 0.f;
    }
    for (int idx = tid; idx < p * m; idx += blockDim.x) mats[Lm.d + idx] = D ? D[idx] : 0.f;
    if (use_chunk_kernels(NP, m)) {
        // chunk kernels K_l; X holds Ad [n n] | V [n m] | W [n m] (q^2 >= n^2 + 2 n m)
        double *Ad = X, *V = X + n * n, *W = V + n * m;
        __syncthreads();
        for (int idx = tid; idx < n * n; idx += blockDim.x) Ad[idx] = E[(idx / n) * q + idx % n];
        auto g0 = [&](int i, int qq) { return E[i * q + n + qq] - (interp ? E[i * q + n + m + qq] : 0.0); };
        auto g1 = [&](int i, int qq) { return interp ? E[i * q + n + m + qq] : 0.0; };
        auto put = [&](int l, const double *M) {  // K_l (l = -1 .. 31) from M [n m] (NULL: G1)
            for (int idx = tid; idx < m * NP; idx += blockDim.x) {
                const int qq = idx / NP, i = idx % NP;
                const double v = i < n ? (M ? M[i * m + qq] : g1(i, qq)) : 0.0;
                mats[Lm.kk + (long)(l + 1) * m * NP + idx] = (float)v;
            }
        };
        for (int idx = tid; idx < n * m; idx += blockDim.x) W[idx] = g1(idx / m, idx % m);
        __syncthreads();
        smem_matmul_rect(Ad, W, V, n, m);  // V = Ad G1
        for (int idx = tid; idx < n * m; idx += blockDim.x) V[idx] += g0(idx / m, idx % m);
        __syncthreads();
        for (int l = 30; l >= 0; --l) {  // K_l = Ad^(30-l) (G0 + Ad G1)
            put(l, V);
            if (l > 0) {
                smem_matmul_rect(Ad, V, W, n, m);
                for (int idx = tid; idx < n * m; idx += blockDim.x) V[idx] = W[idx];
                __syncthreads();
            }
        }
        put(31, nullptr);  // K_31 = G1
        for (int idx = tid; idx < n * m; idx += blockDim.x) V[idx] = g0(idx / m, idx % m);
        __syncthreads();
        for (int r = 0; r < kChunk - 1; ++r) {  // K_{-1} = Ad^31 G0
            smem_matmul_rect(Ad, V, W, n, m);
            for (int idx = tid; idx < n * m; idx += blockDim.x) V[idx] = W[idx];
            __syncthreads();
        }
        put(-1, V);
    }
    // chunk powers: X <- Ad (n x n), then five squarings per level
    __syncthreads();
    for (int idx = tid; idx < n * n; idx += blockDim.x) X[idx] = E[(idx / n) * q + idx % n];
    __syncthreads();
    double *P = X, *Q = Tm;
    for (int l = 0; l < levels; ++l) {
        for (int s = 0; s < 5; ++s) {
            smem_matmul(P, P, Q, n);
            double *t = P;
            P = Q;
            Q = t;
        }
        for (int idx = tid; idx < NP * NP; idx += blockDim.x) {
            const int j = idx / NP, i = idx % NP;
            mats[Lm.pw + l * Lm.ps + idx] = (i < n && j < n) ? (float)P[i * n + j] : 0.f;
        }
    }
}

// ------------------------------------------------------------------ chunk passes
// 16-byte shared-memory load kept inside the step loop: hoisting a whole NP x NP
// matrix out of the loop into registers would spill it to local memory.
__device__ __forceinline__ float4 lds4(const float *p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"((unsigned)__cvta_generic_to_shared(p)));
    return v;
}

// y += M x for M given transposed in shared memory (MT[j][i] = M[i][j]); every lane
// of a warp reads the same row at the same time (a broadcast).
template <int NP>
__device__ __forceinline__ void mv_acc(const float *MT, const float (&x)[NP], float (&y)[NP]) {
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const float xj = x[j];
        if constexpr (NP % 4 == 0) {
#pragma unroll
            for (int i = 0; i < NP; i += 4) {
                const float4 a = lds4(MT + j * NP + i);
                y[i] = fmaf(a.x, xj, y[i]);
                y[i + 1] = fmaf(a.y, xj, y[i + 1]);
                y[i + 2] = fmaf(a.z, xj, y[i + 2]);
                y[i + 3] = fmaf(a.w, xj, y[i + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < NP; ++i) y[i] = fmaf(MT[j * NP + i], xj, y[i]);
        }
    }
}

// NP floats of a level element (16-byte aligned when NP is a multiple of 4).
template <int NP> __device__ __forceinline__ void load_vec(const float *p, float (&v)[NP]) {
    if constexpr (NP % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NP; i += 4) {
            const float4 t = *reinterpret_cast<const float4 *>(p + i);
            v[i] = t.x;
            v[i + 1] = t.y;
            v[i + 2] = t.z;
            v[i + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < NP; ++i) v[i] = p[i];
    }
}
template <int NP> __device__ __forceinline__ void store_vec(float *p, const float (&v)[NP]) {
    if constexpr (NP % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NP; i += 4) *reinterpret_cast<float4 *>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
#pragma unroll
        for (int i = 0; i < NP; ++i) p[i] = v[i];
    }
}

struct LsimArgs {
    long B, T;      // sequences and steps of the input level
    int n, m, p, interp;
    const float *U, *x0;
    float *y, *x;
    const float *mats;
    long mat_pw;    // offset of this level's chunk power (levels >= 1)
    float *agg_in;  // level >= 1: the level's elements (fix: rewritten in place)
    float *agg_out; // end states of this level's chunks
    const float *carry;  // inclusive end states of the level above (NULL: none)
};

// Load the matrices a pass needs into shared memory (float4 copies of 4-float runs).
__device__ __forceinline__ void stage_mats(float *dst, const float *src, long count) {
    for (long i = threadIdx.x * 4L; i < count; i += blockDim.x * 4L)
        *reinterpret_cast<float4 *>(dst + i) = *reinterpret_cast<const float4 *>(src + i);
    __syncthreads();
}

// The input-level passes read and write the samples through shared memory.  A CTA's
// threads own consecutive chunks, whose steps are consecutive in the flattened
// [batch, T] order, and the CTA walks them in sub-blocks of SB steps: per sub-block
// it copies every chunk's SB + 1 input rows (from the step before the sub-block on;
// consecutive threads read consecutive floats of a chunk's rows) and, in the last
// pass, writes the SB output rows back the same way.  Row strides are odd, so threads
// reading their own chunk's rows hit distinct banks.
struct IoPlan {
    int SB;          // steps per sub-block: 1, 2, 4 or 8 (divides the chunk)
    int ustr, ystr;  // floats per chunk: input rows, output rows
};

// Per-CTA chunk table, filled by each thread for its own chunk: the flattened index
// of the chunk's first step (b T + 32 j), the steps left in its sequence from there
// (T - 32 j, capped at 33, beyond which no row of a chunk reaches, so the products
// with m or p below stay small; a large negative number for a thread past the last
// chunk, so no row of it is ever in range) and whether it is a sequence's first chunk
// (whose row before the first step does not exist), so the copy loops need no
// per-element division or 64-bit bounds arithmetic.
struct ChunkTab {
    long flat[kThreadsL];
    int rem[kThreadsL];
    int first[kThreadsL];
};
constexpr int kNoRows = -(1 << 24);

__device__ __forceinline__ void fill_tab(ChunkTab &tab, bool valid, long b, long j, long T) {
    tab.flat[threadIdx.x] = valid ? b * T + j * kChunk : 0;
    tab.rem[threadIdx.x] = valid ? (int)min(T - j * kChunk, (long)kChunk + 1) : kNoRows;
    tab.first[threadIdx.x] = j == 0;
}

// Issue the copies of rows k0 + s SB - 1 .. k0 + s SB + SB - 1 of every chunk (zero
// outside 0 <= k < T) as one commit group; consecutive threads take consecutive
// floats of a chunk's rows.
__device__ __forceinline__ void stage_u(const LsimArgs &A, int m, const IoPlan &io, const ChunkTab &tab, float *su,
                                        int s) {
    const int rows = (io.SB + 1) * m;
    const float inv = 1.0f / (float)rows;  // exact quotient below: e < 2^15, rows <= 144
    const int sb = s * io.SB;
    for (int e = threadIdx.x; e < kThreadsL * rows; e += kThreadsL) {
        const int c = __float2int_rd(((float)e + 0.5f) * inv), w = e - c * rows;
        // row r = w / m is step k0 + sb - 1 + r: inside the sequence when
        // sb - 1 + r < rem, and r > 0 for the first chunk's first sub-block
        const bool ok = w < (tab.rem[c] - sb + 1) * m && (w >= m || sb > 0 || !tab.first[c]);
        const long src = (tab.flat[c] + sb - 1) * m + w;
        cp_async4(su + c * io.ustr + w, A.U + (ok ? src : 0), ok);
    }
    cp_async_commit();
}

// Write the SB output rows of every chunk's sub-block s (steps below T); consecutive
// threads take consecutive floats of a chunk's rows.
__device__ __forceinline__ void store_y(const LsimArgs &A, int p, const IoPlan &io, const ChunkTab &tab,
                                        const float *sy, int s) {
    const int rows = io.SB * p;
    const float inv = 1.0f / (float)rows;
    const int sb = s * io.SB;
    for (int e = threadIdx.x; e < kThreadsL * rows; e += kThreadsL) {
        const int c = __float2int_rd(((float)e + 0.5f) * inv), w = e - c * rows;
        if (w < (tab.rem[c] - sb) * p) A.y[(tab.flat[c] + sb) * p + w] = sy[c * io.ystr + w];
    }
}

// One step of the input level, k >= 1: x <- Ad x + G0 u_{k-1} + G1 u_k (up, uk: the
// staged rows of steps k - 1 and k).  MM > 0: the input width m as a constant.
template <int NP, int MM>
__device__ __forceinline__ void input_step(const LsimArgs &A, const float *sAd, const float *sG0, const float *sG1,
                                           const float *up, const float *uk, float (&x)[NP]) {
    const int m = MM > 0 ? MM : A.m;
    float y[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) y[i] = 0.f;
    mv_acc<NP>(sAd, x, y);
#pragma unroll 4
    for (int q = 0; q < m; ++q) {
        const float u0 = up[q];
#pragma unroll
        for (int i = 0; i < NP; ++i) y[i] = fmaf(sG0[q * NP + i], u0, y[i]);
    }
    if (A.interp) {
#pragma unroll 4
        for (int q = 0; q < m; ++q) {
            const float u1 = uk[q];
#pragma unroll
            for (int i = 0; i < NP; ++i) y[i] = fmaf(sG1[q * NP + i], u1, y[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = y[i];
}

template <int NP>
__device__ __forceinline__ void load_x0(const LsimArgs &A, long b, float (&x)[NP]) {
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = (A.x0 && i < A.n) ? A.x0[b * A.n + i] : 0.f;
}

// Input level, first pass: each thread's chunk from a zero state (chunk 0 from x0);
// writes the chunk's end state.
template <int NP, int MM>
__global__ void __launch_bounds__(kThreadsL) lsim_local0_kernel(const LsimArgs A, const IoPlan io) {
    const int m = MM > 0 ? MM : A.m;
    extern __shared__ __align__(16) float sm[];
    const MatLayout Lm(NP, A.m, A.p, 0);
    const bool kern = use_chunk_kernels(NP, m);
    const long staged = kern ? Lm.pw : Lm.c;  // with the chunk kernels KT
    stage_mats(sm, A.mats, staged);
    float *su = sm + staged;
    const long nch = (A.T + kChunk - 1) / kChunk;
    const long g0 = (long)blockIdx.x * kThreadsL, g = g0 + threadIdx.x;
    const bool valid = g < A.B * nch;
    const long b = valid ? g / nch : 0, j = valid ? g % nch : 0;
    const long k1 = valid ? min(A.T, (j + 1) * kChunk) : 0;
    __shared__ ChunkTab tab;
    fill_tab(tab, valid, b, j, A.T);
    float x[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = 0.f;
    __syncthreads();
    const int nsb = kChunk / io.SB;
    stage_u(A, m, io, tab, su, 0);
    for (int s = 0; s < nsb; ++s) {
        // two input buffers: the next sub-block's copies fly during this one's steps
        if (s + 1 < nsb) {
            stage_u(A, m, io, tab, su + ((s + 1) & 1) * kThreadsL * io.ustr, s + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_all();
        }
        __syncthreads();
        const float *row = su + (s & 1) * kThreadsL * io.ustr + threadIdx.x * io.ustr;
        if (kern && j > 0) {
            // x += K_l u_l for the sub-block's rows l = s SB - 1 (first sub-block only:
            // later ones start at the row the previous one ended with) .. s SB + SB - 1;
            // rows past T were staged as zeros
            for (int r = s == 0 ? 0 : 1; r <= io.SB; ++r) {
                const float *KT = sm + Lm.kk + (long)(s * io.SB + r) * m * NP;
#pragma unroll 4
                for (int q = 0; q < m; ++q) {
                    const float uq = row[r * m + q];
                    if constexpr (NP % 4 == 0) {
#pragma unroll
                        for (int i = 0; i < NP; i += 4) {
                            const float4 kv = lds4(KT + q * NP + i);
                            x[i] = fmaf(kv.x, uq, x[i]);
                            x[i + 1] = fmaf(kv.y, uq, x[i + 1]);
                            x[i + 2] = fmaf(kv.z, uq, x[i + 2]);
                            x[i + 3] = fmaf(kv.w, uq, x[i + 3]);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < NP; ++i) x[i] = fmaf(KT[q * NP + i], uq, x[i]);
                    }
                }
            }
        } else {
            for (int i = 0; i < io.SB; ++i) {
                const long k = j * kChunk + (long)s * io.SB + i;
                if (k >= k1) break;
                if (k == 0)
                    load_x0<NP>(A, b, x);
                else
                    input_step<NP, MM>(A, sm + Lm.ad, sm + Lm.g0, sm + Lm.g1, row + i * m, row + (i + 1) * m, x);
            }
        }
        __syncthreads();
    }
    if (valid) store_vec<NP>(A.agg_out + g * NP, x);
}

// Upper levels: elements e_k (NP floats each) with matrix P = Ad^(32^l):
//   local (FIX false): end state of each chunk of 32 elements from a zero state;
//   fix (FIX true):    states c_k = P c_{k-1} + e_k from the entering state (the
//                      inclusive end state of the previous chunk, one level up),
//                      written over e_k.
template <int NP, bool FIX>
__global__ void __launch_bounds__(kThreadsLv) lsim_level_kernel(const LsimArgs A) {
    extern __shared__ __align__(16) float sm[];
    stage_mats(sm, A.mats + A.mat_pw, up4((long)NP * NP));
    const long nch = (A.T + kChunk - 1) / kChunk;
    const long g = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= A.B * nch) return;
    const long b = g / nch, j = g % nch;
    float x[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = (FIX && j > 0 && A.carry) ? A.carry[(g - 1) * NP + i] : 0.f;
    const long k1 = min(A.T, (j + 1) * kChunk);
    float *e = A.agg_in + (b * A.T + j * kChunk) * NP;
    float en[NP];  // the next element, loaded one step ahead
    load_vec<NP>(e, en);
    for (long k = j * kChunk; k < k1; ++k, e += NP) {
        float y[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) y[i] = en[i];
        if (k + 1 < k1) load_vec<NP>(e + NP, en);
        mv_acc<NP>(sm, x, y);
#pragma unroll
        for (int i = 0; i < NP; ++i) x[i] = y[i];
        if (FIX) store_vec<NP>(e, x);
    }
    if (!FIX) store_vec<NP>(A.agg_out + g * NP, x);
}

// Input level, last pass: each chunk from its entering state; writes y and x.
template <int NP, int MM, int PP>
__global__ void __launch_bounds__(kThreadsL) lsim_out_kernel(const LsimArgs A, const IoPlan io) {
    const int m = MM > 0 ? MM : A.m, p = PP > 0 ? PP : A.p;
    extern __shared__ __align__(16) float sm[];
    const MatLayout Lm(NP, A.m, A.p, 0);
    stage_mats(sm, A.mats, Lm.pw);
    float *su = sm + Lm.pw, *sy = su + 2 * kThreadsL * io.ustr;
    const long nch = (A.T + kChunk - 1) / kChunk;
    const long g0 = (long)blockIdx.x * kThreadsL, g = g0 + threadIdx.x;
    const bool valid = g < A.B * nch;
    const long b = valid ? g / nch : 0, j = valid ? g % nch : 0;
    const long k1 = valid ? min(A.T, (j + 1) * kChunk) : 0;
    float *yrow = sy + threadIdx.x * io.ystr;
    const float *sC = sm + Lm.c, *sD = sm + Lm.d;
    __shared__ ChunkTab tab;
    fill_tab(tab, valid, b, j, A.T);
    float x[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = (valid && j > 0 && A.carry) ? A.carry[(g - 1) * NP + i] : 0.f;
    __syncthreads();
    const int nsb = kChunk / io.SB;
    stage_u(A, m, io, tab, su, 0);
    for (int s = 0; s < nsb; ++s) {
        if (s + 1 < nsb) {
            stage_u(A, m, io, tab, su + ((s + 1) & 1) * kThreadsL * io.ustr, s + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_all();
        }
        __syncthreads();
        const float *row = su + (s & 1) * kThreadsL * io.ustr + threadIdx.x * io.ustr;
        for (int i = 0; i < io.SB; ++i) {
            const long k = j * kChunk + (long)s * io.SB + i;
            if (k >= k1) break;
            const float *uk = row + (i + 1) * m;
            if (k == 0)
                load_x0<NP>(A, b, x);
            else
                input_step<NP, MM>(A, sm + Lm.ad, sm + Lm.g0, sm + Lm.g1, row + i * m, uk, x);
#pragma unroll 4
            for (int r = 0; r < p; ++r) {
                float acc = 0.f;
                if constexpr (NP % 4 == 0) {
#pragma unroll
                    for (int c = 0; c < NP; c += 4) {
                        const float4 cv = lds4(sC + r * NP + c);
                        acc = fmaf(cv.x, x[c], fmaf(cv.y, x[c + 1], fmaf(cv.z, x[c + 2], fmaf(cv.w, x[c + 3], acc))));
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < NP; ++c) acc = fmaf(sC[r * NP + c], x[c], acc);
                }
#pragma unroll 4
                for (int q = 0; q < m; ++q) acc = fmaf(sD[r * m + q], uk[q], acc);
                yrow[i * p + r] = acc;
            }
            if (A.x) {
                float *xk = A.x + (b * A.T + k) * A.n;
#pragma unroll
                for (int c = 0; c < NP; ++c)
                    if (c < A.n) xk[c] = x[c];
            }
        }
        __syncthreads();
        store_y(A, p, io, tab, sy, s);
    }
}

#ifndef PRN_LSIM_IO_FLOATS
#define PRN_LSIM_IO_FLOATS 64
#endif
// Sub-block length: the largest of 8, 4, 2, 1 steps whose staged rows (two input
// buffers, one output buffer) fit PRN_LSIM_IO_FLOATS floats per chunk.
IoPlan io_plan(int m, int p) {
    IoPlan io{1, 0, 0};
    for (int sb = 8; sb >= 1; sb >>= 1) {
        io.SB = sb;
        io.ustr = ((sb + 1) * m) | 1;
        io.ystr = (sb * p) | 1;
        if (2 * io.ustr + io.ystr <= PRN_LSIM_IO_FLOATS) break;
    }
    return io;
}

int pad_state(int n) {
    int np = 1;
    while (np < n) np <<= 1;
    return np;
}

// Element counts per level: T_0 = T, T_{l+1} = ceil(T_l / 32), until a level fits one
// chunk; returns the number of upper levels (each with its chunk power).
int level_sizes(long T, long *Tl) {
    int L = 0;
    Tl[0] = T;
    while (Tl[L] > kChunk) {
        Tl[L + 1] = (Tl[L] + kChunk - 1) / kChunk;
        ++L;
    }
    return L;
}

template <int NP>
cudaError_t launch_np(const LsimReq &r, float *scratch, cudaStream_t st, int *launches) {
    long Tl[16];
    const int L = level_sizes(r.T, Tl);
    const MatLayout Lm(NP, r.m, r.p, L);
    float *mats = scratch;
    // level l >= 1 elements at agg[l]: B x Tl[l] x NP floats
    float *agg[16];
    long off = Lm.total;
    for (int l = 1; l <= L; ++l) {
        agg[l] = scratch + off;
        off = up4(off + r.batch * Tl[l] * NP);
    }
    const int q = r.n + r.m * (r.interp ? 2 : 1);
    const size_t dsmem = 3 * (size_t)q * q * sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(lsim_discretize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)dsmem);
    if (e != cudaSuccess) return e;
    lsim_discretize_kernel<<<1, kDiscThreads, dsmem, st>>>(r.A, r.Bm, r.C, r.D, r.n, r.m, r.p, r.h, r.interp, NP, L,
                                                           mats);
    int nl = 1;
    LsimArgs A;
    A.B = r.batch;
    A.n = r.n;
    A.m = r.m;
    A.p = r.p;
    A.interp = r.interp;
    A.U = r.U;
    A.x0 = r.x0;
    A.y = r.y;
    A.x = r.x;
    A.mats = mats;
    A.carry = nullptr;
    auto grid = [&](long T, int nt) { return (unsigned)((r.batch * ((T + kChunk - 1) / kChunk) + nt - 1) / nt); };
    const IoPlan io = io_plan(r.m, r.p);
    const size_t sm_in =
        (size_t)((use_chunk_kernels(NP, r.m) ? Lm.pw : Lm.c) + 2 * kThreadsL * io.ustr) * sizeof(float);
    const size_t sm_out = (size_t)(Lm.pw + kThreadsL * (2 * io.ustr + io.ystr)) * sizeof(float);
    // m = p in {1, 2, 4}: input and output widths as constants; otherwise run-time widths
    const int w = r.m == r.p && (r.m == 1 || r.m == 2 || r.m == 4) ? r.m : 0;
    const void *k_local0 = w == 1   ? (const void *)&lsim_local0_kernel<NP, 1>
                           : w == 2 ? (const void *)&lsim_local0_kernel<NP, 2>
                           : w == 4 ? (const void *)&lsim_local0_kernel<NP, 4>
                                    : (const void *)&lsim_local0_kernel<NP, 0>;
    const void *k_out = w == 1   ? (const void *)&lsim_out_kernel<NP, 1, 1>
                        : w == 2 ? (const void *)&lsim_out_kernel<NP, 2, 2>
                        : w == 4 ? (const void *)&lsim_out_kernel<NP, 4, 4>
                                 : (const void *)&lsim_out_kernel<NP, 0, 0>;
    if ((e = cudaFuncSetAttribute(k_local0, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_in)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(k_out, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_out)) != cudaSuccess)
        return e;
    IoPlan io_arg = io;
    void *io_args[] = {&A, &io_arg};
    const size_t sm_lv = (size_t)Lm.ps * sizeof(float);
    if (L > 0) {
        A.T = r.T;
        A.agg_out = agg[1];
        if ((e = cudaLaunchKernel(k_local0, dim3(grid(r.T, kThreadsL)), dim3(kThreadsL), io_args, sm_in, st)) !=
            cudaSuccess)
            return e;
        ++nl;
        for (int l = 1; l < L; ++l) {
            A.T = Tl[l];
            A.agg_in = agg[l];
            A.agg_out = agg[l + 1];
            A.mat_pw = Lm.pw + (l - 1) * Lm.ps;
            lsim_level_kernel<NP, false><<<grid(Tl[l], kThreadsLv), kThreadsLv, sm_lv, st>>>(A);
            ++nl;
        }
        for (int l = L; l >= 1; --l) {
            A.T = Tl[l];
            A.agg_in = agg[l];
            A.agg_out = nullptr;
            A.carry = l < L ? agg[l + 1] : nullptr;
            A.mat_pw = Lm.pw + (l - 1) * Lm.ps;
            lsim_level_kernel<NP, true><<<grid(Tl[l], kThreadsLv), kThreadsLv, sm_lv, st>>>(A);
            ++nl;
        }
        A.carry = agg[1];
    }
    A.T = r.T;
    if ((e = cudaLaunchKernel(k_out, dim3(grid(r.T, kThreadsL)), dim3(kThreadsL), io_args, sm_out, st)) != cudaSuccess)
        return e;
    *launches = nl + 1;
    return cudaGetLastError();
}

}  // namespace

int lsim_check(const LsimReq &r) {
    if (r.n < 1 || r.n > kLsimMaxN || r.m < 1 || r.m > kLsimMaxM || r.p < 1 || r.p > kLsimMaxP) return 1;
    if (r.batch < 1 || r.T < 1 || !(r.h > 0.0) || !(r.h < 1e300) || (r.interp != 0 && r.interp != 1)) return 1;
    return 0;
}

size_t lsim_scratch_bytes(const LsimReq &r) {
    long Tl[16];
    const int L = level_sizes(r.T, Tl);
    const int NP = pad_state(r.n);
    long off = MatLayout(NP, r.m, r.p, L).total;
    for (int l = 1; l <= L; ++l) off = up4(off + r.batch * Tl[l] * NP);
    return (size_t)off * sizeof(float);
}

cudaError_t lsim_launch(const LsimReq &r, float *scratch, cudaStream_t st, int *launches) {
    switch (pad_state(r.n)) {
        case 1: return launch_np<1>(r, scratch, st, launches);
        case 2: return launch_np<2>(r, scratch, st, launches);
        case 4: return launch_np<4>(r, scratch, st, launches);
        case 8: return launch_np<8>(r, scratch, st, launches);
        case 16: return launch_np<16>(r, scratch, st, launches);
        default: return launch_np<32>(r, scratch, st, launches);
    }
}

}  // namespace prn
