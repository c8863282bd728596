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
// only: a thread runs 32 consecutive steps from a zero state and emits the chunk's end
// state; those end states form a sequence of the same kind with matrix Ad^32, chunked
// again until one chunk covers a level; a fix-up pass turns every level's end states
// into the states entering the next chunk, top down; the last pass re-runs each
// 32-step chunk from its entering state and writes y (and x).  Every pass is
// independent per thread: no CTA waits on another.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace prn {

namespace {

constexpr int kChunk = 32;     // steps per thread, every level
constexpr int kThreadsL = 128;  // threads per CTA of the chunk passes
constexpr int kDiscThreads = 1024;
constexpr int kTaylor = 14;  // degree; the scaled matrix has 1-norm <= 1/2

__host__ __device__ constexpr long up4(long x) { return (x + 3) & ~3L; }

// Offsets (floats) of the fp32 matrices the discretisation writes, padded to NP:
// AdT [NP][NP] (AdT[j][i] = Ad[i][j]), G0T, G1T [m][NP], Cp [p][NP], Dm [p][m], then
// the transposed chunk powers Ad^(32^l), l = 1 .. levels, [NP][NP] each at a stride of
// ps floats.  Every offset is a multiple of 4 floats (16-byte copies).
struct MatLayout {
    long ad, g0, g1, c, d, pw, ps, total;
    __host__ __device__ MatLayout(int NP, int m, int p, int levels) {
        ps = up4((long)NP * NP);
        ad = 0;
        g0 = up4(ad + (long)NP * NP);
        g1 = up4(g0 + (long)m * NP);
        c = up4(g1 + (long)m * NP);
        d = up4(c + (long)p * NP);
        pw = up4(d + (long)p * m);
        total = pw + levels * ps;
    }
};

// ------------------------------------------------------------------ discretisation (fp64)
// Product of q x q row-major matrices in shared memory, by the whole CTA.
__device__ void smem_matmul(const double *X, const double *Y, double *Z, int q) {
    for (int idx = threadIdx.x; idx < q * q; idx += blockDim.x) {
        const int i = idx / q, j = idx % q;
        double acc = 0.0;
        for (int k = 0; k < q; ++k) acc = fma(X[i * q + k], Y[k * q + j], acc);
        Z[idx] = acc;
    }
    __syncthreads();
}

// One CTA: e^M for M = [[A h, B h, 0], [0, 0, I], [0, 0, 0]] (the last block row and
// column only with the linear hold), by scaling M to 1-norm <= 1/2, a degree-14
// Taylor polynomial in Horner form (truncation below 1e-21 relative), and squaring
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
        while (!(nrm * scale <= 0.5) && s < 1100) {  // NaN stops at the bound
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

// One step of the input level: x <- Ad x + G0 u_{k-1} + G1 u_k (x <- x0 at k = 0).
template <int NP>
__device__ __forceinline__ void input_step(const LsimArgs &A, const float *sAd, const float *sG0, const float *sG1,
                                           long b, long k, float (&x)[NP]) {
    if (k == 0) {
#pragma unroll
        for (int i = 0; i < NP; ++i) x[i] = (A.x0 && i < A.n) ? A.x0[b * A.n + i] : 0.f;
        return;
    }
    float y[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) y[i] = 0.f;
    mv_acc<NP>(sAd, x, y);
    const float *uk = A.U + (b * A.T + k) * A.m;
    for (int q = 0; q < A.m; ++q) {
        const float u0 = __ldg(uk - A.m + q);
#pragma unroll
        for (int i = 0; i < NP; ++i) y[i] = fmaf(sG0[q * NP + i], u0, y[i]);
        if (A.interp) {
            const float u1 = __ldg(uk + q);
#pragma unroll
            for (int i = 0; i < NP; ++i) y[i] = fmaf(sG1[q * NP + i], u1, y[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = y[i];
}

// Input level, first pass: each thread's chunk from a zero state (chunk 0 from x0);
// writes the chunk's end state.
template <int NP>
__global__ void __launch_bounds__(kThreadsL) lsim_local0_kernel(const LsimArgs A) {
    extern __shared__ __align__(16) float sm[];
    const MatLayout Lm(NP, A.m, A.p, 0);
    stage_mats(sm, A.mats, Lm.c);
    const long nch = (A.T + kChunk - 1) / kChunk;
    const long g = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= A.B * nch) return;
    const long b = g / nch, j = g % nch;
    float x[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = 0.f;
    const long k1 = min(A.T, (j + 1) * kChunk);
    for (long k = j * kChunk; k < k1; ++k) input_step<NP>(A, sm + Lm.ad, sm + Lm.g0, sm + Lm.g1, b, k, x);
    float4 *o = reinterpret_cast<float4 *>(A.agg_out + g * NP);
    if constexpr (NP % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NP; i += 4) o[i / 4] = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
    } else {
#pragma unroll
        for (int i = 0; i < NP; ++i) A.agg_out[g * NP + i] = x[i];
    }
}

// Upper levels: elements e_k (NP floats each) with matrix P = Ad^(32^l):
//   local (FIX false): end state of each chunk of 32 elements from a zero state;
//   fix (FIX true):    states c_k = P c_{k-1} + e_k from the entering state (the
//                      inclusive end state of the previous chunk, one level up),
//                      written over e_k.
template <int NP, bool FIX>
__global__ void __launch_bounds__(kThreadsL) lsim_level_kernel(const LsimArgs A) {
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
    for (long k = j * kChunk; k < k1; ++k) {
        float *e = A.agg_in + (b * A.T + k) * NP;
        float y[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) y[i] = e[i];
        mv_acc<NP>(sm, x, y);
#pragma unroll
        for (int i = 0; i < NP; ++i) x[i] = y[i];
        if (FIX) {
#pragma unroll
            for (int i = 0; i < NP; ++i) e[i] = x[i];
        }
    }
    if (!FIX) {
#pragma unroll
        for (int i = 0; i < NP; ++i) A.agg_out[g * NP + i] = x[i];
    }
}

// Input level, last pass: each chunk from its entering state; writes y and x.
template <int NP>
__global__ void __launch_bounds__(kThreadsL) lsim_out_kernel(const LsimArgs A) {
    extern __shared__ __align__(16) float sm[];
    const MatLayout Lm(NP, A.m, A.p, 0);
    stage_mats(sm, A.mats, Lm.pw);
    const long nch = (A.T + kChunk - 1) / kChunk;
    const long g = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= A.B * nch) return;
    const long b = g / nch, j = g % nch;
    float x[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) x[i] = (j > 0 && A.carry) ? A.carry[(g - 1) * NP + i] : 0.f;
    const long k1 = min(A.T, (j + 1) * kChunk);
    const float *sC = sm + Lm.c, *sD = sm + Lm.d;
    for (long k = j * kChunk; k < k1; ++k) {
        input_step<NP>(A, sm + Lm.ad, sm + Lm.g0, sm + Lm.g1, b, k, x);
        const float *uk = A.U + (b * A.T + k) * A.m;
        float *yk = A.y + (b * A.T + k) * A.p;
        for (int r = 0; r < A.p; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < NP; ++i) acc = fmaf(sC[r * NP + i], x[i], acc);
            for (int q = 0; q < A.m; ++q) acc = fmaf(sD[r * A.m + q], __ldg(uk + q), acc);
            yk[r] = acc;
        }
        if (A.x) {
            float *xk = A.x + (b * A.T + k) * A.n;
#pragma unroll
            for (int i = 0; i < NP; ++i)
                if (i < A.n) xk[i] = x[i];
        }
    }
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
    auto grid = [&](long T) { return (unsigned)((r.batch * ((T + kChunk - 1) / kChunk) + kThreadsL - 1) / kThreadsL); };
    const size_t sm_in = (size_t)Lm.c * sizeof(float), sm_out = (size_t)Lm.pw * sizeof(float);
    const size_t sm_lv = (size_t)Lm.ps * sizeof(float);
    if (L > 0) {
        A.T = r.T;
        A.agg_out = agg[1];
        lsim_local0_kernel<NP><<<grid(r.T), kThreadsL, sm_in, st>>>(A);
        ++nl;
        for (int l = 1; l < L; ++l) {
            A.T = Tl[l];
            A.agg_in = agg[l];
            A.agg_out = agg[l + 1];
            A.mat_pw = Lm.pw + (l - 1) * Lm.ps;
            lsim_level_kernel<NP, false><<<grid(Tl[l]), kThreadsL, sm_lv, st>>>(A);
            ++nl;
        }
        for (int l = L; l >= 1; --l) {
            A.T = Tl[l];
            A.agg_in = agg[l];
            A.agg_out = nullptr;
            A.carry = l < L ? agg[l + 1] : nullptr;
            A.mat_pw = Lm.pw + (l - 1) * Lm.ps;
            lsim_level_kernel<NP, true><<<grid(Tl[l]), kThreadsL, sm_lv, st>>>(A);
            ++nl;
        }
        A.carry = agg[1];
    }
    A.T = r.T;
    lsim_out_kernel<NP><<<grid(r.T), kThreadsL, sm_out, st>>>(A);
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
