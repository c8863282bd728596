// deer_tc.cu -- full DEER for the tanh RNN at 32 < n <= 64 with the products of the dense
// Jacobians on the tensor cores (tcgen05, kind::tf32, fp32 accuracy from three TF32
// products).
//
// "Parallelizing non-linear sequential models over the sequence length", Approach and
// Surprising findings / Limitations: each Newton iteration solves the linear recurrence
// delta_t = J_t delta_{t-1} + r_t with dense J_t = diag(1 - f_t^2) A, and composing the
// Jacobians costs O(n^3) per step.  "Para-Seq" README, Main features: the vanilla tanh
// RNN with DEER modes.
//
// Tiles of 128 steps of one sequence; one CTA per SM (8 warps, all 512 TMEM columns).
// Per tile and iteration:
//  1. Cell: U = H A^T for the tile as one 128 x 64 x 64 product (H = h^(k)_{t-1} by
//     rows, written to TMEM as the A operand); f = tanh(U + p), d = 1 - f^2 and
//     r = f - h^(k)_t go to shared memory.
//  2. Chain maps: the tile is four chains of 32 steps.  Walking a chain backward,
//     Q <- Q diag(d_t) A and D <- D + Q r_t (Q = J_end ... J_{t+1}) end with the chain's
//     map delta_end = P delta_before + D.  Warpgroup g runs chains 2g and 2g + 1 as the
//     two 64-row halves of one M = 128 product with its own TMEM columns and mbarrier,
//     so one group's products run while the other handles its result.  A step: each
//     thread loads its row of Q from the accumulator, adds to D, scales the columns by
//     d_t, splits the row into TF32 hi and lo parts and stores both back to TMEM as the
//     next product's A operand; one thread issues lo*hi + hi*lo + hi*hi against the hi
//     and lo parts of A, resident in shared memory (K-major, 128-byte swizzle).
//  3. Carry: the predecessor tile's published delta through the four chain maps; the
//     tile publishes its last delta (epoch-tagged words, an inclusive chain).
//  4. Re-walk: delta_t = d_t (A delta_{t-1}) + r_t from every chain's start, two warps
//     per chain with the thread's row of A in registers, delta_t in place of r_t; then
//     h^(k+1) = h^(k) + delta over the tile with coalesced accesses.
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "staged_tiles.cuh"

namespace prn {
namespace {

constexpr int kN = 64;                    // padded state size
constexpr int kT = 128;                   // steps per tile
constexpr int kChain = 32;                // steps per chain
constexpr int kChains = kT / kChain;      // chains per tile; warps 2c, 2c + 1 own chain c
static_assert(kChain % 2 == 0, "a group waits an even number of times per tile: parities return");
static_assert(kChains * 64 == kThreads, "one thread per row of every chain");

// TMEM columns: group g owns 256 g .. 256 g + 255: two accumulators (the product's K
// halves, so that consecutive MMAs alternate between independent accumulations) and its
// A operand (hi, lo); the cell product uses group 0's.
constexpr int kTmemCols = 512;
__host__ __device__ constexpr int col_acc(int g) { return 256 * g; }  // + 64: second accumulator
__host__ __device__ constexpr int col_ahi(int g) { return 256 * g + 128; }
__host__ __device__ constexpr int col_alo(int g) { return 256 * g + 192; }

// Shared memory, byte offsets from a 1024-byte aligned base.  B operands are K-major
// with the 128-byte swizzle: a row holds 32 K elements (128 bytes) per K block, its
// 16-byte chunk j sits at chunk j ^ (row % 8), 8-row groups are 1024 bytes apart.  Each
// B operand has 128 rows: rows 0..63 the TF32 hi parts, rows 64..127 the lo parts, so
// that one N = 128 product gives A_hi B_hi and A_hi B_lo side by side.
constexpr int kOffB = 0;          // A^T (row j: A[.][j]): B operand of the chain products
constexpr int kOffC = 32768;      // A (row i: A[i][.]): B operand of the cell product
constexpr int kOffD = 65536;      // d [128 steps][64 units], 16-byte chunks swizzled by step
constexpr int kOffR = 98304;      // r, then delta; same layout
constexpr int kOffH = 131072;     // h^(k) of a tile's 128 steps, two buffers of two 128 x 32 boxes
                                  // (TMA layout, 128-byte swizzle: chunk j of row m at j ^ (m % 8))
constexpr int kOffA = 196608;     // A in fp32, row i's 16-byte chunk c at c ^ (i % 16)
constexpr int kOffDl = 212992;    // delta before each chain and after the tile: 5 x 64 floats
constexpr int kOffH0 = 214272;    // the state before the tile's first step, one row per buffer
constexpr int kOffW = 214784;     // W^T [8][64] and the bias [64] (raw inputs)
constexpr int kOffMisc = 217088;  // 4 mbarriers, TMEM base, failure flag, block-max scratch
constexpr int kSmem = kOffMisc + 128 + 1024;  // + slack for the 1024-byte alignment
constexpr int kKb = 16384;        // bytes between the two 32-wide K blocks of a B operand
// Instruction descriptors: D fp32, A and B tf32, both K-major, M = 128, N = 128 or 64.
__host__ __device__ constexpr unsigned idesc_n(int n) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((unsigned)(n >> 3) << 17) | ((unsigned)(128 >> 4) << 24);
}

struct DeerTcArgs {
    int B, T, n, in;
    const float *xproj, *x, *W, *bias, *A, *h0;
    float *h;
    int max_iters;
    float tol;
    int *iters_out;
    float *delta_out, *residual_out;
    Ctl *ctl;
    int *sticky;
    unsigned long long *inc;
    float *side;
    unsigned epoch0;
    Dbg dbg;
};

// Byte offset of 16-byte chunk c (0..15 along K) of `row` (0..127) in a B operand.
__device__ __forceinline__ unsigned opnd_off(int row, int c) {
    return (unsigned)((c >> 3) * kKb + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}
// Float offset of (step t, unit i) in the d and r arrays.
__device__ __forceinline__ int dr_off(int t, int i) { return t * kN + (((i >> 2) ^ (t & 15)) << 2) + (i & 3); }

__device__ __forceinline__ void st_shared_v4(unsigned addr, float a, float b, float c, float d) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
// TF32 part of x rounded to nearest (10 explicit mantissa bits); x - hi is exact in fp32.
__device__ __forceinline__ float tf32_hi(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}

__device__ __forceinline__ void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ unsigned long long sw128_desc(unsigned addr) {
    return (unsigned long long)((addr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// D += A x B: A from TMEM (row m in lane m, K element k in column a + AOFF + k), B in
// shared memory (descriptor b advanced by BOFF 16-byte units).  The offsets are added
// inside the instruction block, so the compiler keeps two bases, not 16 addresses.
template <int NN, int AOFF, int BOFF>
__device__ __forceinline__ void mma_tf32_at(unsigned d, unsigned a, unsigned long long b, unsigned accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b32 ra;\n\t.reg .b64 rb;\n\t"
        "add.u32 ra, %1, %5;\n\t"
        "add.u64 rb, %2, %6;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [ra], rb, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(b), "n"(idesc_n(NN)), "r"(accum), "n"(AOFF), "n"(BOFF)
        : "memory");
}
// K steps S .. E - 1 (8 elements each): A_hi x [B_hi | B_lo] (N = 128) into columns
// d .. d + 127, then A_lo x B_hi (N = 64) into d .. d + 63.  Over K = 64 (S = 0, E = 8)
// the sum of columns d .. d + 63 and d + 64 .. d + 127 is A_lo B_hi + A_hi B_lo + A_hi B_hi.
template <int S, int E>
__device__ __forceinline__ void mma_seq(unsigned d, unsigned a_hi, unsigned a_lo, unsigned long long b) {
    if constexpr (S < E) {
        constexpr int BOFF = ((S >> 2) * kKb + (S & 3) * 32) >> 4;
        mma_tf32_at<128, 8 * S, BOFF>(d, a_hi, b, S > 0 ? 1u : 0u);
        mma_tf32_at<64, 8 * S, BOFF>(d, a_lo, b, 1u);
        mma_seq<S + 1, E>(d, a_hi, a_lo, b);
    }
}
__device__ __forceinline__ void mma_commit(unsigned long long *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
// The whole product (K = 64); `bar` is signalled when it is complete.
__device__ __forceinline__ void mma_3xtf32(unsigned d, unsigned a_hi, unsigned a_lo, unsigned b,
                                           unsigned long long *bar) {
    mma_seq<0, 8>(d, a_hi, a_lo, sw128_desc(b));
    mma_commit(bar);
}

// 16 consecutive TMEM columns of this thread's lane; complete after tcgen05.wait::st.
__device__ __forceinline__ void tmem_st16(unsigned taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])));
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }



// Columns c .. c + 15 of both accumulator halves (one wait for the two loads).
__device__ __forceinline__ void tmem_ld16x2(unsigned taddr, float (&a)[16], float (&b)[16]) {
    unsigned r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31}, [%33];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr), "r"(taddr + 64)
        : "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        a[j] = __uint_as_float(r[j]);
        b[j] = __uint_as_float(r[16 + j]);
    }
}
// The product's row for this thread: the sum of the two accumulator halves.
__device__ __forceinline__ void load_acc(unsigned taddr, float (&q)[64]) {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        float a[16], b[16];
        tmem_ld16x2(taddr + 16 * h, a, b);
#pragma unroll
        for (int j = 0; j < 16; ++j) q[16 * h + j] = a[j] + b[j];
    }
}

// Bounded wait for this CTA's own products.  It does not give up on the abort flag (the
// products finish within microseconds whatever other CTAs do); after a timeout, `bad`
// stays set and later waits return at once.
__device__ __forceinline__ bool mma_wait(unsigned long long *bar, unsigned parity, const DeerTcArgs &A,
                                         volatile int *s_fail, bool &bad) {
    if (bad) return false;
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (!mbar_try(bar, parity)) {
        if (gtimer() - t0 > A.dbg.wait_ns) {
            bad = true;
            *s_fail = 1;
            raise_status(A.sticky, A.ctl, kStTimeout, true);
            return false;
        }
    }
    return true;
}

// Bounded wait for an epoch-tagged word; false on a timeout (status raised) or an abort.
__device__ __forceinline__ bool wait_tagged(const unsigned long long *p, unsigned epoch, float *v,
                                            const DeerTcArgs &A) {
    unsigned long long t0 = 0;
    for (int polls = 0;; ++polls) {
        const unsigned long long w = ld_relaxed_u64(p);
        if ((unsigned)w == epoch) {
            *v = __uint_as_float((unsigned)(w >> 32));
            return true;
        }
        if (ld_relaxed_int(&A.ctl->abort)) return false;
        if (polls == 4) t0 = gtimer();
        if (polls > 4) {
            if (gtimer() - t0 > A.dbg.wait_ns) {
                raise_status(A.sticky, A.ctl, kStTimeout, true);
                return false;
            }
            __nanosleep(32);
        }
    }
}

struct TileCtx {
    unsigned char *base;  // 1024-byte aligned dynamic shared memory
    unsigned sbase, tmem;
    unsigned long long *bars;  // [0], [1]: the groups' products; [2], [3]: the staging buffers
    volatile int *s_fail;
    const CUtensorMap *hmap;   // h as [B*T rows][n] (null: staged with plain loads)
    unsigned ph0, ph1;         // next parity of each group's barrier
    unsigned hph;              // bit b: next parity of staging buffer b's barrier
    int hbuf;                  // staging buffer of the current tile
    bool bad;
};

// Float offset of (row m, unit i) in staging buffer `buf`.
__device__ __forceinline__ int hst_off(int buf, int m, int i) {
    return (kOffH >> 2) + buf * 8192 + (i >> 5) * 4096 + m * 32 + ((((i & 31) >> 2) ^ (m & 7)) << 2) + (i & 3);
}

// Stage h^(k) of the tile at rows y .. y + 127 of [B*T][n] into buffer `buf`: two TMA
// boxes (units 0..31, 32..63; columns at or past n and rows past B*T read as zero).
__device__ __forceinline__ void issue_h(TileCtx &X, int buf, int y) {
    unsigned long long *bar = X.bars + 2 + buf;
    mbar_expect_tx(bar, 32768);
    tma_load_2d(X.base + kOffH + buf * 32768, X.hmap, 0, y, bar);
    tma_load_2d(X.base + kOffH + buf * 32768 + 16384, X.hmap, 32, y, bar);
}
// The same with plain loads (n % 4 != 0): consecutive threads read consecutive units.
__device__ __forceinline__ void stage_h_plain(const DeerTcArgs &A, TileCtx &X, int buf, int b, int t0) {
    float *sm = reinterpret_cast<float *>(X.base);
    const size_t row0 = (size_t)b * A.T + t0;
    for (int e = threadIdx.x; e < kT * kN; e += kThreads) {
        const int m = e >> 6, i = e & 63;
        sm[hst_off(buf, m, i)] = (i < A.n && t0 + m < A.T) ? A.h[(row0 + m) * A.n + i] : 0.f;
    }
}

// Phase 1 over the tile's steps t0 .. t0 + steps - 1: U = H A^T on the tensor cores,
// then f, d and r.  Writes d and r (zero outside the sequence and the state) unless
// residual_only; returns max |r|.  Thread (warp w, lane l) owns step row
// 32 (w % 4) + l and units 32 (w / 4) .. + 31 throughout.  h^(k) of the tile's steps
// is in staging buffer X.hbuf (when have_h); the state before the tile is loaded here.
__device__ __forceinline__ float cell_phase(const DeerTcArgs &A, TileCtx &X, int b, int t0, int steps, bool have_h,
                                            const float *prev_side, bool residual_only) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = A.n, buf = X.hbuf;
    const size_t seq0 = (size_t)b * A.T;
    const int tr = 32 * (warp & 3) + lane, i0 = 32 * (warp >> 2), t = t0 + tr;
    const bool tv = tr < steps;
    const unsigned lane_off = (unsigned)(32 * (warp & 3)) << 16;
    float *smf = reinterpret_cast<float *>(X.base);
    float *hprev = smf + (kOffH0 >> 2) + buf * 64;
    if (tid < kN) {
        // the state before step t0: h0 before the sequence, the side value for the
        // preceding tile's last step, zeros on the first iteration
        float v = 0.f;
        if (tid < n) {
            if (t0 == 0)
                v = A.h0 ? A.h0[(size_t)b * n + tid] : 0.f;
            else if (have_h)
                v = prev_side ? prev_side[tid] : A.h[(seq0 + t0 - 1) * n + tid];
        }
        hprev[tid] = v;
    }
    if (have_h) {
        if (X.hmap) {
            const unsigned par = (X.hph >> buf) & 1u;
            const unsigned long long t_start = gtimer();
            while (!mbar_try(X.bars + 2 + buf, par)) {
                if (gtimer() - t_start > A.dbg.wait_ns) {
                    *X.s_fail = 1;
                    raise_status(A.sticky, A.ctl, kStTimeout, true);
                    break;
                }
            }
            X.hph ^= 1u << buf;
        } else {
            stage_h_plain(A, X, buf, b, t0);
        }
    }
    __syncthreads();
    {
        // row tr of H: the state before step t
        float hv[32];
        if (tr == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 v = *reinterpret_cast<const float4 *>(hprev + i0 + j);
                hv[j] = v.x, hv[j + 1] = v.y, hv[j + 2] = v.z, hv[j + 3] = v.w;
            }
        } else if (have_h) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 v = *reinterpret_cast<const float4 *>(smf + hst_off(buf, tr - 1, i0 + j));
                hv[j] = v.x, hv[j + 1] = v.y, hv[j + 2] = v.z, hv[j + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) hv[j] = 0.f;
        }
        float hi[16], lo[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                hi[j] = tf32_hi(hv[16 * half + j]);
                lo[j] = hv[16 * half + j] - hi[j];
            }
            tmem_st16(X.tmem + lane_off + (unsigned)(col_ahi(0) + i0 + 16 * half), hi);
            tmem_st16(X.tmem + lane_off + (unsigned)(col_alo(0) + i0 + 16 * half), lo);
        }
        tmem_st_wait();
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        mma_3xtf32(X.tmem + col_acc(0), X.tmem + col_ahi(0), X.tmem + col_alo(0), X.sbase + kOffC, X.bars);
    }
    // while the product runs: the inputs of this thread's steps and units
    float pv[32];
    if (A.xproj) {
        const float *xrow = A.xproj + (seq0 + t) * n;
#pragma unroll
        for (int j = 0; j < 32; ++j) pv[j] = (tv && i0 + j < n) ? xrow[i0 + j] : 0.f;
    } else {
        float xv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) xv[q] = (q < A.in && tv) ? A.x[(seq0 + t) * A.in + q] : 0.f;
        const float *sw = smf + (kOffW >> 2), *sb = sw + 8 * kN;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float p = sb[i0 + j];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < A.in) p = fmaf(sw[k * kN + i0 + j], xv[k], p);
            pv[j] = p;
        }
    }
    mma_wait(X.bars, X.ph0, A, X.s_fail, X.bad);
    X.ph0 ^= 1u;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    float *dsm = smf + (kOffD >> 2), *rsm = smf + (kOffR >> 2);
    float res = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float u[16], u2[16];
        tmem_ld16x2(X.tmem + lane_off + (unsigned)(col_acc(0) + i0 + 16 * h), u, u2);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float dv[4], rv[4];
            float4 hk = make_float4(0.f, 0.f, 0.f, 0.f);
            if (have_h) hk = *reinterpret_cast<const float4 *>(smf + hst_off(buf, tr, i0 + 16 * h + 4 * c));
            const float hkv[4] = {hk.x, hk.y, hk.z, hk.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = 16 * h + 4 * c + q;
                const bool v = tv && i0 + j < n;
                const float f = tanh_(u[4 * c + q] + u2[4 * c + q] + pv[j]);
                dv[q] = v ? 1.f - f * f : 0.f;
                rv[q] = v ? f - hkv[q] : 0.f;
                const float ad = fabsf(rv[q]);
                res = (ad > res || isnan(ad)) ? ad : res;
            }
            if (!residual_only) {
                const int o = dr_off(tr, i0 + 16 * h + 4 * c);
                *reinterpret_cast<float4 *>(dsm + o) = make_float4(dv[0], dv[1], dv[2], dv[3]);
                *reinterpret_cast<float4 *>(rsm + o) = make_float4(rv[0], rv[1], rv[2], rv[3]);
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    return res;
}

// Phase 2 for this thread's row of its chain: returns the row of P in q and of D in *D.
__device__ __forceinline__ void chain_phase(const DeerTcArgs &A, TileCtx &X, int steps, float (&q)[64], float *Dout) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = warp >> 2, wq = warp & 3;
    const int cc = warp >> 1, i = (32 * wq + lane) & 63;
    const int tc0 = kChain * cc, tend = min(tc0 + kChain, steps);
    const unsigned lane_off = (unsigned)(32 * wq) << 16;
    const unsigned t_acc = X.tmem + lane_off + (unsigned)col_acc(g);
    const unsigned t_ahi = X.tmem + lane_off + (unsigned)col_ahi(g), t_alo = X.tmem + lane_off + (unsigned)col_alo(g);
    unsigned long long *bar = X.bars + g;
    unsigned ph = g ? X.ph1 : X.ph0;
    const float *dsm = reinterpret_cast<const float *>(X.base + kOffD);
    const float *rsm = reinterpret_cast<const float *>(X.base + kOffR);
    float D4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int s = 0; s < kChain; ++s) {
        const int t = tc0 + kChain - 1 - s;
        if (s > 0) {
            mma_wait(bar, ph, A, X.s_fail, X.bad);
            ph ^= 1u;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        }
        if (t + 1 >= tend) {  // no valid Jacobian after t in this chain: Q = I
#pragma unroll
            for (int j = 0; j < 64; ++j) q[j] = j == i ? 1.f : 0.f;
        } else {
            load_acc(t_acc, q);
        }
        const float *drow = dsm + t * kN, *rrow = rsm + t * kN;
        const int sw = t & 15;
        const unsigned long long bdesc = sw128_desc(X.sbase + kOffB);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            // columns 32 half .. + 31 of Q diag(d_t), then the products over those K
            // elements start while the other half is prepared
#pragma unroll
            for (int bq = 2 * half; bq < 2 * half + 2; ++bq) {
                float hi[16], lo[16];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int c = 4 * bq + c4;
                    const float4 dd = *reinterpret_cast<const float4 *>(drow + ((c ^ sw) << 2));
                    const float4 rr = *reinterpret_cast<const float4 *>(rrow + ((c ^ sw) << 2));
                    D4[0] = fmaf(q[4 * c], rr.x, D4[0]);
                    D4[1] = fmaf(q[4 * c + 1], rr.y, D4[1]);
                    D4[2] = fmaf(q[4 * c + 2], rr.z, D4[2]);
                    D4[3] = fmaf(q[4 * c + 3], rr.w, D4[3]);
                    const float sv[4] = {q[4 * c] * dd.x, q[4 * c + 1] * dd.y, q[4 * c + 2] * dd.z,
                                         q[4 * c + 3] * dd.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        hi[4 * c4 + e] = tf32_hi(sv[e]);
                        lo[4 * c4 + e] = sv[e] - hi[4 * c4 + e];
                    }
                }
                tmem_st16(t_ahi + 16 * bq, hi);
                tmem_st16(t_alo + 16 * bq, lo);
            }
            tmem_st_wait();
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            named_sync(1 + g, 128);
            if (wq == 0 && lane == 0 && !X.bad) {
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const unsigned d = X.tmem + col_acc(g), ah = X.tmem + col_ahi(g), al = X.tmem + col_alo(g);
                if (half == 0) {
                    mma_seq<0, 4>(d, ah, al, bdesc);
                } else {
                    mma_seq<4, 8>(d, ah, al, bdesc);
                    mma_commit(bar);
                }
            }
        }
    }
    mma_wait(bar, ph, A, X.s_fail, X.bad);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (tc0 < steps) {
        load_acc(t_acc, q);
    } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) q[j] = j == i ? 1.f : 0.f;
    }
    *Dout = (D4[0] + D4[1]) + (D4[2] + D4[3]);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// The iterations and the residual pass; every return is taken by the whole CTA.
__device__ __forceinline__ void deer_tc_body(const DeerTcArgs &A, TileCtx &X, unsigned *s_red) {
    const int tid = threadIdx.x, warp = tid >> 5;
    const int n = A.n;
    const int nchunk = (A.T + kT - 1) / kT;
    const long nseq = A.B;
    const long ntiles = nseq * nchunk;
    const int cc = warp >> 1, ii = tid & 63;  // chain and row (unit) of this thread
    float *dl = reinterpret_cast<float *>(X.base + kOffDl);  // dl[c][64]: delta before chain c; [4]: after the tile
    float *rsm = reinterpret_cast<float *>(X.base + kOffR);
    const float *dsm = reinterpret_cast<const float *>(X.base + kOffD);
    int iters = 0;
    float last_delta = 0.f;
    bool stop_all = false;
    for (int k = 0; k < A.max_iters; ++k) {
        const unsigned epoch = A.epoch0 + (unsigned)k + 1u;
        if (blockIdx.x == 0 && tid == 0) A.ctl->delta_bits[(k + 1) % 3] = 0u;
        const float *side_in = A.side + (size_t)(k & 1) * ntiles * kN;
        float *side_out = A.side + (size_t)((k + 1) & 1) * ntiles * kN;
        float my_max = 0.f;
        TileWalk tw(nseq);
        const bool have_h = k > 0;
        if (have_h && X.hmap && tid == 0 && blockIdx.x < ntiles) {
            // the previous iteration's states, written through the generic proxy, are read by TMA
            asm volatile("fence.proxy.async.global;" ::: "memory");
            issue_h(X, X.hbuf, (int)((long)tw.seq * A.T + (long)tw.chunk * kT));
        }
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next(), X.hbuf ^= 1) {
            const int chunk = tw.chunk, b = tw.seq;
            const int t0 = chunk * kT, steps = min(kT, A.T - t0);
            __syncthreads();  // the previous tile is done with d, r, the delta vectors and its staging buffer
            if (have_h && X.hmap && tid == 0 && tile + gridDim.x < ntiles) {
                TileWalk nx = tw;
                nx.next();
                issue_h(X, X.hbuf ^ 1, (int)((long)nx.seq * A.T + (long)nx.chunk * kT));
            }
            cell_phase(A, X, b, t0, steps, have_h, (have_h && chunk > 0) ? side_in + (tile - nseq) * kN : nullptr,
                       false);
            if (*X.s_fail) return;
            float q[64], Dr;
            chain_phase(A, X, steps, q, &Dr);
            __syncthreads();  // every chain map is in registers
            if (tid < kN) {
                float cv = 0.f;
                if (chunk > 0 && !wait_tagged(A.inc + (tile - nseq) * kN + tid, epoch, &cv, A)) *X.s_fail = 1;
                dl[tid] = cv;
            }
            __syncthreads();
            if (*X.s_fail) return;
#pragma unroll 1
            for (int c = 0; c < kChains; ++c) {
                if (cc == c) {
                    const float *dp = dl + c * kN;
                    float a4[4] = {Dr, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float4 v = *reinterpret_cast<const float4 *>(dp + 4 * j);
                        a4[0] = fmaf(q[4 * j], v.x, a4[0]);
                        a4[1] = fmaf(q[4 * j + 1], v.y, a4[1]);
                        a4[2] = fmaf(q[4 * j + 2], v.z, a4[2]);
                        a4[3] = fmaf(q[4 * j + 3], v.w, a4[3]);
                    }
                    const float nd = (a4[0] + a4[1]) + (a4[2] + a4[3]);
                    dl[(c + 1) * kN + ii] = nd;
                    if (c == kChains - 1 && A.dbg.skip_tile != tile)
                        st_relaxed_u64(A.inc + tile * kN + ii, pack_tag(nd, epoch));
                }
                __syncthreads();
            }
            // re-walk of this thread's chain from the delta before it; delta_t replaces r_t
            {
                const int tc0 = kChain * cc, tend = min(tc0 + kChain, steps);
                float a[64];
                const float *arow = reinterpret_cast<const float *>(X.base + kOffA) + ii * kN;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float4 v = *reinterpret_cast<const float4 *>(arow + ((c ^ (ii & 15)) << 2));
                    a[4 * c] = v.x, a[4 * c + 1] = v.y, a[4 * c + 2] = v.z, a[4 * c + 3] = v.w;
                }
                const float *prow = dl + cc * kN;  // delta_{t-1}: plain for the chain's first step,
                int pkey = 0;                      // then the swizzled row t - 1
                for (int t = tc0; t < tend; ++t) {
                    float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float4 v = *reinterpret_cast<const float4 *>(prow + ((j ^ pkey) << 2));
                        a4[0] = fmaf(a[4 * j], v.x, a4[0]);
                        a4[1] = fmaf(a[4 * j + 1], v.y, a4[1]);
                        a4[2] = fmaf(a[4 * j + 2], v.z, a4[2]);
                        a4[3] = fmaf(a[4 * j + 3], v.w, a4[3]);
                    }
                    const int o = dr_off(t, ii);
                    rsm[o] = fmaf(dsm[o], (a4[0] + a4[1]) + (a4[2] + a4[3]), rsm[o]);
                    named_sync(3 + cc, 64);
                    prow = rsm + t * kN;
                    pkey = t & 15;
                }
            }
            __syncthreads();
            // h^(k+1) = h^(k) + delta over the tile, coalesced; the loads go out first
            {
                constexpr int PER = kT * kN / kThreads;
                const float *smf = reinterpret_cast<const float *>(X.base);
                float *hb = A.h + ((size_t)b * A.T + t0) * n;
#pragma unroll
                for (int j = 0; j < PER; ++j) {
                    const int e = tid + j * kThreads, t = e >> 6, i = e & 63;
                    if (t < steps && i < n) {
                        const float nd = rsm[dr_off(t, i)];
                        const float hn = (have_h ? smf[hst_off(X.hbuf, t, i)] : 0.f) + nd;
                        hb[(size_t)t * n + i] = hn;
                        const float ad = fabsf(nd);
                        my_max = (ad > my_max || isnan(nd)) ? ad : my_max;
                        if (t == kT - 1 && chunk < nchunk - 1) side_out[tile * kN + i] = hn;
                    }
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
        float my_res = 0.f;
        TileWalk tw(nseq);
        if (X.hmap && tid == 0 && blockIdx.x < ntiles) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            issue_h(X, X.hbuf, (int)((long)tw.seq * A.T + (long)tw.chunk * kT));
        }
        for (long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, tw.next(), X.hbuf ^= 1) {
            const int t0 = tw.chunk * kT;
            __syncthreads();
            if (X.hmap && tid == 0 && tile + gridDim.x < ntiles) {
                TileWalk nx = tw;
                nx.next();
                issue_h(X, X.hbuf ^ 1, (int)((long)nx.seq * A.T + (long)nx.chunk * kT));
            }
            const float r = cell_phase(A, X, tw.seq, t0, min(kT, A.T - t0), true, nullptr, true);
            my_res = (r > my_res || isnan(r)) ? r : my_res;
            if (*X.s_fail) return;
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

__global__ void __launch_bounds__(kThreads, 1) deer_tc_kernel(const DeerTcArgs A, const __grid_constant__ CUtensorMap hmap,
                                                               int use_tma) {
    extern __shared__ __align__(1024) unsigned char smraw[];
    TileCtx X;
    // offset from the array itself, so that accesses stay in the shared window
    X.base = smraw + ((1024u - (smem_addr(smraw) & 1023u)) & 1023u);
    X.sbase = smem_addr(X.base);
    X.bars = reinterpret_cast<unsigned long long *>(X.base + kOffMisc);
    unsigned *tmem_slot = reinterpret_cast<unsigned *>(X.base + kOffMisc + 32);
    X.s_fail = reinterpret_cast<volatile int *>(X.base + kOffMisc + 36);
    unsigned *s_red = reinterpret_cast<unsigned *>(X.base + kOffMisc + 64);
    X.ph0 = X.ph1 = 0u;
    X.hph = 0u;
    X.hbuf = 0;
    X.hmap = use_tma ? &hmap : nullptr;
    X.bad = false;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        *X.s_fail = 0;
        for (int q = 0; q < 4; ++q) mbar_init(X.bars + q, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    {
        // A in fp32 for the re-walk; W^T and the bias for the cell's raw inputs
        float *smf = reinterpret_cast<float *>(X.base);
        for (int e = tid; e < kN * 16; e += kThreads) {
            const int i = e >> 4, c = e & 15;
            float v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = (i < A.n && 4 * c + q < A.n) ? A.A[(size_t)i * A.n + 4 * c + q] : 0.f;
            *reinterpret_cast<float4 *>(smf + (kOffA >> 2) + i * kN + ((c ^ (i & 15)) << 2)) =
                make_float4(v[0], v[1], v[2], v[3]);
        }
        for (int e = tid; e < 9 * kN; e += kThreads) {
            const int q = e / kN, i = e % kN;
            float v = 0.f;
            if (!A.xproj && i < A.n) v = q < 8 ? (q < A.in ? A.W[(size_t)i * A.in + q] : 0.f) : (A.bias ? A.bias[i] : 0.f);
            smf[(kOffW >> 2) + e] = v;
        }
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // B operands, resident for the launch: row j of the chain products' holds A[.][j]
    // (element (k, j) = A[k][j]); row i of the cell product's holds A[i][.]
    for (int e = tid; e < kN * 16; e += kThreads) {
        const int j = e >> 4, c = e & 15;
        float v[4], w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int k = 4 * c + q;
            v[q] = (j < A.n && k < A.n) ? A.A[(size_t)k * A.n + j] : 0.f;
            w[q] = (j < A.n && k < A.n) ? A.A[(size_t)j * A.n + k] : 0.f;
        }
        const unsigned o = opnd_off(j, c), ol = opnd_off(64 + j, c);
        float h[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) h[q] = tf32_hi(v[q]);
        st_shared_v4(X.sbase + kOffB + o, h[0], h[1], h[2], h[3]);
        st_shared_v4(X.sbase + kOffB + ol, v[0] - h[0], v[1] - h[1], v[2] - h[2], v[3] - h[3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) h[q] = tf32_hi(w[q]);
        st_shared_v4(X.sbase + kOffC + o, h[0], h[1], h[2], h[3]);
        st_shared_v4(X.sbase + kOffC + ol, w[0] - h[0], w[1] - h[1], w[2] - h[2], w[3] - h[3]);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    X.tmem = *tmem_slot;

    deer_tc_body(A, X, s_red);

    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (*X.s_fail) {
        // after a timed-out product wait, give the tensor cores a bounded time to finish
        // before their columns are released
        if (tid == 0 && X.bad) __nanosleep(1000000);
        __syncthreads();
    }
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(X.tmem), "r"(kTmemCols)
                     : "memory");
    }
}

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

}  // namespace

int deer_tc_plan(const NewtonTanhReq &r, int num_sms, Plan *plan) {
    if (r.quasi || r.n <= 32 || r.n > kN) return 1;
    if (!r.xproj && (r.in < 1 || r.in > 8)) return 1;
    const void *kern = reinterpret_cast<const void *>(&deer_tc_kernel);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) return -1;
    plan->kernel = kern;
    plan->dyn_smem = kSmem;
    plan->ntiles = (long)r.B * ((r.T + kT - 1) / kT);
    if (plan->ntiles > 0x7fffffffL) return 1;
    plan->C = kN;
    plan->agg_words = 0;
    plan->inc_words = (size_t)plan->ntiles * kN;
    plan->side_bytes = 2 * (size_t)plan->ntiles * kN * sizeof(float);
    plan->epochs = (unsigned)r.max_iters + 1u;
    plan->variant = 1164;
    plan->threads = kThreads;
    plan->grid = occupancy_grid(plan->kernel, kThreads, kSmem, num_sms, plan->ntiles);
    return plan->grid > 0 ? 0 : -1;
}

cudaError_t deer_tc_launch(const NewtonTanhReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                           cudaStream_t st) {
    DeerTcArgs A;
    A.B = r.B;
    A.T = r.T;
    A.n = r.n;
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
    A.inc = w.inc;
    A.side = w.side;
    A.epoch0 = w.epoch0;
    A.dbg.wait_ns = dbg.wait_ns;
    A.dbg.skip_tile = dbg.skip_tile;
    A.dbg.delta_log = dbg.delta_log;
    A.dbg.delta_log_cap = dbg.delta_log_cap;
    A.dbg.no_halo = 1;
    // the states as a [B*T][n] tensor for TMA: rows of n floats (n % 4 == 0, 16-byte
    // aligned); otherwise the kernel stages them with plain loads
    CUtensorMap hmap;
    memset(&hmap, 0, sizeof(hmap));
    int use_tma = 0;
    EncodeTiledFn fn = encode_fn();
    if (fn && r.n % 4 == 0 && ((uintptr_t)r.h & 15) == 0 && (long)r.B * r.T < (1L << 31)) {
        cuuint64_t dims[2] = {(cuuint64_t)r.n, (cuuint64_t)r.B * r.T};
        cuuint64_t strides[1] = {(cuuint64_t)r.n * 4};
        cuuint32_t box[2] = {32, (cuuint32_t)kT};
        cuuint32_t estr[2] = {1, 1};
        if (fn(&hmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, r.h, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            use_tma = 1;
    }
    void *args[] = {&A, &hmap, &use_tma};
    return cudaLaunchCooperativeKernel(plan.kernel, dim3(plan.grid), dim3(plan.threads), args, plan.dyn_smem, st);
}

}  // namespace prn
