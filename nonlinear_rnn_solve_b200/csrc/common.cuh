// common.cuh -- device building blocks shared by the sm_100a kernels of the library:
// iteration bookkeeping, bounded waits, a grid barrier for persistent cooperative
// kernels, affine scan elements and the chunked scan (CTA scan + decoupled look-back).
//
// The linear recurrence h_t = J_t h_{t-1} + b_t that every Newton iteration solves
// ("Parallelizing non-linear sequential models over the sequence length", Approach:
// the linear recurrence is solved with an associative prefix scan) is a composition
// of affine maps x -> J x + b.  Composition is associative, so a chunk of steps
// reduces to one affine map, and chunks combine in any grouping.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace prn {

constexpr int kThreads = 256;

// ------------------------------------------------------------------ status / control
enum : int { kStNonfinite = 1, kStTimeout = 2, kStNotConverged = 4 };
enum : unsigned { kFlagAgg = 1u, kFlagInc = 2u };  // look-back states

// Per-call control block (zeroed by the host before every launch).
struct Ctl {
    unsigned bar_count;
    unsigned bar_gen;
    unsigned delta_bits[3];  // ring of per-iteration max|delta| (float bits, >= 0)
    unsigned res_bits;       // residual max (float bits)
    int abort;               // set on a timeout: every wait gives up at once
    int pad[9];
};

// Debug / test controls passed by value in every kernel's arguments.
struct Dbg {
    unsigned long long wait_ns;  // bounded-wait limit
    long long skip_tile;         // tile whose look-back publication is withheld (-1 none)
    float *delta_log;            // per-iteration delta (may be null)
    int delta_log_cap;
    int no_halo;                 // 1: tiles always take the carry from the look-back
};

__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_relaxed_int(const int *p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void raise_status(int *sticky, Ctl *ctl, int bit, bool abort) {
    atomicOr(sticky, bit);
    if (abort) atomicExch(&ctl->abort, 1);
}

// Grid-wide barrier for a cooperative (co-resident) grid.  Every wait is bounded:
// it gives up when the per-call abort flag is set or after dbg.wait_ns, raising
// kStTimeout.  Returns false when the kernel must stop.
__device__ __forceinline__ bool grid_sync(Ctl *ctl, int *sticky, const Dbg &dbg) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        unsigned gen = ld_acquire(&ctl->bar_gen);
        __threadfence();
        unsigned arrived = atomicAdd(&ctl->bar_count, 1u);
        if (arrived == gridDim.x - 1) {
            atomicExch(&ctl->bar_count, 0u);
            __threadfence();
            st_release(&ctl->bar_gen, gen + 1);
        } else {
            unsigned long long t0 = gtimer();
            while (ld_acquire(&ctl->bar_gen) == gen) {
                if (ld_relaxed_int(&ctl->abort)) { ok = 0; break; }
                if (gtimer() - t0 > dbg.wait_ns) {
                    raise_status(sticky, ctl, kStTimeout, true);
                    ok = 0;
                    break;
                }
                __nanosleep(64);
            }
        }
        if (ld_relaxed_int(&ctl->abort)) ok = 0;
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// ------------------------------------------------------------------ math
// Logistic function and tanh from the exponential: s(u) = 1 / (1 + e^-u),
// tanh(u) = 2 s(2u) - 1 (textbook identities), with the hardware exp2-based
// __expf and a fast reciprocal.  Absolute error stays near 1e-7, far inside the
// 1e-4 state tolerance; both are deterministic, so Newton converges to the fixed
// point of exactly this cell.
__device__ __forceinline__ float sigm(float u) { return __fdividef(1.0f, 1.0f + __expf(-u)); }
__device__ __forceinline__ float tanh_(float u) { return fmaf(2.0f, sigm(2.0f * u), -1.0f); }

// 2^y and 1/y with the hardware approximations (PTX ex2.approx / rcp.approx, a few
// ulp): with e^u = 2^(u log2 e) folded into the inputs' scale, a logistic function
// costs one fused multiply-add, two special-function operations and one add.
__device__ __forceinline__ float ex2_hw(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}
__device__ __forceinline__ float rcp_hw(float y) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}
constexpr float kLog2e = 1.4426950408889634f;

// The matrix the step map is linearised with (see jmode): the Jacobian as evaluated
// (0), the diagonal of a 2x2 block (1), zero (2, Jacobi) or the identity (3, Picard).
template <int S> __device__ __forceinline__ void apply_jmode(int jmode, float *J) {
    if (jmode == 0) return;
    if (jmode == 1) {
        if (S == 2) {
            J[1 % (S * S)] = 0.f;
            J[2 % (S * S)] = 0.f;
        }
        return;
    }
#pragma unroll
    for (int q = 0; q < S * S; ++q) J[q] = (jmode == 3 && q % (S + 1) == 0) ? 1.f : 0.f;
}

__device__ __forceinline__ bool finitef(float v) { return fabsf(v) <= 3.402823466e38f; }

// ------------------------------------------------------------------ affine elements
// Aff<S>: x -> a x + d with x an S-vector (S = 1 diagonal, S = 2 for 2x2 blocks).
template <int S> struct Aff;
template <> struct Aff<1> {
    float a, d;
    __device__ __forceinline__ static Aff ident() { return {1.f, 0.f}; }
    __device__ __forceinline__ static Aff cst(const float *v) { return {0.f, v[0]}; }
    __device__ __forceinline__ void apply(const float *x, float *y) const { y[0] = fmaf(a, x[0], d); }
    __device__ __forceinline__ Aff shfl_up(unsigned off) const {
        return {__shfl_up_sync(0xffffffffu, a, off), __shfl_up_sync(0xffffffffu, d, off)};
    }
    __device__ __forceinline__ Aff shfl_down(unsigned off) const {
        return {__shfl_down_sync(0xffffffffu, a, off), __shfl_down_sync(0xffffffffu, d, off)};
    }
    __device__ __forceinline__ void to_floats(float *v) const { v[0] = a; v[1] = d; }
    __device__ __forceinline__ static Aff from_floats(const float *v) { return {v[0], v[1]}; }
    // a published aggregate that is a constant map (its value does not depend on the carry)
    __device__ __forceinline__ static bool const_floats(const float *v) { return v[0] == 0.f; }
    __device__ __forceinline__ static void const_value(const float *v, float *x) { x[0] = v[1]; }
    static constexpr int kFloats = 2;
};
template <> struct Aff<2> {
    float a00, a01, a10, a11, d0, d1;
    __device__ __forceinline__ static Aff ident() { return {1.f, 0.f, 0.f, 1.f, 0.f, 0.f}; }
    __device__ __forceinline__ static Aff cst(const float *v) { return {0.f, 0.f, 0.f, 0.f, v[0], v[1]}; }
    __device__ __forceinline__ void apply(const float *x, float *y) const {
        float y0 = fmaf(a00, x[0], fmaf(a01, x[1], d0));
        float y1 = fmaf(a10, x[0], fmaf(a11, x[1], d1));
        y[0] = y0;
        y[1] = y1;
    }
    __device__ __forceinline__ Aff shfl_up(unsigned off) const {
        const unsigned m = 0xffffffffu;
        return {__shfl_up_sync(m, a00, off), __shfl_up_sync(m, a01, off), __shfl_up_sync(m, a10, off),
                __shfl_up_sync(m, a11, off), __shfl_up_sync(m, d0, off), __shfl_up_sync(m, d1, off)};
    }
    __device__ __forceinline__ Aff shfl_down(unsigned off) const {
        const unsigned m = 0xffffffffu;
        return {__shfl_down_sync(m, a00, off), __shfl_down_sync(m, a01, off), __shfl_down_sync(m, a10, off),
                __shfl_down_sync(m, a11, off), __shfl_down_sync(m, d0, off), __shfl_down_sync(m, d1, off)};
    }
    __device__ __forceinline__ void to_floats(float *v) const {
        v[0] = a00; v[1] = a01; v[2] = a10; v[3] = a11; v[4] = d0; v[5] = d1;
    }
    __device__ __forceinline__ static Aff from_floats(const float *v) { return {v[0], v[1], v[2], v[3], v[4], v[5]}; }
    __device__ __forceinline__ static bool const_floats(const float *v) {
        return v[0] == 0.f && v[1] == 0.f && v[2] == 0.f && v[3] == 0.f;
    }
    __device__ __forceinline__ static void const_value(const float *v, float *x) {
        x[0] = v[4];
        x[1] = v[5];
    }
    static constexpr int kFloats = 6;
};

// outer o inner: apply `inner` first, then `outer`.
__device__ __forceinline__ Aff<1> compose(const Aff<1> &inner, const Aff<1> &outer) {
    return {outer.a * inner.a, fmaf(outer.a, inner.d, outer.d)};
}
__device__ __forceinline__ Aff<2> compose(const Aff<2> &i, const Aff<2> &o) {
    Aff<2> r;
    r.a00 = fmaf(o.a00, i.a00, o.a01 * i.a10);
    r.a01 = fmaf(o.a00, i.a01, o.a01 * i.a11);
    r.a10 = fmaf(o.a10, i.a00, o.a11 * i.a10);
    r.a11 = fmaf(o.a10, i.a01, o.a11 * i.a11);
    r.d0 = fmaf(o.a00, i.d0, fmaf(o.a01, i.d1, o.d0));
    r.d1 = fmaf(o.a10, i.d0, fmaf(o.a11, i.d1, o.d1));
    return r;
}
// Element for one step of a recurrence, from a Jacobian (S x S row-major) and an offset.
template <int S> __device__ __forceinline__ Aff<S> make_aff(const float *J, const float *d);
template <> __device__ __forceinline__ Aff<1> make_aff<1>(const float *J, const float *d) { return {J[0], d[0]}; }
template <> __device__ __forceinline__ Aff<2> make_aff<2>(const float *J, const float *d) {
    return {J[0], J[1], J[2], J[3], d[0], d[1]};
}

// ------------------------------------------------------------------ cp.async
// Asynchronous copies global -> shared, 16 or 4 bytes; src_bytes 0 / valid false
// zero-fills the destination without reading the source.
__device__ __forceinline__ void cp_async16(float *dst, const float *src, int src_bytes) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(float *dst, const float *src, bool valid) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ tile walk
// Grid-stride walk over tiles numbered tile = chunk * nseq + seq (seq fastest): the
// coordinates advance by gridDim.x tiles per step without dividing (plans keep tile
// counts below 2^31).
struct TileWalk {
    int nseq, step_ch, step_sq, chunk, seq;
    __device__ __forceinline__ explicit TileWalk(long n) : nseq((int)n) {
        step_ch = (int)(gridDim.x / (unsigned)nseq);
        step_sq = (int)(gridDim.x % (unsigned)nseq);
        chunk = (int)(blockIdx.x / (unsigned)nseq);
        seq = (int)(blockIdx.x % (unsigned)nseq);
    }
    __device__ __forceinline__ void next() {
        chunk += step_ch;
        seq += step_sq;
        if (seq >= nseq) {
            seq -= nseq;
            ++chunk;
        }
    }
};

// ------------------------------------------------------------------ chunked scan
// Look-back workspace: every published float travels in one 64-bit word together
// with the 32-bit epoch of the iteration that wrote it, so a reader that sees the
// current epoch in a word also sees that word's value (single-copy atomic 64-bit
// access): no fences and no separate flag are needed.  Epochs are unique per
// context across launches (the host hands out a fresh range for every launch), so
// words left by earlier launches or iterations never match.
//   agg [ntiles][C][Aff<S>::kFloats]  tile aggregate per channel (published first)
//   inc [ntiles][C][S]                carried state at the tile's last step
template <int S> struct LookBack {
    unsigned long long *agg;
    unsigned long long *inc;
};

__device__ __forceinline__ unsigned long long pack_tag(float v, unsigned epoch) {
    return ((unsigned long long)__float_as_uint(v) << 32) | epoch;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

template <int S, int C, int NT = kThreads, class E = Aff<S>> struct ScanSmem {
    static constexpr int NW = NT / 32;
    E wtot[NW][C];  // per-warp totals (scan order)
    float carry[C][S];   // carry entering the tile, per channel
};

// Inclusive composition, in scan order, of the per-thread elements of one tile.
// Threads are laid out tid = s * C + c (s = scan position, c = channel); C divides 32.
// On return: `excl` is the composition of the elements before this thread's
// position (identity for s = 0) and `total` (valid in warp 0, lanes c < C) is the
// tile's aggregate for channel c.
template <int S, int C, int NT = kThreads, class E = Aff<S>>
__device__ __forceinline__ void cta_scan(const E &e, ScanSmem<S, C, NT, E> &sm, E &excl, E &total) {
    static_assert(32 % C == 0, "C must divide 32");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    E inc = e;
#pragma unroll
    for (int off = C; off < 32; off <<= 1) {
        E o = inc.shfl_up(off);
        if (lane >= off) inc = compose(o, inc);
    }
    E wex = inc.shfl_up(C);
    if (lane < C) wex = E::ident();
    if (lane >= 32 - C) sm.wtot[warp][lane - (32 - C)] = inc;
    __syncthreads();
    const int c = lane % C;
    E pre = E::ident();
    for (int w = 0; w < warp; ++w) pre = compose(pre, sm.wtot[w][c]);
    excl = compose(pre, wex);
    if (warp == 0 && lane < C) {
        E t = E::ident();
#pragma unroll
        for (int w = 0; w < ScanSmem<S, C, NT, E>::NW; ++w) t = compose(t, sm.wtot[w][lane]);
        total = t;
    }
}

// Decoupled look-back, in three parts, run by warp 0 with lane = i * C + c (window
// slot i, channel c).  Every wait is bounded (abort flag, dbg.wait_ns).
//
// publish_agg: lanes c < C publish the tile aggregate (tiles with chunk > 0).
template <int S, int C, class E = Aff<S>>
__device__ __forceinline__ void publish_agg(const LookBack<S> &lb, const E &total, long tile, int chunk,
                                            unsigned epoch, const Dbg &dbg) {
    constexpr int KF = E::kFloats;
    const int lane = threadIdx.x & 31;
    if (chunk == 0 || lane >= C || dbg.skip_tile == tile) return;
    float tv[KF];
    total.to_floats(tv);
#pragma unroll
    for (int q = 0; q < KF; ++q) st_relaxed_u64(lb.agg + (tile * C + lane) * KF + q, pack_tag(tv[q], epoch));
}

// resolve_carry: the carried state entering `tile`, valid in lanes c < C.  Walks the
// predecessors (tile - nseq, tile - 2 nseq, ...) in windows of 32 / C, composing their
// aggregates until a known value: an inclusive value, the start of the sequence (carry
// `base`), or an aggregate whose matrix part is exactly zero (a constant map: nothing
// before it can change the carry; long tiles of a contractive recurrence underflow to
// this).  The warp polls together and never waits for slots behind the first known
// value.  Returns false on a timeout / abort.
template <int S> __device__ __forceinline__ bool aff_is_const(const float *v) {
#pragma unroll
    for (int q = 0; q < S * S; ++q)
        if (v[q] != 0.f) return false;
    return true;
}

template <int S, int C, class E = Aff<S>>
__device__ bool resolve_carry(const LookBack<S> &lb, long tile, int chunk, long nseq, unsigned epoch,
                              const float *base, float *carry, Ctl *ctl, int *sticky, const Dbg &dbg) {
    constexpr int WIN = 32 / C;
    constexpr int KF = E::kFloats;
    const int lane = threadIdx.x & 31, i = lane / C, c = lane % C;
    if (chunk == 0) {
#pragma unroll
        for (int q = 0; q < S; ++q) carry[q] = base[q];
        return true;
    }
    E acc = E::ident();  // composition of everything between here and the window
    long pred = tile - nseq;
    int pchunk = chunk - 1;
    for (;;) {
        const int my_chunk = pchunk - i;
        const long my_tile = pred - (long)i * nseq;
        unsigned long long t0 = 0;
        int polls = 0;
        E v;
        unsigned st;  // 0 not ready, 1 aggregate, 2 known value
        for (;;) {
            st = 2u;
            if (my_chunk < 0) {
                v = E::cst(base);
            } else {
                unsigned long long wi[S], wa[KF];
#pragma unroll
                for (int q = 0; q < S; ++q) wi[q] = ld_relaxed_u64(lb.inc + (my_tile * C + c) * S + q);
#pragma unroll
                for (int q = 0; q < KF; ++q) wa[q] = ld_relaxed_u64(lb.agg + (my_tile * C + c) * KF + q);
                bool inc_ok = true, agg_ok = true;
                float iv[S], av[KF];
#pragma unroll
                for (int q = 0; q < S; ++q) {
                    inc_ok &= (unsigned)wi[q] == epoch;
                    iv[q] = __uint_as_float((unsigned)(wi[q] >> 32));
                }
#pragma unroll
                for (int q = 0; q < KF; ++q) {
                    agg_ok &= (unsigned)wa[q] == epoch;
                    av[q] = __uint_as_float((unsigned)(wa[q] >> 32));
                }
                if (inc_ok) {
                    v = E::cst(iv);
                } else if (agg_ok) {
                    v = E::from_floats(av);
                    st = E::const_floats(av) ? 2u : 1u;
                } else {
                    st = 0u;
                }
            }
            // every channel of a slot sees the same tile; a slot is known only if all
            // its channels are (C lanes per slot)
            const unsigned known = __ballot_sync(0xffffffffu, st == 2u);
            const unsigned ready = __ballot_sync(0xffffffffu, st != 0u);
            unsigned slot_known = 0, slot_ready = 0;
#pragma unroll
            for (int w = 0; w < WIN; ++w) {
                const unsigned m = (C == 32 ? 0xffffffffu : ((1u << C) - 1u)) << (w * C);
                if ((known & m) == m) slot_known |= 1u << w;
                if ((ready & m) == m) slot_ready |= 1u << w;
            }
            const int first = slot_known ? __ffs(slot_known) - 1 : WIN;
            const int need_n = first + 1 < WIN ? first + 1 : WIN;  // slots 0 .. first must be ready
            const unsigned need_w = need_n >= 32 ? 0xffffffffu : ((1u << need_n) - 1u);
            if ((slot_ready & need_w) == need_w) {
                // reduce the window up to the first known slot; slot 0 is the nearest
                // predecessor (applied last)
                if (i > first) v = E::ident();
#pragma unroll
                for (int off = C; off < 32; off <<= 1) {
                    E o = v.shfl_down(off);
                    if (lane + off < 32) v = compose(o, v);
                }
                acc = compose(v, acc);
                if (first < WIN) {
                    float z[S];
#pragma unroll
                    for (int q = 0; q < S; ++q) z[q] = 0.f;
                    acc.apply(z, carry);  // acc is a constant map here
                    return true;
                }
                break;  // whole window of aggregates: continue with the next window
            }
            ++polls;  // warp-uniform
            int bad = 0;
            if (lane == 0) {
                if (ld_relaxed_int(&ctl->abort)) bad = 1;
                if (polls == 4) t0 = gtimer();
                if (polls > 4 && gtimer() - t0 > dbg.wait_ns) {
                    raise_status(sticky, ctl, kStTimeout, true);
                    bad = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, bad, 0)) return false;
            if (polls > 4) __nanosleep(20);
        }
        pred -= (long)WIN * nseq;
        pchunk -= WIN;
    }
}

// publish_inc: lanes c < C publish the tile's inclusive value total(carry).
template <int S, int C, class E = Aff<S>>
__device__ __forceinline__ void publish_inc(const LookBack<S> &lb, const E &total, const float *carry, long tile,
                                            unsigned epoch, const Dbg &dbg) {
    const int lane = threadIdx.x & 31;
    if (lane >= C || dbg.skip_tile == tile) return;
    float incv[S];
    total.apply(carry, incv);
#pragma unroll
    for (int q = 0; q < S; ++q) st_relaxed_u64(lb.inc + (tile * C + lane) * S + q, pack_tag(incv[q], epoch));
}

// The whole look-back for one tile: publish the aggregate, resolve the carry, publish
// the inclusive value, leave the carry in sm.carry.  Returns false on a timeout.
// `halo` (optional, channel c): the composed map of the steps just before the tile,
// evaluated by the tile itself; when its matrix part is exactly zero it is a constant
// whose value is the carry, and no predecessor is read.
template <int S, int C, int NT = kThreads, class E = Aff<S>>
__device__ bool look_back(const LookBack<S> &lb, ScanSmem<S, C, NT, E> &sm, const E &total, long tile,
                          int chunk, long nseq, unsigned epoch, const float *base /* [S], channel c */,
                          Ctl *ctl, int *sticky, const Dbg &dbg, const E *halo = nullptr) {
    const int lane = threadIdx.x & 31;
    publish_agg<S, C, E>(lb, total, tile, chunk, epoch, dbg);
    float carry[S];
    bool known = false;
    if (halo != nullptr && chunk > 0) {
        float hv[E::kFloats];
        halo->to_floats(hv);
        known = __all_sync(0xffffffffu, lane >= C || E::const_floats(hv));
        if (known) E::const_value(hv, carry);
    }
    if (!known && !resolve_carry<S, C, E>(lb, tile, chunk, nseq, epoch, base, carry, ctl, sticky, dbg)) return false;
    publish_inc<S, C, E>(lb, total, carry, tile, epoch, dbg);
    if (lane < C) {
#pragma unroll
        for (int q = 0; q < S; ++q) sm.carry[lane][q] = carry[q];
    }
    return true;
}

// Block-wide max of a non-negative float (NaN propagates as a NaN bit pattern).
template <int NT = kThreads> __device__ __forceinline__ unsigned block_max_bits(float v, unsigned *s_red) {
    unsigned b = isnan(v) ? 0x7fc00000u : __float_as_uint(fabsf(v));
#pragma unroll
    for (int off = 16; off; off >>= 1) b = max(b, __shfl_xor_sync(0xffffffffu, b, off));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) s_red[warp] = b;
    __syncthreads();
    unsigned r = 0;
    if (threadIdx.x == 0)
        for (int w = 0; w < NT / 32; ++w) r = max(r, s_red[w]);
    __syncthreads();
    return r;  // valid in thread 0
}

}  // namespace prn
