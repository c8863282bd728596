// staged_tiles.cuh -- shared-memory staging for the long-sequence Newton kernels:
// TMA (cp.async.bulk.tensor, no multicast) copies with mbarrier completion, the 128-byte swizzle of TMA rows, and the TmaLong tile layout (H = 1).
#pragma once
#include <cuda.h>

#include "cells.cuh"
#include "common.cuh"
#include "newton_common.cuh"

namespace prn {


__device__ __forceinline__ unsigned smem_addr(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(unsigned long long *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(unsigned long long *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try(unsigned long long *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<unsigned long long>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Like mbar_try, but a thread whose phase is not complete is suspended in hardware
// until it completes or about `ns` nanoseconds pass (no issue slots spent polling).
__device__ __forceinline__ bool mbar_try_sleep(unsigned long long *bar, unsigned parity, unsigned ns) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Hint: bring a 2-D box into L2 ahead of its load (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<unsigned long long>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

// Copy n floats (n % 4 == 0) from a 16-byte aligned global address into consecutive
// segments of `seg` floats placed `str` floats apart; bytes at or beyond `end` are
// zero-filled.  Consecutive threads copy consecutive 16-byte chunks (coalesced).
template <int NT>
__device__ __forceinline__ void copy_segments(float *dst, int seg, int str, const float *src, int n,
                                              const float *end) {
    for (int f = 4 * threadIdx.x; f < n; f += 4 * NT) {
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

// ---------------------------------------------------------------- TMA long layout, H == 1
// A slab of the tile is a run of 128-byte rows; TMA writes row r's 16-byte chunk j at
// chunk position j ^ (r % 8) of its 1024-byte group.  Thread s's segment of `SEG` floats
// (8, 16 or 32) is part of one row, so its 128-bit reads land on distinct bank groups
// across each quarter-warp.
template <int SEG> __device__ __forceinline__ float4 *swz_chunk(float *region, int s, int j) {
    const int f = s * SEG + 4 * j;  // float offset of the chunk in the slab
    const int row = f >> 5, lc = (f >> 2) & 7;
    return reinterpret_cast<float4 *>(region + row * 32 + ((lc ^ (row & 7)) << 2));
}
__device__ __forceinline__ float swz_float(const float *region, int f) {
    const int row = f >> 5, lc = (f >> 2) & 7;
    return region[row * 32 + ((lc ^ (row & 7)) << 2) + (f & 3)];
}

template <class Cell, int IN, int LL, int NT, int HL = 0> struct TmaLong {
    static constexpr int S = Cell::S, C = 1, L = LL, SUB = NT, TCH = SUB * L, PW = IN;
    static constexpr int HALO = HL;
    static constexpr int SEGP = L * PW, SEGH = L * S;
    static_assert(SEGP == 8 || SEGP == 16 || SEGP == 32, "input segment must be part of one 128-byte row");
    static_assert(SEGH == 8 || SEGH == 16 || SEGH == 32, "state segment must be part of one 128-byte row");
    static constexpr int XFLOATS = TCH * PW, HFLOATS = TCH * S;
    static_assert(XFLOATS / 32 <= 256 && HFLOATS / 32 <= 256, "TMA box height");
    // regions: X | H | OUT (two, by tile parity), each a multiple of 1024 bytes
    static constexpr int OFFH = XFLOATS, OFFO = XFLOATS + HFLOATS;
    static constexpr int SMEM_FLOATS = XFLOATS + 3 * HFLOATS;
    static constexpr int OUT_STRIDE = HFLOATS;  // offset of the second staging tile
    static constexpr bool kTma = true;

    __device__ static void issue(const NewtonDiagArgs &A, const StagedMaps &M, float *sm, unsigned long long *bar,
                                 int b, int, int tch0, bool with_h) {
        const int rowx = (int)(((long)b * A.T + tch0) * PW / 32), rowh = (int)(((long)b * A.T + tch0) * S / 32);
        mbar_expect_tx(bar, (unsigned)(XFLOATS + (with_h ? HFLOATS : 0)) * 4u);
        tma_load_2d(sm, &M.x, 0, rowx, bar);
        if (with_h) tma_load_2d(sm + OFFH, &M.h, 0, rowh, bar);
    }
    // the same boxes into L2, one tile ahead of issue()
    __device__ static void prefetch(const NewtonDiagArgs &A, const StagedMaps &M, int b, int tch0, bool with_h) {
        tma_prefetch_2d(&M.x, 0, (int)(((long)b * A.T + tch0) * PW / 32));
        if (with_h) tma_prefetch_2d(&M.h, 0, (int)(((long)b * A.T + tch0) * S / 32));
    }
    __device__ static void load_group(float *sm, int s, int, int grp, float pv[4][PW], float hv[4][S], bool with_h) {
        float tp[4 * PW];
#pragma unroll
        for (int q = 0; q < PW; ++q) {
            const float4 v = *swz_chunk<SEGP>(sm, s, grp * PW + q);
            tp[4 * q] = v.x;
            tp[4 * q + 1] = v.y;
            tp[4 * q + 2] = v.z;
            tp[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int q = 0; q < PW; ++q) pv[j][q] = tp[j * PW + q];
        if (with_h) {
            float th[4 * S];
#pragma unroll
            for (int q = 0; q < S; ++q) {
                const float4 v = *swz_chunk<SEGH>(sm + OFFH, s, grp * S + q);
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
        for (int q = 0; q < S; ++q) hp[q] = swz_float(sm + OFFH, s * SEGH - S + q);
    }
    // results of steps 4*grp .. 4*grp + 3 of thread s, into the staging tile
    __device__ static void put_group(const NewtonDiagArgs &, float *sm, int s, int, int grp, const float hn[4][S], int,
                                     int, int) {
#pragma unroll
        for (int q = 0; q < S; ++q) {
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = hn[(4 * q + e) / S][(4 * q + e) % S];
            *swz_chunk<SEGH>(sm + OFFO, s, grp * S + q) = make_float4(v[0], v[1], v[2], v[3]);
        }
    }
    // coalesced 16-byte stores of the staged results of the tile (the caller puts a
    // barrier between the put_group writes and this)
    __device__ static void flush(const NewtonDiagArgs &A, float *sm, int b, int, int tch0) {
        const int valid = min(TCH, A.T - tch0) * S;
        float *g = A.h + ((size_t)b * A.T + tch0) * S;
        const float *o = sm + OFFO;
        for (int c = threadIdx.x; 4 * c < valid; c += NT) {
            const int row = c >> 3, lc = c & 7;
            const float4 v = *reinterpret_cast<const float4 *>(o + row * 32 + ((lc ^ (row & 7)) << 2));
            *reinterpret_cast<float4 *>(g + 4 * c) = v;
        }
    }
};

}  // namespace prn
