// proj.cu -- the input projection xproj = x W^T + bias, the method's one dense
// contraction (the input term W x_t of every cell does not depend on the state, so it
// is computed once per forward pass; "Para-Seq" README, Main features: GRU/LSTM layers
// with input projections).
//
// bf16 path: a tcgen05 GEMM.  Persistent CTAs compute 128 x 256 fp32 tiles of xproj:
//   warp 0  (one elected thread) streams 128x64 tiles of x and 256x64 tiles of W into a
//           4-stage shared-memory ring with TMA (128-byte swizzle, no multicast);
//   warp 1  allocates 2 x 256 TMEM columns and (one elected thread) issues
//           tcgen05.mma.cta_group::1.kind::f16 (M = 128, N = 256, K = 16, bf16 x bf16 ->
//           fp32 in TMEM), releasing each stage with tcgen05.commit;
//   warps 2-9 drain the other accumulator: warp w owns TMEM lanes 32 (w % 4) .. + 31 (tile
//           rows) and columns 128 ((w - 2) / 4) .. + 127; a thread pulls its 128 columns
//           out of TMEM with one wait, hands the accumulator back at once, then adds the
//           bias and stores fp32 rows (so the next tile's MMAs never wait on the stores).
// Every mbarrier wait is bounded (%globaltimer); on a timeout the CTA raises the
// status bit, frees its TMEM and returns.
// fp32 path: a CUDA-core tiled GEMM (x and W both fp32).
#include <cuda.h>

#include <algorithm>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/pararnn.h"
#include "common.cuh"
#include "internal.h"

namespace prn {

namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 256;
constexpr int THREADS = 320;  // TMA warp, MMA warp, 8 epilogue warps
// The bias is copied into shared memory after the stage ring when it has at most this
// many entries (the ring leaves about 34 KB of the 227 KB): the epilogue then reads it as
// shared-memory broadcasts instead of global loads that the output stream keeps evicting
// from L1.
constexpr int BIAS_SMEM = 8192;
constexpr unsigned long long WAIT_NS = 2000000000ull;

__device__ __forceinline__ unsigned smem_u32(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(unsigned bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(unsigned bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(unsigned bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on an mbarrier phase; false on timeout or when the CTA aborted.
__device__ __forceinline__ bool mbar_wait(unsigned bar, unsigned parity, volatile int *abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (!mbar_try(bar, parity)) {
        if (*abort_flag) return false;
        if (gtimer() - t0 > WAIT_NS) return false;
    }
    return true;
}
__device__ __forceinline__ void tma_load_2d(unsigned dst, const CUtensorMap *map, int x, int y, unsigned bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// 128 consecutive TMEM columns of this thread's lane (four 32-column loads, one wait).
__device__ __forceinline__ void tmem_ld128(unsigned taddr, float (&v)[128]) {
    unsigned r[128];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%128];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%129];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95}, [%130];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%131];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
        : "r"(taddr), "r"(taddr + 32), "r"(taddr + 64), "r"(taddr + 96)
        : "memory");
#pragma unroll
    for (int j = 0; j < 128; ++j) v[j] = __uint_as_float(r[j]);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ unsigned long long smem_desc(unsigned addr) {
    return (unsigned long long)((addr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}
// Instruction descriptor: D fp32, A and B bf16, both K-major, N = 256, M = 128.
constexpr unsigned IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((unsigned)(BN >> 3) << 17) | ((unsigned)(BM >> 4) << 24);

// Persistent CTAs (one per SM) walk the output tiles n-fastest, so the CTAs that run
// at the same time share rows of x in L2 (W stays resident).  The accumulator is
// double-buffered in TMEM (2 x 256 columns): the epilogue warps drain tile i while the
// MMA thread accumulates tile i + 1, and the TMA producer runs ahead across tiles.
__global__ void __launch_bounds__(THREADS, 1)
    proj_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const float *__restrict__ bias, float *__restrict__ y, int M, int N, int K, int ksplit,
                     int *sticky) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char *smem = reinterpret_cast<unsigned char *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) unsigned long long bar_full[STAGES], bar_empty[STAGES], acc_full[2], acc_empty[2];
    __shared__ unsigned tmem_base_sh;
    __shared__ volatile int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kblocks = (K + BK - 1) / BK;
    const int mtiles = (M + BM - 1) / BM, ntiles_n = (N + BN - 1) / BN;
    const int ntiles = mtiles * ntiles_n;
    // work item = tile * ksplit + part: part p accumulates K blocks [p kblocks / ksplit,
    // (p + 1) kblocks / ksplit) into its own M x N slab of y (summed afterwards in a
    // fixed order); ksplit = 1 is the plain product
    const int nitems = ntiles * ksplit;
    // 32-byte vector stores need 32-byte aligned rows
    const bool vec8 = (N & 7) == 0 && ((uintptr_t)y & 31) == 0;
    const bool bias_sm = bias && N <= BIAS_SMEM;
    float *const bias_s = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES);  // [N] when bias_sm
    if (bias_sm)
        for (int i = threadIdx.x; i < N; i += THREADS) bias_s[i] = __ldg(bias + i);

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bar_full[s]), 1);
            mbar_init(smem_u32(&bar_empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);
            mbar_init(smem_u32(&acc_empty[a]), 8);  // one arrival per epilogue warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(2 * TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const unsigned tmem = tmem_base_sh;

    if (warp == 0) {
        if (lane == 0) {  // TMA producer, continuous over this CTA's tiles
            int it = 0;
            for (int item = blockIdx.x; item < nitems && !abort_flag; item += gridDim.x) {
                const int tile = item / ksplit, part = item % ksplit;
                const int m0 = (tile / ntiles_n) * BM, n0 = (tile % ntiles_n) * BN;
                const int kb0 = part * kblocks / ksplit, kb1 = (part + 1) * kblocks / ksplit;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    const unsigned ph = (unsigned)(it / STAGES) & 1u;
                    if (!mbar_wait(smem_u32(&bar_empty[s]), ph ^ 1u, &abort_flag)) { abort_flag = 1; break; }
                    unsigned char *sa = smem + s * STAGE_BYTES;
                    const unsigned fb = smem_u32(&bar_full[s]);
                    mbar_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(smem_u32(sa), &tmA, kb * BK, m0, fb);
                    tma_load_2d(smem_u32(sa + A_BYTES), &tmB, kb * BK, n0, fb);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // MMA issuer
            int it = 0, ti = 0;
            for (int item = blockIdx.x; item < nitems && !abort_flag; item += gridDim.x, ++ti) {
                const int part = item % ksplit;
                const int kb0 = part * kblocks / ksplit, kb1 = (part + 1) * kblocks / ksplit;
                const int a = ti & 1;
                const unsigned acc = tmem + (unsigned)(a * TMEM_COLS);
                // the epilogue has drained this accumulator (its previous tile)
                if (!mbar_wait(smem_u32(&acc_empty[a]), ((unsigned)(ti >> 1) & 1u) ^ 1u, &abort_flag)) {
                    abort_flag = 1;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    const unsigned ph = (unsigned)(it / STAGES) & 1u;
                    if (!mbar_wait(smem_u32(&bar_full[s]), ph, &abort_flag)) { abort_flag = 1; break; }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const unsigned a0 = smem_u32(smem + s * STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const unsigned long long ad = smem_desc(a0 + k * 32), bd = smem_desc(b0 + k * 32);
                        const unsigned accum = (kb > kb0 || k > 0) ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred p;\n\t"
                            "setp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(acc),
                            "l"(ad), "l"(bd), "r"(IDESC), "r"(accum)
                            : "memory");
                    }
                    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                     smem_u32(&bar_empty[s]))
                                 : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&acc_full[a]))
                             : "memory");
            }
        }
    } else {
        // epilogue: warps 2..9 own TMEM lanes 32*(warp % 4) .. +31 (tile rows) and one
        // 128-column half of the tile
        const int q = warp & 3, hcol = (warp - 2) >> 2;
        int ti = 0;
        for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++ti) {
            const int tile = item / ksplit, part = item % ksplit;
            const int a = ti & 1;
            const int m0 = (tile / ntiles_n) * BM, n0 = (tile % ntiles_n) * BN + 128 * hcol;
            const int row = m0 + q * 32 + lane;
            const bool ok =
                __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[a]), (unsigned)(ti >> 1) & 1u, &abort_flag));
            if (!ok) {
                abort_flag = 1;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            float v[128];
            tmem_ld128(tmem + ((unsigned)(q * 32) << 16) + (unsigned)(a * TMEM_COLS + 128 * hcol), v);
            // this half of the accumulator is in registers: hand it back
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&acc_empty[a])) : "memory");
            if (row < M) {
                float *yr = y + (size_t)part * M * N + (size_t)row * N;
#pragma unroll
                for (int c = 0; c < 128; c += 8) {
                    const int col = n0 + c;
                    const bool full = col + 8 <= N;
                    float w[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) w[j] = v[c + j];
                    if (bias) {
                        if (full) {
                            float4 b0, b1;
                            if (bias_sm) {  // 16-byte aligned: the ring is 1024-byte aligned, col % 8 == 0
                                b0 = *reinterpret_cast<const float4 *>(bias_s + col);
                                b1 = *reinterpret_cast<const float4 *>(bias_s + col + 4);
                            } else {
                                b0 = __ldg(reinterpret_cast<const float4 *>(bias + col));
                                b1 = __ldg(reinterpret_cast<const float4 *>(bias + col + 4));
                            }
                            w[0] += b0.x, w[1] += b0.y, w[2] += b0.z, w[3] += b0.w;
                            w[4] += b1.x, w[5] += b1.y, w[6] += b1.z, w[7] += b1.w;
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (col + j < N) w[j] += __ldg(bias + col + j);
                        }
                    }
                    if (full && vec8) {
                        // whole 32-byte sectors per lane
                        asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(yr + col),
                                     "f"(w[0]), "f"(w[1]), "f"(w[2]), "f"(w[3]), "f"(w[4]), "f"(w[5]), "f"(w[6]),
                                     "f"(w[7])
                                     : "memory");
                    } else if (full && (N & 3) == 0) {
                        *reinterpret_cast<float4 *>(yr + col) = make_float4(w[0], w[1], w[2], w[3]);
                        *reinterpret_cast<float4 *>(yr + col + 4) = make_float4(w[4], w[5], w[6], w[7]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (col + j < N) yr[col + j] = w[j];
                    }
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (abort_flag && threadIdx.x == 0) atomicOr(sticky, kStTimeout);
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * TMEM_COLS) : "memory");
    }
}

}  // namespace gemm

// ------------------------------------------------------------------ fp32 (CUDA cores)
// 64 x 64 output tile per 256-thread CTA, 4 x 4 outputs per thread, K in steps of 16.
__global__ void __launch_bounds__(256) proj_f32_kernel(const float *__restrict__ x, const float *__restrict__ W,
                                                       const float *__restrict__ bias, float *__restrict__ y, int M,
                                                       int N, int K) {
    __shared__ float xs[16][64 + 4], ws[16][64 + 4];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int m0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int e = threadIdx.x; e < 16 * 64; e += 256) {
            const int r = e / 16, kk = e % 16;
            xs[kk][r] = (m0 + r < M && k0 + kk < K) ? x[(size_t)(m0 + r) * K + k0 + kk] : 0.f;
            ws[kk][r] = (n0 + r < N && k0 + kk < K) ? W[(size_t)(n0 + r) * K + k0 + kk] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) y[(size_t)m * N + n] = acc[i][j] + (bias ? bias[n] : 0.f);
        }
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

// 2-D bf16 row-major [rows, K] tensor, boxes of 64 (K) x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *ptr, int rows, int K, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)gemm::BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// bf16 needs K % 8 == 0 (16-byte row pitch for TMA); fp32 has no extra condition.
int proj_check(int x_dtype, int M, int K, int N) {
    if (x_dtype == PARARNN_BF16 && (K % 8) != 0) return PARARNN_EINVAL;
    if ((long long)M * N > (1ll << 40)) return PARARNN_EINVAL;
    return PARARNN_OK;
}

namespace {

// y[i] = sum_p parts[p][i] (+ bias[i % N]), the parts added in order p = 0, 1, ...
__global__ void split_sum_kernel(const float *__restrict__ parts, int ksplit, size_t n, const float *__restrict__ bias,
                                 int N, float *__restrict__ y) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        float acc = parts[i];
        for (int p = 1; p < ksplit; ++p) acc += parts[(size_t)p * n + i];
        if (bias) acc += bias[i % N];
        y[i] = acc;
    }
}

// K blocks split into ksplit parts when the output has fewer tiles than there are SMs and
// that shortens the product: the work items fill ceil(tiles * s / SMs) waves of kblocks / s
// blocks each (about 0.3 us per block on the layer shapes), and the parts cost (s + 1) M N
// 4 bytes of HBM traffic to sum.  (With a wave or more of tiles the extra epilogue and
// summing traffic outweighed the better balance on the 6144 x 2048 weight gradient.)
int choose_ksplit(int M, int N, int K, int sms, size_t ws_floats) {
    const long tiles = (long)((M + gemm::BM - 1) / gemm::BM) * ((N + gemm::BN - 1) / gemm::BN);
    const int kblocks = (K + gemm::BK - 1) / gemm::BK;
    if (tiles >= sms) return 1;
    int best = 1;
    double best_us = 1e300;
    for (int s = 1; s <= kMaxKsplit; ++s) {
        if (s > 1 && (kblocks / s < 8 || (size_t)s * M * N > ws_floats)) break;
        const long waves = (tiles * s + sms - 1) / sms;
        const double us = waves * ((kblocks + s - 1) / s) * 0.3 + (s > 1 ? (s + 1) * 4.0 * M * N / 6.5e6 : 0.0);
        if (us < best_us) {
            best_us = us;
            best = s;
        }
    }
    return best;
}

}  // namespace

cudaError_t proj_launch_split(int x_dtype, const void *x, const void *W, const float *bias, float *y, int M, int K,
                              int N, int, cudaStream_t st, int *launches, int *sticky, float *ws, size_t ws_floats) {
    *launches = 0;
    if (x_dtype == PARARNN_F32) {
        dim3 grid((M + 63) / 64, (N + 63) / 64);
        proj_f32_kernel<<<grid, 256, 0, st>>>(static_cast<const float *>(x), static_cast<const float *>(W), bias, y,
                                              M, N, K);
        *launches = 1;
        return cudaGetLastError();
    }
    CUtensorMap ta, tb;
    if (!make_map(&ta, x, M, K, gemm::BM) || !make_map(&tb, W, N, K, gemm::BN)) return cudaErrorInvalidValue;
    // the stage ring, its 1024-byte alignment slack and the bias table (when it is used)
    const int smem_max = gemm::STAGES * gemm::STAGE_BYTES + 1024 + gemm::BIAS_SMEM * (int)sizeof(float);
    const int smem = gemm::STAGES * gemm::STAGE_BYTES + 1024 +
                     ((bias && N <= gemm::BIAS_SMEM) ? N * (int)sizeof(float) : 0);
    cudaError_t e =
        cudaFuncSetAttribute(gemm::proj_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int ksplit = ws ? choose_ksplit(M, N, K, sms, ws_floats) : 1;
    const long tiles = (long)((M + gemm::BM - 1) / gemm::BM) * ((N + gemm::BN - 1) / gemm::BN);
    const int grid = (int)std::min<long>(tiles * ksplit, sms);  // persistent: one CTA per SM
    if (ksplit == 1) {
        gemm::proj_bf16_kernel<<<grid, gemm::THREADS, smem, st>>>(ta, tb, bias, y, M, N, K, 1, sticky);
        *launches = 1;
        return cudaGetLastError();
    }
    gemm::proj_bf16_kernel<<<grid, gemm::THREADS, smem, st>>>(ta, tb, nullptr, ws, M, N, K, ksplit, sticky);
    const size_t n = (size_t)M * N;
    split_sum_kernel<<<(int)std::min<size_t>((n + 255) / 256, (size_t)sms * 16), 256, 0, st>>>(ws, ksplit, n, bias, N,
                                                                                              y);
    *launches = 2;
    return cudaGetLastError();
}

cudaError_t proj_launch(int x_dtype, const void *x, const void *W, const float *bias, float *y, int M, int K, int N,
                        int num_sms, cudaStream_t st, int *launches, int *sticky) {
    return proj_launch_split(x_dtype, x, W, bias, y, M, K, N, num_sms, st, launches, sticky, nullptr, 0);
}

}  // namespace prn
