// proj.cu -- the input projection xproj = x W^T + bias, the method's one dense
// contraction (the input term W x_t of every cell does not depend on the state, so it
// is computed once per forward pass; "Para-Seq" README, Main features: GRU/LSTM layers
// with input projections).
//
// bf16 path: a tcgen05 GEMM.  Each CTA computes one 128 x 256 fp32 tile of xproj:
//   warp 0  (one elected thread) streams 128x64 tiles of x and 256x64 tiles of W into a
//           4-stage shared-memory ring with TMA (128-byte swizzle, no multicast);
//   warp 1  allocates 256 TMEM columns and (one elected thread) issues
//           tcgen05.mma.cta_group::1.kind::f16 (M = 128, N = 256, K = 16, bf16 x bf16 ->
//           fp32 in TMEM), releasing each stage with tcgen05.commit;
//   warps 2-5 read the accumulator with tcgen05.ld (32 lanes x 16 columns per load), add
//           the bias and store fp32 rows.
// Every mbarrier wait is bounded (%globaltimer); on a timeout the CTA raises the
// status bit, frees its TMEM and returns.
// fp32 path: a CUDA-core tiled GEMM (x and W both fp32).
#include <cuda.h>
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
constexpr int THREADS = 192;
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
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ unsigned long long smem_desc(unsigned addr) {
    return (unsigned long long)((addr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}
// Instruction descriptor: D fp32, A and B bf16, both K-major, N = 256, M = 128.
constexpr unsigned IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((unsigned)(BN >> 3) << 17) | ((unsigned)(BM >> 4) << 24);

__global__ void __launch_bounds__(THREADS, 1)
    proj_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const float *__restrict__ bias, float *__restrict__ y, int M, int N, int K, int *sticky) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char *smem = reinterpret_cast<unsigned char *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) unsigned long long bar_full[STAGES], bar_empty[STAGES], bar_acc;
    __shared__ unsigned tmem_base_sh;
    __shared__ volatile int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    const int kblocks = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bar_full[s]), 1);
            mbar_init(smem_u32(&bar_empty[s]), 1);
        }
        mbar_init(smem_u32(&bar_acc), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const unsigned tmem = tmem_base_sh;

    if (warp == 0) {
        if (lane == 0) {  // TMA producer
            for (int kb = 0; kb < kblocks; ++kb) {
                const int s = kb % STAGES;
                const unsigned ph = (unsigned)(kb / STAGES) & 1u;
                if (!mbar_wait(smem_u32(&bar_empty[s]), ph ^ 1u, &abort_flag)) { abort_flag = 1; break; }
                unsigned char *sa = smem + s * STAGE_BYTES;
                const unsigned fb = smem_u32(&bar_full[s]);
                mbar_expect_tx(fb, STAGE_BYTES);
                tma_load_2d(smem_u32(sa), &tmA, kb * BK, m0, fb);
                tma_load_2d(smem_u32(sa + A_BYTES), &tmB, kb * BK, n0, fb);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // MMA issuer
            for (int kb = 0; kb < kblocks; ++kb) {
                const int s = kb % STAGES;
                const unsigned ph = (unsigned)(kb / STAGES) & 1u;
                if (!mbar_wait(smem_u32(&bar_full[s]), ph, &abort_flag)) { abort_flag = 1; break; }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const unsigned a0 = smem_u32(smem + s * STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
                for (int k = 0; k < BK / 16; ++k) {
                    const unsigned long long ad = smem_desc(a0 + k * 32), bd = smem_desc(b0 + k * 32);
                    const unsigned accum = (kb > 0 || k > 0) ? 1u : 0u;
                    asm volatile(
                        "{\n\t.reg .pred p;\n\t"
                        "setp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                        "l"(ad), "l"(bd), "r"(IDESC), "r"(accum)
                        : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&bar_empty[s]))
                             : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(&bar_acc))
                         : "memory");
        }
    } else {
        // epilogue: warps 2..5 own TMEM lanes 32*(warp % 4) .. +31, i.e. tile rows
        const int q = warp & 3;
        const int row = m0 + q * 32 + lane;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_acc), 0u, &abort_flag));
        if (!ok) abort_flag = 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                unsigned r[16];
                const unsigned taddr = tmem + ((unsigned)(q * 32) << 16) + (unsigned)c;
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                    "%13, %14, %15}, [%16];"
                    : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                      "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                      "=r"(r[15])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                const int col = n0 + c;
                if (row < M) {
                    float *yr = y + (size_t)row * N + col;
                    if (col + 16 <= N && (N & 3) == 0) {
#pragma unroll
                        for (int j = 0; j < 16; j += 4) {
                            float4 v;
                            v.x = __uint_as_float(r[j]) + (bias ? __ldg(bias + col + j) : 0.f);
                            v.y = __uint_as_float(r[j + 1]) + (bias ? __ldg(bias + col + j + 1) : 0.f);
                            v.z = __uint_as_float(r[j + 2]) + (bias ? __ldg(bias + col + j + 2) : 0.f);
                            v.w = __uint_as_float(r[j + 3]) + (bias ? __ldg(bias + col + j + 3) : 0.f);
                            *reinterpret_cast<float4 *>(yr + j) = v;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (col + j < N) yr[j] = __uint_as_float(r[j]) + (bias ? __ldg(bias + col + j) : 0.f);
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
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

cudaError_t proj_launch(int x_dtype, const void *x, const void *W, const float *bias, float *y, int M, int K, int N,
                        int, cudaStream_t st, int *launches, int *sticky) {
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
    const int smem = gemm::STAGES * gemm::STAGE_BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(gemm::proj_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((M + gemm::BM - 1) / gemm::BM, (N + gemm::BN - 1) / gemm::BN);
    gemm::proj_bf16_kernel<<<grid, gemm::THREADS, smem, st>>>(ta, tb, bias, y, M, N, K, sticky);
    *launches = 1;
    return cudaGetLastError();
}

}  // namespace prn
