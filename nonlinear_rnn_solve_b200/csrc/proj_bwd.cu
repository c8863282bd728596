// proj_bwd.cu -- the reverse pass of the input projection xproj = x W^T + bias: for
// L = <grad_xproj, xproj>, grad_x = grad_xproj W, grad_W = grad_xproj^T x and
// grad_bias = the column sums of grad_xproj.  With the adjoint of the recurrence
// (adjoint.cu) this completes the gradient of a trainable layer ("Para-Seq" README,
// Main features: GRU/LSTM layers trained with the parallel solver and an adjoint
// backward).
//
// bf16 path (x, W bf16; tcgen05 tensor cores): grad_xproj is rounded to bf16 (nearest,
// ties to even) once, into a row-major copy and a transposed copy, while its column
// sums are taken in fp32; x and W are transposed once; then both products run on the
// projection GEMM of proj.cu, which contracts two K-major operands:
//   grad_x [M, K] = gx_bf16 [M, N] . (W^T [K, N])^T      (contraction over N)
//   grad_W [N, K] = gx_bf16^T [N, M] . (x^T [K, M])^T    (contraction over M)
// fp32 path (x, W fp32): CUDA-core products on strided operands, no copies.
// The bias gradient is summed per block of rows and then over blocks, in a fixed
// order (deterministic).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/pararnn.h"
#include "common.cuh"
#include "internal.h"

namespace prn {

namespace {

constexpr int TT = 64;  // transpose / conversion tile (TT x TT)

__device__ __forceinline__ unsigned short bf16_bits_rne(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// One CTA per (column tile, block of `rpb` rows) of gx [M, N]: column sums into
// part[row block][N]; with WRITE, also the bf16 copies gb [M, N] and gbt [N, M].
template <bool WRITE>
__global__ void __launch_bounds__(256) gx_prep_kernel(const float *__restrict__ gx, unsigned short *__restrict__ gb,
                                                      unsigned short *__restrict__ gbt, float *__restrict__ part,
                                                      int M, int N, int rpb) {
    __shared__ unsigned short tile[TT][TT + 2];
    __shared__ float colsum[16][TT];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;  // 4 columns x rows ty, ty + 16, ...
    const int n0 = blockIdx.x * TT;
    const int r_begin = blockIdx.y * rpb, r_end = min(M, r_begin + rpb);
    float cs[4] = {0.f, 0.f, 0.f, 0.f};
    for (int m0 = r_begin; m0 < r_end; m0 += TT) {
#pragma unroll
        for (int i = 0; i < TT / 16; ++i) {
            const int r = ty + 16 * i, m = m0 + r;
            float v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                v[j] = (m < r_end && n < N) ? gx[(size_t)m * N + n] : 0.f;
                cs[j] += v[j];
            }
            if (WRITE) {
                unsigned short h[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    h[j] = bf16_bits_rne(v[j]);
                    tile[r][tx * 4 + j] = h[j];
                }
                if (m < r_end) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (n0 + tx * 4 + j < N) gb[(size_t)m * N + n0 + tx * 4 + j] = h[j];
                }
            }
        }
        if (WRITE) {
            __syncthreads();
            // transposed tile: row n of gbt takes this tile's rows m0 .. m0 + TT - 1
            for (int e = threadIdx.x; e < TT * TT; e += 256) {
                const int c = e / TT, r = e % TT;  // consecutive threads: consecutive m
                const int n = n0 + c, m = m0 + r;
                if (n < N && m < r_end) gbt[(size_t)n * M + m] = tile[r][c];
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) colsum[ty][tx * 4 + j] = cs[j];
    __syncthreads();
    if (threadIdx.x < TT && n0 + threadIdx.x < N) {
        float acc = 0.f;
        for (int i = 0; i < 16; ++i) acc += colsum[i][threadIdx.x];
        part[(size_t)blockIdx.y * N + n0 + threadIdx.x] = acc;
    }
}

__global__ void colsum_reduce_kernel(const float *__restrict__ part, float *__restrict__ out, int R, int N) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float acc = 0.f;
    for (int r = 0; r < R; ++r) acc += part[(size_t)r * N + n];
    out[n] = acc;
}

// at [C, R] = a [R, C]^T, bf16 bit patterns, TT x TT tiles through shared memory.
__global__ void __launch_bounds__(256) transpose_u16_kernel(const unsigned short *__restrict__ a,
                                                            unsigned short *__restrict__ at, int R, int C) {
    __shared__ unsigned short tile[TT][TT + 2];
    const int r0 = blockIdx.x * TT, c0 = blockIdx.y * TT;  // row tiles on x: no 65535 limit
    for (int e = threadIdx.x; e < TT * TT; e += 256) {
        const int r = e / TT, c = e % TT;
        tile[r][c] = (r0 + r < R && c0 + c < C) ? a[(size_t)(r0 + r) * C + c0 + c] : (unsigned short)0;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < TT * TT; e += 256) {
        const int c = e / TT, r = e % TT;
        if (c0 + c < C && r0 + r < R) at[(size_t)(c0 + c) * R + r0 + r] = tile[r][c];
    }
}

// The same for R and C multiples of 4 (every bf16 operand here): 8-byte loads and stores,
// a warp moving two 128-byte row pieces per access.  Lane l of a store takes column
// c = 2 w + l / 16 (w the warp's pair) and rows 4 (l % 16) .. + 3 of the tile, read
// from shared memory with a row pitch of 33 words (two-way conflicts at most).
__global__ void __launch_bounds__(256) transpose_u16x4_kernel(const unsigned short *__restrict__ a,
                                                              unsigned short *__restrict__ at, int R, int C) {
    __shared__ unsigned short tile[TT][TT + 2];
    const int r0 = blockIdx.x * TT, c0 = blockIdx.y * TT;  // row tiles on x: no 65535 limit
    for (int e = threadIdx.x; e < TT * TT / 4; e += 256) {
        const int r = e / (TT / 4), c = 4 * (e % (TT / 4));
        uint2 v = make_uint2(0u, 0u);
        if (r0 + r < R && c0 + c < C) v = *reinterpret_cast<const uint2 *>(a + (size_t)(r0 + r) * C + c0 + c);
        unsigned *d = reinterpret_cast<unsigned *>(&tile[r][c]);  // 4-byte aligned: even pitch, c % 4 == 0
        d[0] = v.x;
        d[1] = v.y;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < TT * TT / 4; e += 256) {
        const int c = e / (TT / 4), r = 4 * (e % (TT / 4));
        if (c0 + c < C && r0 + r < R) {
            const unsigned lo = tile[r][c] | ((unsigned)tile[r + 1][c] << 16);
            const unsigned hi = tile[r + 2][c] | ((unsigned)tile[r + 3][c] << 16);
            *reinterpret_cast<uint2 *>(at + (size_t)(c0 + c) * R + r0 + r) = make_uint2(lo, hi);
        }
    }
}

// at = a^T with the vector kernel when the rows allow it
void transpose_u16(const unsigned short *a, unsigned short *at, int R, int C, cudaStream_t st) {
    const dim3 grid((R + TT - 1) / TT, (C + TT - 1) / TT);
    if (R % 4 == 0 && C % 4 == 0 && ((uintptr_t)a & 7) == 0 && ((uintptr_t)at & 7) == 0)
        transpose_u16x4_kernel<<<grid, 256, 0, st>>>(a, at, R, C);
    else
        transpose_u16_kernel<<<grid, 256, 0, st>>>(a, at, R, C);
}

// fp32 C [M, N] = sum_k A(m, k) B(n, k) with A(m, k) = A[m sam + k sak] and
// B(n, k) = B[n sbn + k sbk]: 64 x 64 tile per CTA, 4 x 4 outputs per thread.
__global__ void __launch_bounds__(256) gemm_f32_strided_kernel(const float *__restrict__ A, long sam, long sak,
                                                               const float *__restrict__ B, long sbn, long sbk,
                                                               float *__restrict__ Cm, int M, int N, int K) {
    __shared__ float as[16][64 + 4], bs[16][64 + 4];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int m0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int e = threadIdx.x; e < 16 * 64; e += 256) {
            // k fastest when the operand is k-contiguous, row fastest otherwise
            const int ka = sak == 1 ? e % 16 : e / 64, ra = sak == 1 ? e / 16 : e % 64;
            const int kb = sbk == 1 ? e % 16 : e / 64, rb = sbk == 1 ? e / 16 : e % 64;
            as[ka][ra] = (m0 + ra < M && k0 + ka < K) ? A[(m0 + ra) * sam + (k0 + ka) * sak] : 0.f;
            bs[kb][rb] = (n0 + rb < N && k0 + kb < K) ? B[(n0 + rb) * sbn + (k0 + kb) * sbk] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = as[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = bs[kk][tx * 4 + j];
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
            if (n < N) Cm[(size_t)m * N + n] = acc[i][j];
        }
    }
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

int row_blocks(int M) {
    // enough CTAs to fill the GPU for the column sums, each covering whole TT-row tiles
    const int tiles = (M + TT - 1) / TT;
    return std::max(1, std::min(tiles, 64));
}

// grad_x = gb W and grad_W = gbt x on the tensor cores, from the bf16 copies gb [M, N]
// and gbt [N, M] already in the scratch (layout: column-sum parts, gb, gbt, x^T, W^T,
// K-split parts of grad_W).
cudaError_t bf16_products(const void *x, const void *W, float *grad_x, float *grad_W, int M, int K, int N,
                          void *scratch, int num_sms, cudaStream_t st, int *launches, int *sticky) {
    *launches = 0;
    char *ws = static_cast<char *>(scratch) + up256((size_t)row_blocks(M) * N * sizeof(float));
    const unsigned short *gb = reinterpret_cast<const unsigned short *>(ws);
    ws += up256((size_t)M * N * 2);
    const unsigned short *gbt = reinterpret_cast<const unsigned short *>(ws);
    ws += up256((size_t)M * N * 2);
    unsigned short *xT = reinterpret_cast<unsigned short *>(ws);
    ws += up256((size_t)M * K * 2);
    unsigned short *WT = reinterpret_cast<unsigned short *>(ws);
    ws += up256((size_t)N * K * 2);
    float *kws = reinterpret_cast<float *>(ws);  // K-split parts of grad_W
    cudaError_t e;
    int l = 0;
    if (grad_x) {
        transpose_u16(static_cast<const unsigned short *>(W), WT, N, K, st);
        ++*launches;
        if ((e = proj_launch(PARARNN_BF16, gb, WT, nullptr, grad_x, M, N, K, num_sms, st, &l, sticky)) != cudaSuccess)
            return e;
        *launches += l;
    }
    if (grad_W) {
        transpose_u16(static_cast<const unsigned short *>(x), xT, M, K, st);
        ++*launches;
        // an N x K output over a long contraction (M): few tiles, so the K blocks may be
        // split across more CTAs and the parts summed in order
        if ((e = proj_launch_split(PARARNN_BF16, gbt, xT, nullptr, grad_W, N, M, K, num_sms, st, &l, sticky, kws,
                                   (size_t)kMaxKsplit * N * K)) != cudaSuccess)
            return e;
        *launches += l;
    }
    return cudaGetLastError();
}

}  // namespace

size_t proj_bwd_scratch_bytes(int x_dtype, int M, int K, int N) {
    const size_t part = up256((size_t)row_blocks(M) * N * sizeof(float));
    if (x_dtype != PARARNN_BF16) return part;
    // + the parts of a K-split grad_W product (N x K each)
    return part + 2 * up256((size_t)M * N * 2) + up256((size_t)M * K * 2) + up256((size_t)N * K * 2) +
           up256((size_t)kMaxKsplit * N * K * sizeof(float));
}

int proj_bwd_check(int x_dtype, int M, int K, int N) {
    // bf16: every operand of the two products has rows of a multiple of 8 elements
    // (16-byte pitch for the tensor-memory copies)
    if (x_dtype == PARARNN_BF16 && (M % 8 || K % 8 || N % 8)) return PARARNN_EINVAL;
    if ((long long)M * N > (1ll << 40) || (long long)M * K > (1ll << 40)) return PARARNN_EINVAL;
    return PARARNN_OK;
}

cudaError_t proj_bwd_launch(int x_dtype, const float *gx, const void *x, const void *W, float *grad_x, float *grad_W,
                            float *grad_bias, int M, int K, int N, void *scratch, int num_sms, cudaStream_t st,
                            int *launches, int *sticky) {
    *launches = 0;
    char *ws = static_cast<char *>(scratch);
    const int R = row_blocks(M);
    float *part = reinterpret_cast<float *>(ws);
    ws += up256((size_t)R * N * sizeof(float));
    const int rpb = ((M + R - 1) / R + TT - 1) / TT * TT;
    const dim3 prep_grid((N + TT - 1) / TT, R);
    cudaError_t e;
    if (x_dtype == PARARNN_F32) {
        if (grad_bias) {
            gx_prep_kernel<false><<<prep_grid, 256, 0, st>>>(gx, nullptr, nullptr, part, M, N, rpb);
            colsum_reduce_kernel<<<(N + 255) / 256, 256, 0, st>>>(part, grad_bias, R, N);
            *launches += 2;
        }
        const float *xf = static_cast<const float *>(x), *Wf = static_cast<const float *>(W);
        if (grad_x) {  // grad_x[m, k] = sum_n gx[m, n] W[n, k]
            gemm_f32_strided_kernel<<<dim3((M + 63) / 64, (K + 63) / 64), 256, 0, st>>>(gx, N, 1, Wf, 1, K, grad_x, M,
                                                                                       K, N);
            ++*launches;
        }
        if (grad_W) {  // grad_W[n, k] = sum_m gx[m, n] x[m, k]
            gemm_f32_strided_kernel<<<dim3((N + 63) / 64, (K + 63) / 64), 256, 0, st>>>(gx, 1, N, xf, 1, K, grad_W, N,
                                                                                       K, M);
            ++*launches;
        }
        return cudaGetLastError();
    }
    unsigned short *gb = reinterpret_cast<unsigned short *>(ws);
    gx_prep_kernel<true><<<prep_grid, 256, 0, st>>>(gx, gb, gb + up256((size_t)M * N * 2) / 2, part, M, N, rpb);
    ++*launches;
    if (grad_bias) {
        colsum_reduce_kernel<<<(N + 255) / 256, 256, 0, st>>>(part, grad_bias, R, N);
        ++*launches;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int l = 0;
    e = bf16_products(x, W, grad_x, grad_W, M, K, N, scratch, num_sms, st, &l, sticky);
    *launches += l;
    return e;
}

unsigned short *proj_bwd_gb(void *scratch, int M, int N) {
    return reinterpret_cast<unsigned short *>(static_cast<char *>(scratch) +
                                              up256((size_t)row_blocks(M) * N * sizeof(float)));
}

unsigned short *proj_bwd_gbt(void *scratch, int M, int N) { return proj_bwd_gb(scratch, M, N) + up256((size_t)M * N * 2) / 2; }

cudaError_t proj_bwd_from_bf16_launch(const void *x, const void *W, float *grad_x, float *grad_W, int M, int K, int N,
                                      bool have_gbt, void *scratch, int num_sms, cudaStream_t st, int *launches,
                                      int *sticky) {
    *launches = 0;
    unsigned short *gb = proj_bwd_gb(scratch, M, N), *gbt = proj_bwd_gbt(scratch, M, N);
    if (grad_W && !have_gbt) {
        transpose_u16(gb, gbt, M, N, st);
        ++*launches;
    }
    int l = 0;
    const cudaError_t e = bf16_products(x, W, grad_x, grad_W, M, K, N, scratch, num_sms, st, &l, sticky);
    *launches += l;
    return e;
}

}  // namespace prn
