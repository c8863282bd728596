// api.cu -- the C ABI declared in include/pararnn.h: argument checks, the context's
// device workspace, and stream-ordered launches of the sm_100a kernels.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>

#include "../../include/pararnn.h"
#include "common.cuh"
#include "internal.h"

struct pararnn_ctx {
    int device = 0;
    cudaStream_t stream = nullptr;
    int num_sms = 0;
    void *ws = nullptr;        // workspace: control block, flags, aggregates, side buffers
    size_t ws_bytes = 0;
    void *scratch = nullptr;   // plain scratch of the projection backward (bf16 copies)
    size_t scratch_bytes = 0;
    int *sticky = nullptr;     // sticky device status word
    prn::DbgHost dbg;
    int last_launches = 0;
    unsigned long long epoch_next = 0;  // look-back epochs handed out so far
};

namespace {

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool misaligned(const void *p) { return p && ((uintptr_t)p & 15u); }

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Make the workspace at least `need` bytes (grows, never shrinks).
int ensure_ws(pararnn_ctx *ctx, size_t need) {
    if (ctx->ws_bytes >= need) return PARARNN_OK;
    if (ctx->ws) {
        if (cudaStreamSynchronize(ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
        cudaFree(ctx->ws);
        ctx->ws = nullptr;
        ctx->ws_bytes = 0;
    }
    size_t sz = std::max(need, (size_t)1 << 20);
    if (cudaMalloc(&ctx->ws, sz) != cudaSuccess) {
        cudaGetLastError();
        return PARARNN_ENOMEM;
    }
    if (cudaMemset(ctx->ws, 0, sz) != cudaSuccess) return PARARNN_ECUDA;
    ctx->ws_bytes = sz;
    return PARARNN_OK;
}

// Carve the workspace for a plan and zero the control block on the stream.  Layout:
// [control block | look-back aggregates | look-back inclusive values | side buffers].
// Look-back words carry the epoch that wrote them; every launch takes a fresh epoch
// range, and when the 32-bit range would wrap the look-back words are zeroed.
int prepare(pararnn_ctx *ctx, const prn::Plan &plan, prn::Work *w) {
    if (plan.ntiles > 0x7fffffffL) return PARARNN_EUNSUPPORTED;  // kernels number tiles in 32 bits
    const size_t ctl_b = up256(sizeof(prn::Ctl));
    const size_t ag_b = up256(plan.agg_words * 8), in_b = up256(plan.inc_words * 8), sd_b = up256(plan.side_bytes);
    int rc = ensure_ws(ctx, ctl_b + ag_b + in_b + sd_b);
    if (rc) return rc;
    char *base = static_cast<char *>(ctx->ws);
    w->ctl = reinterpret_cast<prn::Ctl *>(base);
    w->agg = reinterpret_cast<unsigned long long *>(base + ctl_b);
    w->inc = reinterpret_cast<unsigned long long *>(base + ctl_b + ag_b);
    w->side = reinterpret_cast<float *>(base + ctl_b + ag_b + in_b);
    w->sticky = ctx->sticky;
    if (ctx->epoch_next + plan.epochs + 2 >= 0xffffffffull) {
        if (cudaMemsetAsync(base + ctl_b, 0, ctx->ws_bytes - ctl_b, ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
        ctx->epoch_next = 0;
    }
    w->epoch0 = (unsigned)ctx->epoch_next;
    ctx->epoch_next += plan.epochs;
    if (cudaMemsetAsync(base, 0, ctl_b, ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
    return PARARNN_OK;
}

// Make the plain scratch buffer at least `need` bytes (grows, never shrinks).
int ensure_scratch(pararnn_ctx *ctx, size_t need) {
    if (ctx->scratch_bytes >= need) return PARARNN_OK;
    if (ctx->scratch) {
        if (cudaStreamSynchronize(ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
        cudaFree(ctx->scratch);
        ctx->scratch = nullptr;
        ctx->scratch_bytes = 0;
    }
    if (cudaMalloc(&ctx->scratch, need) != cudaSuccess) {
        cudaGetLastError();
        return PARARNN_ENOMEM;
    }
    ctx->scratch_bytes = need;
    return PARARNN_OK;
}

int cuda_rc(cudaError_t e) {
    if (e == cudaSuccess) return PARARNN_OK;
    cudaGetLastError();
    return PARARNN_ECUDA;
}

}  // namespace

extern "C" {

int pararnn_create(pararnn_ctx **out, int device, void *cuda_stream) {
    if (!out) return PARARNN_EINVAL;
    *out = nullptr;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
        cudaGetLastError();
        return ndev > 0 ? PARARNN_EINVAL : PARARNN_ECUDA;
    }
    DeviceGuard g(device);
    if (!g.ok) return PARARNN_ECUDA;
    pararnn_ctx *ctx = new pararnn_ctx();
    ctx->device = device;
    ctx->stream = static_cast<cudaStream_t>(cuda_stream);
    if (cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
        cudaMalloc(&ctx->sticky, 256) != cudaSuccess || cudaMemset(ctx->sticky, 0, 256) != cudaSuccess) {
        cudaGetLastError();
        if (ctx->sticky) cudaFree(ctx->sticky);
        delete ctx;
        return PARARNN_ECUDA;
    }
    *out = ctx;
    return PARARNN_OK;
}

int pararnn_destroy(pararnn_ctx *ctx) {
    if (!ctx) return PARARNN_EINVAL;
    DeviceGuard g(ctx->device);
    cudaStreamSynchronize(ctx->stream);
    if (ctx->ws) cudaFree(ctx->ws);
    if (ctx->scratch) cudaFree(ctx->scratch);
    if (ctx->sticky) cudaFree(ctx->sticky);
    delete ctx;
    return PARARNN_OK;
}

int pararnn_set_stream(pararnn_ctx *ctx, void *cuda_stream) {
    if (!ctx) return PARARNN_EINVAL;
    ctx->stream = static_cast<cudaStream_t>(cuda_stream);
    return PARARNN_OK;
}

int pararnn_newton_forward(pararnn_ctx *ctx, const float *xproj, const pararnn_params *p, const float *h0,
                           float *h_out, int max_iters, float tol, int *iters_out, float *final_delta_out,
                           float *residual_out) {
    if (!ctx || !p || !h_out || !iters_out) return PARARNN_EINVAL;
    if (p->B < 1 || p->T < 1 || p->H < 1 || max_iters < 0 || max_iters > (1 << 30)) return PARARNN_EINVAL;
    if (!(tol == tol)) return PARARNN_EINVAL;
    if (p->solver < PARARNN_SOLVER_NEWTON || p->solver > PARARNN_SOLVER_ELK) return PARARNN_EINVAL;
    if (p->solver == PARARNN_SOLVER_ELK && !(p->damping >= 0.f && p->damping < 3.0e38f)) return PARARNN_EINVAL;
    // linearisation of the fixed-point scheme: zero (Jacobi), identity (Picard), else the cell's
    const int jm_solver = p->solver == PARARNN_SOLVER_JACOBI ? 2 : p->solver == PARARNN_SOLVER_PICARD ? 3 : 0;
    const bool fused = xproj == nullptr;
    if (fused && (!p->x || !p->W || p->in < 1 || p->in > 8)) return PARARNN_EINVAL;
    if (misaligned(xproj) || misaligned(h_out) || misaligned(h0) || (fused && misaligned(p->x)))
        return PARARNN_EALIGN;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    ctx->last_launches = 0;
    prn::Plan plan;
    prn::Work w;
    int rc;
    if (p->cell == PARARNN_GRU_DIAG || p->cell == PARARNN_LSTM_CIFG_PEEP || p->cell == PARARNN_LSTM_CIFG_PEEP_QUASI) {
        const int lstm = p->cell != PARARNN_GRU_DIAG;
        const int jmode = jm_solver ? jm_solver : (p->cell == PARARNN_LSTM_CIFG_PEEP_QUASI ? 1 : 0);
        if (!p->a || (lstm && !p->peep)) return PARARNN_EINVAL;
        prn::NewtonDiagReq r{lstm, jmode, p->B, p->T, p->H, p->in, xproj, p->x, p->W, p->bias, p->a, p->peep, h0, h_out,
                             max_iters, tol, iters_out, final_delta_out, residual_out, ctx->dbg.wide_variant};
        const bool elk = p->solver == PARARNN_SOLVER_ELK;
        if ((elk ? prn::elk_plan(r, ctx->num_sms, &plan) : prn::newton_diag_plan(r, ctx->num_sms, &plan)))
            return PARARNN_ECUDA;
        if ((rc = prepare(ctx, plan, &w))) return rc;
        if (max_iters == 0) {
            const size_t n = (size_t)p->B * p->T * p->H * (lstm ? 2 : 1);
            if (cudaMemsetAsync(h_out, 0, n * sizeof(float), ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
        }
        rc = cuda_rc(elk ? prn::elk_launch(r, p->damping, plan, w, ctx->dbg, ctx->stream)
                         : prn::newton_diag_launch(r, plan, w, ctx->dbg, ctx->stream));
    } else if (p->cell == PARARNN_RNN_TANH_DENSE || p->cell == PARARNN_RNN_TANH_QUASI) {
        if (!p->A) return PARARNN_EINVAL;
        if (p->H > 64) return PARARNN_EUNSUPPORTED;
        // Jacobi and Picard have diagonal linearisations: they run on the quasi (diagonal)
        // kernel; ELK takes the diagonal of the Jacobian for either cell (quasi-ELK)
        const bool elk = p->solver == PARARNN_SOLVER_ELK;
        const int quasi = p->cell == PARARNN_RNN_TANH_QUASI || jm_solver != 0;
        prn::NewtonTanhReq r{quasi, jm_solver, p->B, p->T, p->H, p->in, xproj, p->x, p->W,
                             p->bias, p->A, h0, h_out, max_iters, tol, iters_out, final_delta_out, residual_out};
        int prc = elk ? prn::elk_tanh_plan(r, ctx->num_sms, &plan) : prn::newton_tanh_plan(r, ctx->num_sms, &plan);
        if (prc == 1) return PARARNN_EUNSUPPORTED;
        if (prc) return PARARNN_ECUDA;
        if ((rc = prepare(ctx, plan, &w))) return rc;
        if (max_iters == 0) {
            const size_t n = (size_t)p->B * p->T * p->H;
            if (cudaMemsetAsync(h_out, 0, n * sizeof(float), ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
        }
        rc = cuda_rc(elk ? prn::elk_tanh_launch(r, p->damping, plan, w, ctx->dbg, ctx->stream)
                         : prn::newton_tanh_launch(r, plan, w, ctx->dbg, ctx->stream));
    } else {
        return PARARNN_EINVAL;
    }
    if (rc == PARARNN_OK) ctx->last_launches = 1;
    return rc;
}

int pararnn_linear_scan(pararnn_ctx *ctx, int kind, const float *J, const float *b, const float *h0, float *h_out,
                        int B, int T, int N, int reverse) {
    if (!ctx || !J || !b || !h_out) return PARARNN_EINVAL;
    if (B < 1 || T < 1 || N < 1 || (reverse != 0 && reverse != 1)) return PARARNN_EINVAL;
    if (kind != PARARNN_SCAN_DIAG && kind != PARARNN_SCAN_BLOCK2 && kind != PARARNN_SCAN_DENSE)
        return PARARNN_EINVAL;
    if (kind == PARARNN_SCAN_DENSE && N > 64) return PARARNN_EUNSUPPORTED;
    if (misaligned(J) || misaligned(b) || misaligned(h0) || misaligned(h_out)) return PARARNN_EALIGN;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    ctx->last_launches = 0;
    prn::ScanReq r{kind, B, T, N, reverse, J, b, h0, h_out};
    prn::Plan plan;
    prn::Work w;
    int rc;
    if (kind == PARARNN_SCAN_DENSE) {
        int prc = prn::scan_dense_plan(r, ctx->num_sms, &plan);
        if (prc == 1) return PARARNN_EUNSUPPORTED;
        if (prc) return PARARNN_ECUDA;
        if ((rc = prepare(ctx, plan, &w))) return rc;
        rc = cuda_rc(prn::scan_dense_launch(r, plan, w, ctx->dbg, ctx->stream));
    } else {
        if (prn::scan_diag_plan(r, ctx->num_sms, &plan)) return PARARNN_ECUDA;
        if ((rc = prepare(ctx, plan, &w))) return rc;
        rc = cuda_rc(prn::scan_diag_launch(r, plan, w, ctx->dbg, ctx->stream));
    }
    if (rc == PARARNN_OK) ctx->last_launches = 1;
    return rc;
}

int pararnn_adjoint_backward(pararnn_ctx *ctx, const float *xproj, const pararnn_params *p, const float *h0,
                             const float *h, const float *grad_h, float *grad_xproj, float *grad_params,
                             float *grad_h0) {
    if (!ctx || !p || !xproj || !h || !grad_h || !grad_xproj || !grad_params) return PARARNN_EINVAL;
    if (p->B < 1 || p->T < 1 || p->H < 1) return PARARNN_EINVAL;
    // the quasi backend changes the iteration only: the adjoint at the solution is the
    // exact-Jacobian one for both LSTM cells
    if (p->cell != PARARNN_GRU_DIAG && p->cell != PARARNN_LSTM_CIFG_PEEP && p->cell != PARARNN_LSTM_CIFG_PEEP_QUASI)
        return PARARNN_EUNSUPPORTED;
    const int lstm = p->cell != PARARNN_GRU_DIAG;
    if (!p->a || (lstm && !p->peep)) return PARARNN_EINVAL;
    if (misaligned(xproj) || misaligned(h) || misaligned(grad_h) || misaligned(grad_xproj) || misaligned(h0) ||
        misaligned(grad_h0))
        return PARARNN_EALIGN;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    ctx->last_launches = 0;
    prn::AdjointReq r{lstm, p->B, p->T, p->H, xproj, p->a, p->peep, h0, h, grad_h, grad_xproj, grad_params, grad_h0};
    prn::Plan plan;
    prn::Work w;
    int rc;
    if (prn::adjoint_plan(r, ctx->num_sms, &plan)) return PARARNN_ECUDA;
    if ((rc = prepare(ctx, plan, &w))) return rc;
    const size_t np = (size_t)(lstm ? 5 : 3) * p->H;
    if (cudaMemsetAsync(grad_params, 0, np * sizeof(float), ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
    rc = cuda_rc(prn::adjoint_launch(r, plan, w, ctx->dbg, ctx->stream));
    if (rc == PARARNN_OK) ctx->last_launches = 1;
    return rc;
}

int pararnn_layer_backward(pararnn_ctx *ctx, const float *xproj, const pararnn_params *p, const float *h0,
                           const float *h, const float *grad_h, const void *x, const void *W, int K, float *grad_x,
                           float *grad_W, float *grad_bias, float *grad_params, float *grad_h0) {
    if (!ctx || !p || !xproj || !h || !grad_h || !x || !W || !grad_params || K < 1) return PARARNN_EINVAL;
    if (p->B < 1 || p->T < 1 || p->H < 1) return PARARNN_EINVAL;
    if (p->cell != PARARNN_GRU_DIAG && p->cell != PARARNN_LSTM_CIFG_PEEP && p->cell != PARARNN_LSTM_CIFG_PEEP_QUASI)
        return PARARNN_EUNSUPPORTED;
    const int lstm = p->cell != PARARNN_GRU_DIAG;
    if (!p->a || (lstm && !p->peep)) return PARARNN_EINVAL;
    if ((long long)p->B * p->T > 0x7fffffffLL || 3LL * p->H > 0x7fffffffLL) return PARARNN_EINVAL;
    const int M = p->B * p->T, N = 3 * p->H;
    if (int chk = prn::proj_bwd_check(PARARNN_BF16, M, K, N)) return chk;
    if (misaligned(xproj) || misaligned(h) || misaligned(grad_h) || misaligned(h0) || misaligned(grad_h0) ||
        misaligned(x) || misaligned(W) || misaligned(grad_x) || misaligned(grad_W) || misaligned(grad_bias))
        return PARARNN_EALIGN;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    ctx->last_launches = 0;
    prn::AdjointReq r{lstm, p->B, p->T, p->H, xproj, p->a, p->peep, h0, h, grad_h, nullptr, grad_params, grad_h0};
    prn::Plan plan;
    // the adjoint writes bf16 grad_xproj straight into the projection's scratch when its
    // TMA-fed tiles cover the shape; otherwise fp32 grad_xproj goes through the scratch
    r.out_bf16 = true;
    const int wide = prn::adjoint_wide_plan(r, ctx->num_sms, &plan);
    if (wide < 0) return PARARNN_ECUDA;
    const size_t pbytes = prn::proj_bwd_scratch_bytes(PARARNN_BF16, M, K, N);
    int rc = ensure_scratch(ctx, pbytes + (wide ? (size_t)M * N * sizeof(float) : 0));
    if (rc) return rc;
    bool have_gbt = false;
    if (wide == 0) {
        r.grad_xproj_bf16 = prn::proj_bwd_gb(ctx->scratch, M, N);
        r.grad_bias = grad_bias;
        // ParaGRU: the adjoint also writes the transposed copy that grad_W's product reads
        have_gbt = grad_W && prn::adjoint_wide_writes_transpose(r);
        if (have_gbt) r.grad_xproj_bf16_t = prn::proj_bwd_gbt(ctx->scratch, M, N);
    } else {
        r.out_bf16 = false;
        r.grad_xproj = reinterpret_cast<float *>(static_cast<char *>(ctx->scratch) + pbytes);
        if (prn::adjoint_plan(r, ctx->num_sms, &plan)) return PARARNN_ECUDA;
    }
    prn::Work w;
    if ((rc = prepare(ctx, plan, &w))) return rc;
    const size_t np = (size_t)(lstm ? 5 : 3) * p->H;
    if (cudaMemsetAsync(grad_params, 0, np * sizeof(float), ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
    int launches = 1;
    if (wide == 0 && grad_bias) {
        if (cudaMemsetAsync(grad_bias, 0, (size_t)N * sizeof(float), ctx->stream) != cudaSuccess) return PARARNN_ECUDA;
    }
    if ((rc = cuda_rc(prn::adjoint_launch(r, plan, w, ctx->dbg, ctx->stream)))) return rc;
    int l = 0;
    if (wide == 0)
        rc = cuda_rc(prn::proj_bwd_from_bf16_launch(x, W, grad_x, grad_W, M, K, N, have_gbt, ctx->scratch,
                                                    ctx->num_sms, ctx->stream, &l, ctx->sticky));
    else
        rc = cuda_rc(prn::proj_bwd_launch(PARARNN_BF16, r.grad_xproj, x, W, grad_x, grad_W, grad_bias, M, K, N,
                                          ctx->scratch, ctx->num_sms, ctx->stream, &l, ctx->sticky));
    if (rc == PARARNN_OK) ctx->last_launches = launches + l;
    return rc;
}

int pararnn_input_proj(pararnn_ctx *ctx, const void *x, int x_dtype, const void *W, const float *bias,
                       float *xproj, int M, int K, int N) {
    if (!ctx || !x || !W || !xproj || M < 1 || K < 1 || N < 1) return PARARNN_EINVAL;
    if (x_dtype != PARARNN_F32 && x_dtype != PARARNN_BF16) return PARARNN_EINVAL;
    if (misaligned(x) || misaligned(W) || misaligned(xproj) || misaligned(bias)) return PARARNN_EALIGN;
    int chk = prn::proj_check(x_dtype, M, K, N);
    if (chk) return chk;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    ctx->last_launches = 0;
    int launches = 0;
    int rc = cuda_rc(prn::proj_launch(x_dtype, x, W, bias, xproj, M, K, N, ctx->num_sms, ctx->stream, &launches, ctx->sticky));
    if (rc == PARARNN_OK) ctx->last_launches = launches;
    return rc;
}

int pararnn_input_proj_backward(pararnn_ctx *ctx, const float *grad_xproj, const void *x, int x_dtype, const void *W,
                                float *grad_x, float *grad_W, float *grad_bias, int M, int K, int N) {
    if (!ctx || !grad_xproj || !x || !W || M < 1 || K < 1 || N < 1) return PARARNN_EINVAL;
    if (x_dtype != PARARNN_F32 && x_dtype != PARARNN_BF16) return PARARNN_EINVAL;
    if (misaligned(grad_xproj) || misaligned(x) || misaligned(W) || misaligned(grad_x) || misaligned(grad_W) ||
        misaligned(grad_bias))
        return PARARNN_EALIGN;
    int chk = prn::proj_bwd_check(x_dtype, M, K, N);
    if (chk) return chk;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    ctx->last_launches = 0;
    // a buffer of its own: the look-back workspace must only ever hold epoch-tagged words
    int rc0 = ensure_scratch(ctx, prn::proj_bwd_scratch_bytes(x_dtype, M, K, N));
    if (rc0) return rc0;
    int launches = 0;
    int rc = cuda_rc(prn::proj_bwd_launch(x_dtype, grad_xproj, x, W, grad_x, grad_W, grad_bias, M, K, N, ctx->scratch,
                                          ctx->num_sms, ctx->stream, &launches, ctx->sticky));
    if (rc == PARARNN_OK) ctx->last_launches = launches;
    return rc;
}

int pararnn_lsim(pararnn_ctx *ctx, const float *A, const float *Bm, const float *C, const float *D, int n, int m, int p,
                 const float *U, const float *x0, double dt, int interp, int batch, int T, float *y_out,
                 float *x_out) {
    if (!ctx || !A || !Bm || !C || !U || !y_out) return PARARNN_EINVAL;
    prn::LsimReq r{A, Bm, C, D, n, m, p, U, x0, dt, interp, batch, T, y_out, x_out};
    if (prn::lsim_check(r)) return PARARNN_EINVAL;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    ctx->last_launches = 0;
    int rc = ensure_scratch(ctx, prn::lsim_scratch_bytes(r));
    if (rc) return rc;
    int launches = 0;
    rc = cuda_rc(prn::lsim_launch(r, static_cast<float *>(ctx->scratch), ctx->stream, &launches));
    if (rc == PARARNN_OK) ctx->last_launches = launches;
    return rc;
}

int pararnn_get_status(pararnn_ctx *ctx, int *device_status) {
    if (!ctx || !device_status) return PARARNN_EINVAL;
    DeviceGuard g(ctx->device);
    if (!g.ok) return PARARNN_ECUDA;
    if (cudaStreamSynchronize(ctx->stream) != cudaSuccess) return cuda_rc(cudaGetLastError());
    int v = 0;
    if (cudaMemcpy(&v, ctx->sticky, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PARARNN_ECUDA;
    if (cudaMemset(ctx->sticky, 0, sizeof(int)) != cudaSuccess) return PARARNN_ECUDA;
    if (v & prn::kStTimeout)
        *device_status = PARARNN_ETIMEOUT;
    else if (v & prn::kStNonfinite)
        *device_status = PARARNN_ENONFINITE;
    else if (v & prn::kStNotConverged)
        *device_status = PARARNN_NOTCONVERGED;
    else
        *device_status = PARARNN_OK;
    return PARARNN_OK;
}

const char *pararnn_strerror(int s) {
    switch (s) {
        case PARARNN_OK: return "ok";
        case PARARNN_NOTCONVERGED: return "not converged: iteration cap reached with delta >= tol";
        case PARARNN_EINVAL: return "invalid argument (null pointer, enum or shape)";
        case PARARNN_EALIGN: return "pointer not 16-byte aligned";
        case PARARNN_ECUDA: return "CUDA error";
        case PARARNN_ENOMEM: return "workspace allocation failed";
        case PARARNN_ENONFINITE: return "non-finite iterate or residual";
        case PARARNN_ETIMEOUT: return "bounded device wait ran out";
        case PARARNN_EUNSUPPORTED: return "unsupported configuration";
        case PARARNN_ESCRATCH: return "problem exceeds the static scratch of the allocation-free entry point";
        default: return "unknown status";
    }
}

int pararnn_debug_set(pararnn_ctx *ctx, int knob, long long value) {
    if (!ctx) return PARARNN_EINVAL;
    switch (knob) {
        case 1:
            if (value <= 0) return PARARNN_EINVAL;
            ctx->dbg.wait_ns = (unsigned long long)value;
            return PARARNN_OK;
        case 2: ctx->dbg.skip_tile = value; return PARARNN_OK;
        case 3: ctx->dbg.delta_log = reinterpret_cast<float *>((uintptr_t)value); return PARARNN_OK;
        case 4:
            if (value < 0) return PARARNN_EINVAL;
            ctx->dbg.delta_log_cap = (int)value;
            return PARARNN_OK;
        case 5: ctx->dbg.no_halo = value != 0; return PARARNN_OK;
        case 6:
            if (value != 0 && value != 8 && value != 16 && value != 32) return PARARNN_EINVAL;
            ctx->dbg.wide_variant = (int)value;
            return PARARNN_OK;
        default: return PARARNN_EINVAL;
    }
}

int pararnn_last_launch_count(pararnn_ctx *ctx) { return ctx ? ctx->last_launches : 0; }

}  // extern "C"
