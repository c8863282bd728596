/*
 * pararnn.h -- C ABI of the B200 (sm_100a) library that evaluates nonlinear RNNs
 * over the whole sequence at once with Newton (DEER) or quasi-Newton iterations.
 *
 * Method, as the pages describe it:
 *   - "Parallelizing non-linear sequential models over the sequence length"
 *     (Lim et al.), summary, "Approach": the recurrence is restated as a fixed-point
 *     problem solved by Newton's method; each iteration linearises the model with its
 *     Jacobians and solves the resulting linear recurrence with a parallel prefix scan.
 *   - "ParaRNN: Unlocking Parallel Training of Nonlinear RNNs for Large Language
 *     Models", abstract: the whole sequence is one system of equations solved with
 *     Newton's iterations and parallel reductions; GRU and LSTM adaptations.
 *   - "Towards Scalable and Stable Parallelization of Nonlinear RNNs", Abstract:
 *     quasi-Newton (diagonal Jacobian) variants converge comparably and cost less.
 *   - "Para-Seq" README, "Main features": diagonal ParaGRU, CIFG/peephole ParaLSTM with
 *     2x2 block scans, vanilla tanh RNN, dense/diagonal/2x2-block associative scans
 *     and reverse adjoint scans; "Quick example": batch-first tensors.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     batch-first, contiguous.  The library never frees or keeps them.
 *   - Calls are asynchronous and ordered on the context's stream; outputs are ready
 *     when that stream reaches the point of the call.  Device-side conditions
 *     (non-finite values, a bounded wait that ran out) are reported through
 *     pararnn_get_status.
 *   - Return value: PARARNN_OK (0) or a negative PARARNN_E* code; on an error
 *     nothing was enqueued.
 *   - Vector paths need 16-byte aligned base pointers (PARARNN_EALIGN otherwise).
 *   - A context owns only its device workspace (iteration bookkeeping, chunk
 *     aggregates for the scan's look-back); it grows on demand with cudaMalloc
 *     and is released by pararnn_destroy.  A context is not thread-safe; use one
 *     per host thread or stream.
 *
 * Shapes (G = 3 gates for GRU and LSTM, 1 for the tanh RNN; n = H for the tanh RNN):
 *   x      [B, T, in]          W   [G*H, in] (row g*H + u feeds gate g of unit u)
 *   xproj  [B, T, G, H] fp32   bias [G*H]
 *   GRU    state [B, T, H]      h0 [B, H]      a [3, H] = (a_z, a_r, a_c)
 *   LSTM   state [B, T, H, 2] as (c, h) pairs; h0 [B, H, 2]; a [3, H] = (a_f, a_g, a_o);
 *          peep [2, H] = (w_f, w_o)
 *   tanh   state [B, T, n]      h0 [B, n]      A [n, n] (A[i][j] multiplies h_j)
 * Output element t of the state is h_{t+1}; h0 is the state before the first step.
 */
#ifndef PARARNN_H
#define PARARNN_H

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------- */
#define PARARNN_OK 0
#define PARARNN_NOTCONVERGED 1   /* reported by get_status: the cap was reached with delta >= tol */
#define PARARNN_EINVAL (-1)      /* null pointer, bad enum or bad shape */
#define PARARNN_EALIGN (-2)      /* a pointer is not 16-byte aligned */
#define PARARNN_ECUDA (-3)       /* a CUDA call or launch failed */
#define PARARNN_ENOMEM (-4)      /* workspace allocation failed */
#define PARARNN_ENONFINITE (-5)  /* device: an iterate or residual became NaN or Inf */
#define PARARNN_ETIMEOUT (-6)    /* device: a bounded wait (look-back, grid barrier) ran out */
#define PARARNN_EUNSUPPORTED (-7) /* valid request outside what the library implements */

typedef enum {
    PARARNN_GRU_DIAG = 0,        /* diagonal ParaGRU, diagonal Jacobian */
    PARARNN_LSTM_CIFG_PEEP = 1,  /* CIFG + peephole ParaLSTM, 2x2 Jacobian per unit */
    PARARNN_RNN_TANH_DENSE = 2,  /* vanilla tanh RNN, full n x n Jacobian (DEER) */
    PARARNN_RNN_TANH_QUASI = 3,  /* vanilla tanh RNN, diagonal of the Jacobian (quasi-DEER) */
    PARARNN_LSTM_CIFG_PEEP_QUASI = 4 /* ParaLSTM with the diagonal scan backend: each 2x2 block
                                        replaced by its diagonal in the Newton iteration ("Para-Seq"
                                        README, Main features: structured block and diagonal scan
                                        backends); same fixed point, same adjoint */
} pararnn_cell;

typedef enum { PARARNN_SCAN_DIAG = 0, PARARNN_SCAN_BLOCK2 = 1, PARARNN_SCAN_DENSE = 2 } pararnn_scan_kind;

typedef enum { PARARNN_F32 = 0, PARARNN_BF16 = 1 } pararnn_dtype;

typedef struct pararnn_ctx pararnn_ctx;

/* Cell description and parameters (device pointers).  Unused fields may be NULL.
 * x/W/bias are read only when xproj is NULL ("fused projection", in <= 8): the
 * projection W x_t + bias is then recomputed inside the solver at every iteration
 * instead of being stored, which is cheaper for narrow inputs. */
typedef struct {
    int cell;              /* pararnn_cell */
    int B, T, H;           /* batch, steps, units (tanh RNN: state size n) */
    int in;                /* input width, fused projection only */
    const float *a;        /* [3, H]  GRU / LSTM recurrent diagonals */
    const float *peep;     /* [2, H]  LSTM peepholes */
    const float *A;        /* [n, n]  tanh RNN recurrent matrix */
    const float *x;        /* [B, T, in] fp32 (fused projection) */
    const float *W;        /* [G*H, in] fp32 (fused projection) */
    const float *bias;     /* [G*H] fp32 or NULL (fused projection) */
    int solver;            /* pararnn_solver (0 = Newton) */
    float damping;         /* ELK: Levenberg-Marquardt damping lambda >= 0 */
} pararnn_params;

/* Fixed-point scheme of pararnn_newton_forward ("Para-Seq" README, Main features:
 * sequential, Jacobi, Picard, DEER and quasi-DEER modes).  All share the loop
 * "linearise at h^(k), solve h^(k+1)_t = J_t h^(k+1)_{t-1} + f_t - J_t h^(k)_{t-1} by
 * scan" and differ in J_t: the cell's Jacobian (NEWTON; its diagonal for the *_QUASI
 * cells), zero (JACOBI: h^(k+1)_t = f(h^(k)_{t-1}), every step in parallel), or the
 * identity (PICARD: the increments f(h^(k)_{t-1}) - h^(k)_{t-1} are summed along t).
 * Every scheme reaches the rollout; after k iterations the first k states are exact. */
typedef enum {
    PARARNN_SOLVER_NEWTON = 0,
    PARARNN_SOLVER_JACOBI = 1,
    PARARNN_SOLVER_PICARD = 2,
    /* ELK ("Towards Scalable and Stable Parallelization of Nonlinear RNNs", Abstract):
     * the Levenberg-Marquardt step of the stacked system, i.e. the minimiser of
     * sum_t |x_t - J_t x_{t-1} - r_t|^2 + damping sum_t |x_t|^2 (x = h^(k+1) - h^(k),
     * r_t = f_t - h^(k)_t), computed by a parallel Kalman filter and smoother.  J_t is
     * the ParaGRU's diagonal Jacobian, the ParaLSTM's full 2x2 block per unit
     * (PARARNN_LSTM_CIFG_PEEP: ELK) or its diagonal (PARARNN_LSTM_CIFG_PEEP_QUASI:
     * quasi-ELK), and the diagonal of the tanh RNN's Jacobian (either tanh cell id,
     * n <= 64: quasi-ELK).  damping = 0 gives the undamped step of the same
     * linearisation; larger damping shortens the steps. */
    PARARNN_SOLVER_ELK = 3
} pararnn_solver;

/* Create a context on `device` that enqueues on `cuda_stream` (a cudaStream_t, or
 * NULL for the legacy default stream).  *ctx is NULL on failure. */
int pararnn_create(pararnn_ctx **ctx, int device, void *cuda_stream);
/* Synchronise the context's stream, free its workspace and the context. */
int pararnn_destroy(pararnn_ctx *ctx);
/* Change the stream later calls enqueue on. */
int pararnn_set_stream(pararnn_ctx *ctx, void *cuda_stream);

/* Input projection, the method's one dense contraction:
 *   xproj[m, n] = sum_k x[m, k] * W[n, k] + bias[n]      (M = B*T, N = G*H, K = in)
 * x [M, K] and W [N, K] are both bf16 (x_dtype = PARARNN_BF16, tcgen05 tensor cores,
 * fp32 accumulation) or both fp32 (PARARNN_F32, CUDA cores); bias fp32 [N] or NULL;
 * xproj fp32 [M, N].  Implied by the cells of the pages: the input term W x_t does
 * not depend on the state, so it is computed once per forward pass.
 * Shapes: any M, N >= 1; bf16 needs K % 8 == 0 (16-byte rows for the tensor-memory
 * copies), fp32 any K; M * N <= 2^40.  x, W, bias and xproj 16-byte aligned.
 * Returns EINVAL (null pointer, bad dtype or shape), EALIGN, or ECUDA (launch). */
int pararnn_input_proj(pararnn_ctx *ctx, const void *x, int x_dtype, const void *W,
                       const float *bias, float *xproj, int M, int K, int N);

/* Reverse pass of the input projection, for L = <grad_xproj, x W^T + bias>:
 *   grad_x [M, K] = grad_xproj [M, N] W,   grad_W [N, K] = grad_xproj^T x,
 *   grad_bias [N] = column sums of grad_xproj
 * (the projection is linear, so these are its exact gradients; with
 * pararnn_adjoint_backward they complete the gradient of a trainable layer:
 * "Para-Seq" README, Main features).  grad_xproj fp32 [M, N].  x and W as for
 * pararnn_input_proj: both bf16 (x_dtype PARARNN_BF16: grad_xproj is rounded to bf16,
 * nearest-even, for the tensor-core products, fp32 accumulation; the bias gradient
 * sums the fp32 values) or both fp32 (CUDA cores).  Each of grad_x, grad_W, grad_bias
 * may be NULL (not computed); outputs are overwritten, not accumulated.
 * Shapes: M, K, N >= 1; bf16 needs M, K, N multiples of 8 (16-byte rows of every
 * operand, including the transposed copies); M * N and M * K <= 2^40.  All pointers
 * 16-byte aligned.  The context keeps a scratch buffer of the bf16 copies
 * (4 M N + 2 M K + 2 N K bytes) and of the parts of a weight gradient whose product is
 * split along M (16 N K bytes; taken when grad_W has fewer 128 x 256 output tiles than
 * the GPU has SMs, the parts summed in a fixed order) for later calls.
 * Returns EINVAL, EALIGN, ENOMEM or ECUDA. */
int pararnn_input_proj_backward(pararnn_ctx *ctx, const float *grad_xproj, const void *x, int x_dtype,
                                const void *W, float *grad_x, float *grad_W, float *grad_bias, int M, int K,
                                int N);

/* Newton (DEER) / quasi-Newton forward solve of the whole sequence
 * ("Parallelizing non-linear sequential models over the sequence length", Approach;
 * quasi: "Towards Scalable and Stable Parallelization of Nonlinear RNNs", Abstract).
 * From the initial guess h^(0)_t = 0 (t >= 1), each iteration k evaluates the cell and
 * its Jacobian at every step from h^(k)_{t-1}, solves h^(k+1)_t = J_t h^(k+1)_{t-1} + b_t,
 * b_t = f_t - J_t h^(k)_{t-1}, and stops after the first iteration whose
 *   delta_k = max over all state elements |h^(k+1) - h^(k)|
 * is < tol (strict; tol <= 0 runs exactly max_iters iterations), or at max_iters.
 *   xproj      [B, T, G, H] projected inputs (bias included), or NULL to use p->x/W/bias
 *   h0         initial state, or NULL for zeros
 *   h_out      [B, T, H] (LSTM [B, T, H, 2]; tanh [B, T, n]) receives the final iterate
 *   iters_out  device int: number of Newton updates applied (counting the one whose
 *              delta fell below tol); max_iters = 0 leaves h_out = 0 and writes 0
 *   final_delta_out  device float or NULL: delta of the last iteration
 *   residual_out     device float or NULL: max |h_t - f(h_{t-1}, x_t)| at the result
 * Supported: GRU and LSTM any H; tanh RNN with n <= 64 (EUNSUPPORTED above), every
 * solver for every cell.  B, T >= 1.
 * Carries across tiles: the long-sequence tiles (ParaGRU with H = 1 and raw inputs; the
 * tanh RNN at n = 8 with inputs of width 4, quasi) first evaluate the steps just before
 * them (63 and 128) and, when every entry of those steps' composed Jacobian is at most
 * 2^-40 in magnitude, take that map's offset as the carry; the neglected term is at most
 * 2^-40 times the update entering those steps.  Otherwise, and in every other layout,
 * the carry is the scan's own (a look-back over the preceding tiles).  Debug knob 5
 * turns the first way off. */
int pararnn_newton_forward(pararnn_ctx *ctx, const float *xproj, const pararnn_params *p,
                           const float *h0, float *h_out, int max_iters, float tol,
                           int *iters_out, float *final_delta_out, float *residual_out);

/* Standalone linear recurrence by a chunked parallel scan
 * ("Para-Seq" README, Main features: dense, diagonal and 2x2 block associative scans,
 * plus reverse adjoint scans).
 *   forward (reverse = 0):  out_t = J_t out_{t-1} + b_t,        out_{-1} = h0 (or 0)
 *   reverse (reverse = 1):  out_t = b_t + J_{t+1}^T out_{t+1},  out_{T-1} = b_{T-1} + h0 (or 0)
 * kind DIAG:   J, b, out [B, T, N];             h0 [B, N]
 * kind BLOCK2: J [B, T, N, 2, 2] (row-major 2x2), b, out [B, T, N, 2]; h0 [B, N, 2]
 * kind DENSE:  J [B, T, N, N] (J[i][j] multiplies out_j), b, out [B, T, N]; h0 [B, N]; N <= 64 */
int pararnn_linear_scan(pararnn_ctx *ctx, int kind, const float *J, const float *b,
                        const float *h0, float *h_out, int B, int T, int N, int reverse);

/* Fixed-step simulation of the linear time-invariant system dx/dt = A x + B u,
 * y = C x + D u, by a chunked parallel scan ("Para-Seq" README, Quick example
 * `lsim(A, B, C, D, U, t)`, and the `src.ode_solvers` row of Main features; Notes and
 * limitations: fixed-step time grids only).  Samples t_k = t_0 + k dt, k = 0 .. T-1:
 *   x_0 = x0 (or 0),  x_k = Ad x_{k-1} + G0 u_{k-1} + G1 u_k,  y_k = C x_k + D u_k,
 * where one step of the ODE is solved exactly for an input held over the step
 * (interp = 0: Ad = e^{A dt}, G0 = int_0^dt e^{A s} ds B, G1 = 0) or varying linearly
 * between samples (interp = 1).  The discretisation runs on the device in fp64; the
 * recurrence in fp32.
 *   A [n, n], Bm [n, m], C [p, n], D [p, m] or NULL (no feedthrough): row-major, device
 *   U [batch, T, m];  x0 [batch, n] or NULL;  y_out [batch, T, p];  x_out [batch, T, n]
 *   or NULL (states not written).  All fp32 device pointers, caller-owned.
 * 1 <= n <= 32, 1 <= m <= 16, 1 <= p <= 32, batch >= 1, T >= 1, 0 < dt finite,
 * interp 0 or 1.  The context keeps a scratch buffer (the discretised matrices and
 * about batch * T * n' / 31 floats of chunk states, n' = n rounded up to a power of
 * two) for later calls.
 * Returns EINVAL, ENOMEM or ECUDA. */
int pararnn_lsim(pararnn_ctx *ctx, const float *A, const float *Bm, const float *C, const float *D, int n, int m,
                 int p, const float *U, const float *x0, double dt, int interp, int batch, int T, float *y_out,
                 float *x_out);

/* Adjoint backward at the states h returned by pararnn_newton_forward, for
 * L = sum_t <grad_h_t, h_t> ("Para-Seq" README, Main features: adjoint backward with
 * reverse adjoint scans; DEER summary, Surprising findings: the backward pass is one
 * linear solve).  With every Jacobian evaluated at the given states:
 *   lambda_t = grad_h_t + J_{t+1}^T lambda_{t+1},  lambda_{T-1} = grad_h_{T-1}
 *   grad_xproj_t = (df_t/dp_t)^T lambda_t;  grad_params = sum_{b,t} (df_t/dtheta)^T lambda_t;
 *   grad_h0 = J_0^T lambda_0.
 * GRU and LSTM, xproj path only (p->x unused).
 *   grad_h      like h (LSTM: (dL/dc, dL/dh) pairs)
 *   grad_xproj  [B, T, 3, H]
 *   grad_params GRU [3, H] = d/d(a_z, a_r, a_c); LSTM [5, H] = d/d(a_f, a_g, a_o, w_f, w_o)
 *               (overwritten).  Summation: when NPAR * H <= 12288 each CTA accumulates
 *               its terms in a shared-memory table with shared atomics and the per-CTA
 *               tables are summed over CTAs in a fixed order; otherwise each tile adds
 *               its per-unit sums with global float atomics.  Either way the order of
 *               additions inside a CTA depends on thread timing, so the last bits can
 *               differ between runs.
 *   grad_h0     like h0, or NULL */
int pararnn_adjoint_backward(pararnn_ctx *ctx, const float *xproj, const pararnn_params *p,
                             const float *h0, const float *h, const float *grad_h,
                             float *grad_xproj, float *grad_params, float *grad_h0);

/* Backward pass of a whole trainable layer, input projection included: the adjoint of
 * pararnn_adjoint_backward followed by the reverse pass of pararnn_input_proj_backward
 * for bf16 x and W ("Para-Seq" README, Main features: trainable layers with adjoint
 * backward), with grad_xproj never stored in fp32: the adjoint rounds it to bf16
 * (nearest even, the operand the two tensor-core products read, exactly as
 * pararnn_input_proj_backward rounds it) and sums its fp32 values into grad_bias.
 *   xproj, p, h0, h, grad_h, grad_params, grad_h0 as for pararnn_adjoint_backward
 *   x [B*T, K] bf16, W [3H, K] bf16 (the projection of pararnn_input_proj)
 *   grad_x [B*T, K], grad_W [3H, K], grad_bias [3H]: fp32, each may be NULL (not computed)
 * grad_x and grad_W equal those of pararnn_adjoint_backward + pararnn_input_proj_backward
 * bit for bit; grad_bias sums the same fp32 terms with one float atomic per lane, gate
 * and tile, so its last bits can differ between runs.  Shapes without the adjoint's
 * TMA-fed tiles (H not a multiple of 32, or a parameter table over 12288 floats) take
 * those two calls' path through an fp32 buffer in the scratch.
 * Shapes: B*T, K and 3H multiples of 8, as for pararnn_input_proj_backward.  The
 * context's scratch grows to the projection backward's plus, on the fallback path,
 * 4 * B*T * 3H bytes.  Returns EINVAL, EALIGN, EUNSUPPORTED, ENOMEM or ECUDA. */
int pararnn_layer_backward(pararnn_ctx *ctx, const float *xproj, const pararnn_params *p, const float *h0,
                           const float *h, const float *grad_h, const void *x, const void *W, int K,
                           float *grad_x, float *grad_W, float *grad_bias, float *grad_params,
                           float *grad_h0);

/* Synchronise the context's stream and report (then clear) device-side conditions:
 * *device_status = PARARNN_OK, PARARNN_ENONFINITE or PARARNN_ETIMEOUT (first seen). */
int pararnn_get_status(pararnn_ctx *ctx, int *device_status);

/* Static text for a status code. */
const char *pararnn_strerror(int status);

/* Diagnostics.
 * knob 1: bounded-wait limit in nanoseconds (default 1e9).
 * knob 2: tile index whose look-back publication is withheld (-1 = none); used
 *         only by the failure-detection test to make a successor's wait run out.
 * knob 3: device pointer (float*) receiving delta_k of every Newton iteration, with
 *         knob 4 its capacity (0 disables).
 * knob 5: non-zero makes the long-sequence Newton tiles take every carry from the
 *         look-back, never from their own halo (tests of the look-back path).
 * knob 6: channels per tile of the wide-layer Newton kernel (H % 32 == 0, xproj
 *         given): 8, 16 or 32; 0 is the default (32). */
int pararnn_debug_set(pararnn_ctx *ctx, int knob, long long value);

/* Number of kernels the last call launched on the stream. */
int pararnn_last_launch_count(pararnn_ctx *ctx);

/* ---- Allocation-free variant (no counterpart in the pages) ------------------------
 * pararnn_linear_scan_noalloc computes exactly what pararnn_linear_scan computes for
 * kind PARARNN_SCAN_DIAG or PARARNN_SCAN_BLOCK2, for callers that cannot call
 * cudaMalloc: programs whose device memory belongs to another allocator, loops that
 * must not pay the implicit device synchronisation of an allocation, services that
 * must not meet out-of-memory after start-up.  It takes no context and allocates
 * nothing: its scratch (control block and look-back words) is one static device
 * array of PARARNN_NOALLOC_SCRATCH_BYTES that every device loading the library keeps
 * until the process exits.
 *   - Runs on the calling thread's current device, on `cuda_stream` (NULL = legacy
 *     default stream).  Inputs and outputs are caller-owned device memory as for
 *     pararnn_linear_scan.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress, which
 *     allocates nothing).  The first call on a device, and the first call after the
 *     device's primary context was re-created (cudaDeviceReset), clears the array;
 *     make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents: calls that
 *     overlap on the GPU (other streams, other host threads on the same device) race
 *     and must be serialised by the caller.
 *   - status_out: required device int (PARARNN_EINVAL when NULL), set to 0 by the
 *     call; non-zero afterwards means a bounded wait of the scan ran out (the output
 *     is then not valid).  It is the only place such a timeout is reported.
 *   - Returns PARARNN_ESCRATCH, before enqueuing anything, when the problem's scratch
 *     exceeds the array: diag needs about 24 bytes per tile channel, i.e. roughly
 *     B*N*T/128*24 bytes for N >= 32 (B*N*T up to ~89 million) and B*T/4096*24 bytes for
 *     N = 1; block2 about B*N*T bytes for N >= 32. */
#define PARARNN_ESCRATCH (-8)
#define PARARNN_NOALLOC_SCRATCH_BYTES (16u << 20)
int pararnn_linear_scan_noalloc(int kind, const float *J, const float *b, const float *h0, float *h_out,
                                int B, int T, int N, int reverse, int *status_out, void *cuda_stream);

#ifdef __cplusplus
}
#endif
#endif /* PARARNN_H */
