// internal.h -- host-side interfaces between the C ABI (api.cu) and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace prn {

struct Ctl;
struct Dbg;

// Workspace carved by the host for one launch.
struct Work {
    Ctl *ctl;                  // per-call control block (zeroed before the launch)
    int *sticky;               // sticky device status (cleared by get_status)
    unsigned long long *agg;   // look-back: tile aggregates, epoch-tagged words
    unsigned long long *inc;   // look-back: tile inclusive values, epoch-tagged words
    float *side;               // Newton: last state of every tile, two parities
    unsigned epoch0;           // this launch uses epochs epoch0 + 1 .. epoch0 + plan.epochs
};

// What a launch needs (filled by the *_plan functions).
struct Plan {
    long ntiles = 0;
    int grid = 0;
    int C = 0;                     // channels per tile
    size_t agg_words = 0, inc_words = 0, side_bytes = 0;
    unsigned epochs = 2;           // look-back epochs the launch may consume
    const void *kernel = nullptr;  // for the launch
    int dyn_smem = 0;
    int variant = 0;
    int tch = 0;                   // steps per tile
    int staged = 0;                // Newton: staged kernel (args + tensor maps)
    int staged_tma = 0;            // staged kernel fed by TMA
    int S = 1;                     // state components per unit
    int threads = 256;             // threads per CTA
    int halo_w = 1;                // side-buffer values per tile boundary and channel
    int tab = 0;                   // adjoint: shared-memory gradient table variant
};

struct DbgHost {
    unsigned long long wait_ns = 1000000000ull;
    long long skip_tile = -1;
    float *delta_log = nullptr;
    int delta_log_cap = 0;
    int no_halo = 0;
    int wide_variant = 0;
};

// ---- Newton forward, diagonal / 2x2-block cells (GRU, LSTM) -----------------------
struct NewtonDiagReq {
    int cell;   // 0 GRU, 1 LSTM
    int jmode;  // linearisation: 0 Jacobian, 1 LSTM block diagonal, 2 zero (Jacobi), 3 identity (Picard)
    int B, T, H, in;
    const float *xproj, *x, *W, *bias, *a, *peep, *h0;
    float *h;
    int max_iters;
    float tol;
    int *iters_out;
    float *delta_out, *residual_out;
    int variant = 0;  // tile shape of the wide-layer kernel (0: the default)
};
int newton_diag_plan(const NewtonDiagReq &r, int num_sms, Plan *plan);
int newton_staged_plan(const NewtonDiagReq &r, int num_sms, Plan *plan);  // 1: shape not covered
cudaError_t newton_diag_launch(const NewtonDiagReq &r, const Plan &plan, const Work &w,
                               const DbgHost &dbg, cudaStream_t st);

// ELK (damped Newton by Kalman smoothing) for the diagonal linearisations (elk.cu).
int elk_plan(const NewtonDiagReq &r, int num_sms, Plan *plan);
cudaError_t elk_launch(const NewtonDiagReq &r, float lambda, const Plan &plan, const Work &w, const DbgHost &dbg,
                       cudaStream_t st);

// ---- Newton forward, tanh RNN (dense DEER and quasi-DEER) -------------------------
struct NewtonTanhReq {
    int quasi;
    int jmode;  // 0: the cell's (quasi) Jacobian, 2 zero (Jacobi), 3 identity (Picard)
    int B, T, n, in;
    const float *xproj, *x, *W, *bias, *A, *h0;
    float *h;
    int max_iters;
    float tol;
    int *iters_out;
    float *delta_out, *residual_out;
};
int newton_tanh_plan(const NewtonTanhReq &r, int num_sms, Plan *plan);
// ELK for the tanh RNN (quasi-ELK: the diagonal of its Jacobian), n <= 64; 1: unsupported
int elk_tanh_plan(const NewtonTanhReq &r, int num_sms, Plan *plan);
cudaError_t elk_tanh_launch(const NewtonTanhReq &r, float lambda, const Plan &plan, const Work &w,
                            const DbgHost &dbg, cudaStream_t st);
cudaError_t newton_tanh_launch(const NewtonTanhReq &r, const Plan &plan, const Work &w,
                               const DbgHost &dbg, cudaStream_t st);
// quasi-DEER at n == 8 with raw inputs of width 1, 2 or 4 (tanh_quasi8.cu); 1: not covered
int tanh_quasi8_plan(const NewtonTanhReq &r, int num_sms, Plan *plan);
cudaError_t tanh_quasi8_launch(const NewtonTanhReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                               cudaStream_t st);
// full DEER at 32 < n <= 64 with the Jacobian products on the tensor cores (deer_tc.cu); 1: not covered
int deer_tc_plan(const NewtonTanhReq &r, int num_sms, Plan *plan);
cudaError_t deer_tc_launch(const NewtonTanhReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                           cudaStream_t st);

// ---- standalone linear scan -------------------------------------------------------
struct ScanReq {
    int kind;  // 0 diag, 1 block2, 2 dense
    int B, T, N, reverse;
    const float *J, *b, *h0;
    float *out;
};
int scan_diag_plan(const ScanReq &r, int num_sms, Plan *plan);   // kinds diag, block2
cudaError_t scan_diag_launch(const ScanReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                             cudaStream_t st);
int scan_dense_plan(const ScanReq &r, int num_sms, Plan *plan);  // kind dense
cudaError_t scan_dense_launch(const ScanReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                              cudaStream_t st);

// ---- adjoint backward (GRU, LSTM) --------------------------------------------------
struct AdjointReq {
    int cell;  // 0 GRU, 1 LSTM
    int B, T, H;
    const float *xproj, *a, *peep, *h0, *h, *g;
    float *grad_xproj, *grad_params, *grad_h0;
    // layer backward: grad_xproj rounded to bf16 (nearest even) instead of fp32, and its
    // column sums (fp32 values) added into grad_bias [3 H] (zeroed by the caller); the
    // TMA-fed tiles only (H % 32 == 0)
    bool out_bf16 = false;
    unsigned short *grad_xproj_bf16 = nullptr;
    // and its transpose [3 H][B T] (ParaGRU tiles of 8 steps per thread, T % 8 == 0); null: none
    unsigned short *grad_xproj_bf16_t = nullptr;
    float *grad_bias = nullptr;
};
// Whether the wide adjoint's bf16 variant writes the transposed copy for this shape.
bool adjoint_wide_writes_transpose(const AdjointReq &r);
int adjoint_plan(const AdjointReq &r, int num_sms, Plan *plan);
// TMA-fed tiles for H % 32 == 0 (adjoint_wide.cu); 1: shape not covered
int adjoint_wide_plan(const AdjointReq &r, int num_sms, Plan *plan);
cudaError_t adjoint_wide_launch(const AdjointReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                                cudaStream_t st);
cudaError_t adjoint_launch(const AdjointReq &r, const Plan &plan, const Work &w, const DbgHost &dbg,
                           cudaStream_t st);

// ---- input projection ---------------------------------------------------------------
int proj_check(int x_dtype, int M, int K, int N);
cudaError_t proj_launch(int x_dtype, const void *x, const void *W, const float *bias, float *y, int M,
                        int K, int N, int num_sms, cudaStream_t st, int *launches, int *sticky);
// The same, allowed to split K into up to kMaxKsplit parts summed through `ws` (ws_floats
// floats) when the output has too few tiles for the SMs.
constexpr int kMaxKsplit = 4;
cudaError_t proj_launch_split(int x_dtype, const void *x, const void *W, const float *bias, float *y, int M, int K,
                              int N, int num_sms, cudaStream_t st, int *launches, int *sticky, float *ws,
                              size_t ws_floats);

// ---- input projection backward ------------------------------------------------------
int proj_bwd_check(int x_dtype, int M, int K, int N);
size_t proj_bwd_scratch_bytes(int x_dtype, int M, int K, int N);
// The bf16 path from a bf16 grad_xproj that the caller wrote at proj_bwd_gb(scratch, M, N)
// (no fp32 copy, no bias sums): grad_x and grad_W only.
// have_gbt: the transposed copy is there too (proj_bwd_gbt(scratch, M, N)).
unsigned short *proj_bwd_gb(void *scratch, int M, int N);
unsigned short *proj_bwd_gbt(void *scratch, int M, int N);
cudaError_t proj_bwd_from_bf16_launch(const void *x, const void *W, float *grad_x, float *grad_W, int M, int K, int N,
                                      bool have_gbt, void *scratch, int num_sms, cudaStream_t st, int *launches,
                                      int *sticky);
cudaError_t proj_bwd_launch(int x_dtype, const float *gx, const void *x, const void *W, float *grad_x, float *grad_W,
                            float *grad_bias, int M, int K, int N, void *scratch, int num_sms, cudaStream_t st,
                            int *launches, int *sticky);

// Helpers.
// Fixed-step linear simulation (lsim.cu).
constexpr int kLsimMaxN = 32, kLsimMaxM = 16, kLsimMaxP = 32;
struct LsimReq {
    const float *A, *Bm, *C, *D;  // [n,n], [n,m], [p,n], [p,m] or NULL
    int n, m, p;
    const float *U, *x0;  // [batch,T,m], [batch,n] or NULL
    double h;             // time step
    int interp;           // 0 held input, 1 linear between samples
    long batch, T;
    float *y, *x;         // [batch,T,p], [batch,T,n] or NULL
};
int lsim_check(const LsimReq &r);
size_t lsim_scratch_bytes(const LsimReq &r);
cudaError_t lsim_launch(const LsimReq &r, float *scratch, cudaStream_t st, int *launches);

int occupancy_grid(const void *kernel, int threads, size_t smem, int num_sms, long ntiles);

}  // namespace prn
