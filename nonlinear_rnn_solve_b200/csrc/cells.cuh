// cells.cuh -- the recurrent cells of the method, per unit, in fp32 registers.
//
// "Para-Seq" README, Main features: the diagonal ParaGRU (its Jacobian is diagonal)
// and the CIFG/peephole ParaLSTM (a 2x2 Jacobian block per unit, "structured block"
// scans).  "ParaRNN" abstract: adaptations of GRU and LSTM that keep the Newton
// system cheap.  Cell equations (per unit, p = projected input of each gate):
//
// ParaGRU     z = s(p_z + a_z h), r = s(p_r + a_r h), c = tanh(p_c + a_c (r h)),
//             f = (1 - z) h + z c                               (state h, Jacobian 1x1)
// ParaLSTM    phi = s(p_f + a_f h + w_f c), g = tanh(p_g + a_g h),
//             c' = phi c + (1 - phi) g,  o = s(p_o + a_o h + w_o c'),  h' = o tanh(c')
//             (input gate = 1 - forget gate; forget peephole reads c_{t-1}, output
//             peephole the new c_t; state (c, h), Jacobian 2x2 row-major)
#pragma once
#include "common.cuh"

namespace prn {

struct GruCell {
    static constexpr int S = 1;
    static constexpr int NPAR = 3;  // recurrent diagonals a_z, a_r, a_c
    float az, ar, ac;
    float qz, qr, qc;  // the same, times pre(g)
    // Exponent scale of gate g: s(u) = 1 / (1 + 2^(-u log2 e)), tanh(u) = 2 s(2u) - 1.
    __host__ __device__ static constexpr float pre(int g) { return g == 2 ? -2.f * kLog2e : -kLog2e; }
    __device__ __forceinline__ void load(const float *a, const float *, int H, int h) {
        az = __ldg(a + h);
        ar = __ldg(a + H + h);
        ac = __ldg(a + 2 * H + h);
        qz = pre(0) * az;
        qr = pre(1) * ar;
        qc = pre(2) * ac;
    }
    // f and J = df/dh at previous state hp, from q_g = pre(g) p_g.
    __device__ __forceinline__ void eval_pre(const float q[3], const float *hp, float *f, float *J) const {
        const float h = hp[0];
        const float z = rcp_hw(1.f + ex2_hw(fmaf(qz, h, q[0])));
        const float r = rcp_hw(1.f + ex2_hw(fmaf(qr, h, q[1])));
        const float c = fmaf(2.f, rcp_hw(1.f + ex2_hw(fmaf(qc, r * h, q[2]))), -1.f);
        const float cmh = c - h;
        f[0] = fmaf(z, cmh, h);
        // df/dh = (1 - z) + (c - h) dz a_z + z dc a_c (r + h dr a_r),
        // dz = z (1 - z), dr = r (1 - r), dc = 1 - c^2
        const float dz = fmaf(-z, z, z), dr = fmaf(-r, r, r), dc = fmaf(-c, c, 1.f);
        const float j0 = fmaf(az, cmh * dz, 1.f - z);
        J[0] = fmaf(ac, (z * dc) * fmaf(h * ar, dr, r), j0);
    }
    __device__ __forceinline__ void eval(const float p[3], const float *hp, float *f, float *J) const {
        const float q[3] = {pre(0) * p[0], pre(1) * p[1], pre(2) * p[2]};
        eval_pre(q, hp, f, J);
    }
    // Adjoint partials: f, J, df/dp (3) and the factors that turn df/dp into df/da:
    // df/da_z = df/dp_z * h, df/da_r = df/dp_r * h, df/da_c = df/dp_c * (r h).
    __device__ __forceinline__ void partials(const float p[3], const float *hp, float *J, float *dp,
                                             float *fac) const {
        const float h = hp[0];
        const float z = sigm(fmaf(az, h, p[0]));
        const float r = sigm(fmaf(ar, h, p[1]));
        const float c = tanh_(fmaf(ac, r * h, p[2]));
        const float dz = z * (1.f - z), dr = r * (1.f - r), dc = 1.f - c * c;
        J[0] = (1.f - z) + (c - h) * dz * az + z * dc * ac * fmaf(h * dr, ar, r);
        dp[0] = (c - h) * dz;
        dp[1] = z * dc * ac * h * dr;
        dp[2] = z * dc;
        fac[0] = h;
        fac[1] = r * h;
    }
};

struct LstmCell {
    static constexpr int S = 2;
    static constexpr int NPAR = 5;  // a_f, a_g, a_o, w_f, w_o
    float af, ag, ao, wf, wo;
    __host__ __device__ static constexpr float pre(int) { return 1.f; }
    __device__ __forceinline__ void load(const float *a, const float *peep, int H, int h) {
        af = __ldg(a + h);
        ag = __ldg(a + H + h);
        ao = __ldg(a + 2 * H + h);
        wf = __ldg(peep + h);
        wo = __ldg(peep + H + h);
    }
    __device__ __forceinline__ void eval(const float p[3], const float *sp, float *f, float *J) const {
        const float c = sp[0], h = sp[1];
        const float phi = sigm(fmaf(wf, c, fmaf(af, h, p[0])));
        const float g = tanh_(fmaf(ag, h, p[1]));
        const float cn = fmaf(phi, c - g, g);
        const float o = sigm(fmaf(wo, cn, fmaf(ao, h, p[2])));
        const float tc = tanh_(cn);
        f[0] = cn;
        f[1] = o * tc;
        const float dphi = phi * (1.f - phi), dg = 1.f - g * g, dout = o * (1.f - o), dtc = 1.f - tc * tc;
        const float dcc = fmaf((c - g) * dphi, wf, phi);
        const float dch = fmaf((c - g) * dphi, af, (1.f - phi) * dg * ag);
        const float kap = fmaf(dout * wo, tc, o * dtc);  // total dh'/dc'
        J[0] = dcc;
        J[1] = dch;
        J[2] = kap * dcc;
        J[3] = fmaf(dout * ao, tc, kap * dch);
    }
    __device__ __forceinline__ void eval_pre(const float p[3], const float *sp, float *f, float *J) const {
        eval(p, sp, f, J);
    }
    // dp is [2][3] = d(c', h')/d(p_f, p_g, p_o); fac = (h_{t-1}, c_{t-1}, c_t):
    // d/da_f = d/dp_f * h, d/da_g = d/dp_g * h, d/da_o = d/dp_o * h,
    // d/dw_f = d/dp_f * c_{t-1}, d/dw_o = d/dp_o * c_t.
    __device__ __forceinline__ void partials(const float p[3], const float *sp, float *J, float *dp,
                                             float *fac) const {
        const float c = sp[0], h = sp[1];
        const float phi = sigm(fmaf(wf, c, fmaf(af, h, p[0])));
        const float g = tanh_(fmaf(ag, h, p[1]));
        const float cn = fmaf(phi, c - g, g);
        const float o = sigm(fmaf(wo, cn, fmaf(ao, h, p[2])));
        const float tc = tanh_(cn);
        const float dphi = phi * (1.f - phi), dg = 1.f - g * g, dout = o * (1.f - o), dtc = 1.f - tc * tc;
        const float dcc = fmaf((c - g) * dphi, wf, phi);
        const float dch = fmaf((c - g) * dphi, af, (1.f - phi) * dg * ag);
        const float kap = fmaf(dout * wo, tc, o * dtc);
        J[0] = dcc;
        J[1] = dch;
        J[2] = kap * dcc;
        J[3] = fmaf(dout * ao, tc, kap * dch);
        const float dpf = (c - g) * dphi, dpg = (1.f - phi) * dg;
        dp[0] = dpf;
        dp[1] = dpg;
        dp[2] = 0.f;
        dp[3] = kap * dpf;
        dp[4] = kap * dpg;
        dp[5] = dout * tc;
        fac[0] = h;
        fac[1] = c;
        fac[2] = cn;
    }
};

}  // namespace prn
