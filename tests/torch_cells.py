"""PyTorch reference cells wired to the three cells of the method (float64, CPU).

These are the independent pins for the oracle: the cell maps are evaluated by
PyTorch's own ``GRUCell`` / ``LSTMCell`` / ``RNNCell`` (library routines), with
weight matrices built so that the library cell computes the diagonal ParaGRU,
the CIFG + peephole ParaLSTM and the vanilla tanh RNN.  Nothing here restates
the oracle's formulas; Jacobians and gradients come from autograd and linear
solves come from ``torch.linalg.solve``.

Input to every cell is the projected input p_t = xproj[b, t] (gates stacked),
so the library's input weights are selection matrices.
"""
from __future__ import annotations

import torch
from torch.func import functional_call

f64 = torch.float64


def _eye(H):
    return torch.eye(H, dtype=f64)


def _Z(H, W=None):
    return torch.zeros(H, W if W is not None else H, dtype=f64)


class GRU:
    """Diagonal ParaGRU through torch.nn.GRUCell.

    torch: r = s(W_ir x + W_hr h), z_t = s(W_iz x + W_hz h),
           n = tanh(W_in x + r * (W_hn h)), h' = (1 - z_t) n + z_t h.
    With z_t = 1 - z (sigmoid of the negated pre-activation) this is
    h' = (1 - z) h + z n, the diagonal ParaGRU with candidate n = c.
    """

    def __init__(self, H, a):
        self.H = H
        self.cell = torch.nn.GRUCell(3 * H, H, bias=True, dtype=f64)
        self.a = a  # tensor [3, H]: (a_z, a_r, a_c)

    def params(self, a=None):
        a = self.a if a is None else a
        H = self.H
        I, Z = _eye(H), _Z(H)
        # input features: [p_z | p_r | p_c]; torch gate rows: (r, z, n)
        w_ih = torch.cat([torch.cat([Z, I, Z], 1), torch.cat([-I, Z, Z], 1),
                          torch.cat([Z, Z, I], 1)], 0)
        w_hh = torch.cat([torch.diag(a[1]), -torch.diag(a[0]), torch.diag(a[2])], 0)
        zb = torch.zeros(3 * H, dtype=f64)
        return {"weight_ih": w_ih, "weight_hh": w_hh, "bias_ih": zb, "bias_hh": zb}

    def step(self, p, h, a=None):
        """p [B, 3, H], h [B, H] -> h' [B, H]."""
        return functional_call(self.cell, self.params(a), (p.reshape(p.shape[0], -1), h))


class LSTM:
    """CIFG + peephole ParaLSTM through torch.nn.LSTMCell (state (c, h) per unit).

    torch: i, f, g, o gates; c' = f c + i g; h' = o tanh(c').
    The library input is [p_f | p_g | p_o | c_prev | c_new]: the forget peephole
    reads c_prev, the output peephole reads c_new.  A first call (c_new = 0, which
    only the output gate reads) yields c'; a second call with c_new = c' yields h'.
    CIFG: the input gate is the sigmoid of the negated forget pre-activation.
    """

    def __init__(self, H, a, peep):
        self.H = H
        self.cell = torch.nn.LSTMCell(5 * H, H, bias=True, dtype=f64)
        self.a, self.peep = a, peep  # a [3, H] (a_f, a_g, a_o); peep [2, H] (w_f, w_o)

    def params(self, a=None, peep=None):
        a = self.a if a is None else a
        peep = self.peep if peep is None else peep
        H = self.H
        I, Z = _eye(H), _Z(H)
        wf, wo = torch.diag(peep[0]), torch.diag(peep[1])
        rows = [
            torch.cat([-I, Z, Z, -wf, Z], 1),  # i = 1 - f
            torch.cat([I, Z, Z, wf, Z], 1),    # f
            torch.cat([Z, I, Z, Z, Z], 1),     # g
            torch.cat([Z, Z, I, Z, wo], 1),    # o
        ]
        w_ih = torch.cat(rows, 0)
        w_hh = torch.cat([-torch.diag(a[0]), torch.diag(a[0]), torch.diag(a[1]),
                          torch.diag(a[2])], 0)
        zb = torch.zeros(4 * H, dtype=f64)
        return {"weight_ih": w_ih, "weight_hh": w_hh, "bias_ih": zb, "bias_hh": zb}

    def step(self, p, s, a=None, peep=None):
        """p [B, 3, H], s [B, H, 2] as (c, h) -> s' [B, H, 2]."""
        prm = self.params(a, peep)
        c, h = s[..., 0], s[..., 1]
        B = p.shape[0]
        pf = p.reshape(B, -1)
        _, c1 = functional_call(self.cell, prm, (torch.cat([pf, c, torch.zeros_like(c)], 1), (h, c)))
        h2, c2 = functional_call(self.cell, prm, (torch.cat([pf, c, c1], 1), (h, c)))
        return torch.stack([c2, h2], -1)


class TANH:
    """Vanilla tanh RNN through torch.nn.RNNCell: h' = tanh(A h + p)."""

    def __init__(self, n, A):
        self.n = n
        self.cell = torch.nn.RNNCell(n, n, bias=True, nonlinearity="tanh", dtype=f64)
        self.A = A

    def params(self, A=None):
        A = self.A if A is None else A
        zb = torch.zeros(self.n, dtype=f64)
        return {"weight_ih": _eye(self.n), "weight_hh": A, "bias_ih": zb, "bias_hh": zb}

    def step(self, p, h, A=None):
        """p [B, 1, n], h [B, n] -> h' [B, n]."""
        return functional_call(self.cell, self.params(A), (p[:, 0], h))


def make(cell, H, prm):
    t = lambda k: torch.as_tensor(prm[k], dtype=f64)
    if cell == "gru":
        return GRU(H, t("a"))
    if cell == "lstm":
        return LSTM(H, t("a"), t("peep"))
    return TANH(H, t("A"))


def rollout(lib, xproj, h0):
    """Sequential rollout with the library cell.  xproj [B,T,G,H] tensor."""
    T = xproj.shape[1]
    out, h = [], h0
    for t in range(T):
        h = lib.step(xproj[:, t], h)
        out.append(h)
    return torch.stack(out, 1)


def stacked_residual(lib, xproj, h0, hs, **kw):
    """F_t = h_t - cell(h_{t-1}, p_t) for all t (the system Newton solves)."""
    T = xproj.shape[1]
    prev = torch.cat([h0[:, None], hs[:, :-1]], 1)
    outs = [lib.step(xproj[:, t], prev[:, t], **kw) for t in range(T)]
    return hs - torch.stack(outs, 1)


def newton_stacked(lib, xproj, h0, iters, quasi=False, state_shape=None):
    """Newton on the stacked system F(h) = 0 with a dense solve per iteration.

    The Jacobian dF/dh comes from autograd; ``quasi`` keeps only the diagonal of
    each sub-diagonal block -J_t (the quasi-Newton approximation).
    Returns the list of iterates h^(1..iters).
    """
    hs = torch.zeros(state_shape, dtype=f64)
    B, T = hs.shape[:2]
    D = hs[0, 0].numel()
    out = []
    for _ in range(iters):
        F = stacked_residual(lib, xproj, h0, hs)
        Jf = torch.autograd.functional.jacobian(
            lambda v: stacked_residual(lib, xproj, h0, v.reshape(hs.shape)).reshape(-1),
            hs.reshape(-1))
        if quasi:
            N = B * T * D
            Jm = Jf.reshape(B, T, D, B, T, D).clone()
            off = ~torch.eye(D, dtype=torch.bool)
            for b in range(B):
                for t in range(1, T):
                    blk = Jm[b, t, :, b, t - 1, :]
                    blk[off] = 0.0
            Jf = Jm.reshape(N, N)
        step = torch.linalg.solve(Jf, F.reshape(-1))
        hs = hs - step.reshape(hs.shape)
        out.append(hs.clone())
    return out
