"""Seeded synthetic workloads for the Newton/DEER evaluation of nonlinear RNNs.

This module only draws random inputs; it holds none of the method's arithmetic
(no cell, no Jacobian, no scan).  Both the CUDA path and the fp64 CPU oracle are
fed from the arrays it returns, so the two sides always see bit-identical inputs.

Workload shapes follow the pages: the DEER benchmark of a GRU with a 1M-step
sequence, batch 16 and state size 1 ("Parallelizing non-linear sequential models
over the sequence length", Key results), LLM-width ParaGRU / ParaLSTM layers
("ParaRNN: Unlocking Parallel Training of Nonlinear RNNs for Large Language
Models", abstract) and a vanilla tanh RNN at state sizes 8 and 64, where the
summary reports that the speedup collapses (same DEER page, Surprising findings).

Draw order (fixed, so that a seed names one input set):
  numpy.random.Generator(PCG64(seed)), all draws in float64, in this order:
  x; W per gate (row-major [H, in] each); recurrent diagonals per gate;
  peepholes (f, o); biases per gate; A then U (tanh RNN); upstream gradient.
Values are then cast to float32, and rounded to bfloat16 (round to nearest even)
where the workload says the input is bf16.  ``N(0, v)`` means variance v.

Layouts (row-major, batch first):
  x      [B, T, in]
  W      [G*H, in]   row g*H + u feeds gate g of unit u   (tanh RNN: U [n, in])
  bias   [G*H]                                              (tanh RNN: b [n])
  a      [3, H]      GRU (z, r, c) / LSTM (f, g, o) recurrent diagonals
  peep   [2, H]      LSTM peepholes (w_f, w_o)
  A      [n, n]      tanh RNN recurrent matrix, A[i, j] multiplies h_j into unit i
  h0     [B, H] (GRU), [B, H, 2] (LSTM, (c, h) pairs), [B, n] (tanh)
  g      upstream dL/dstate, the shape of the states; LSTM (dL/dc, dL/dh) pairs
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GRU, LSTM, TANH = "gru", "lstm", "tanh"


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: cell, sizes, distributions and solver settings."""

    name: str
    cell: str          # "gru" | "lstm" | "tanh"
    B: int
    T: int
    H: int             # units (GRU/LSTM) or state size n (tanh)
    inp: int           # input width
    seed: int
    tol: float         # convergence tolerance on max|dh|; 0 disables the test
    max_iters: int     # Newton cap
    bf16: bool         # x and W are bf16 values
    quasi: bool = False  # tanh RNN: diagonal (quasi-DEER) Jacobian
    backward: bool = False
    residual: bool = False
    # distribution parameters
    w_dist: str = "uniform_fan_in"   # or "normal"
    w_var: float = 0.0
    a_range: float = 0.5
    bias_var: float = 0.0            # 0 -> biases are zero
    forget_bias: float = 0.0

    @property
    def G(self) -> int:
        return 1 if self.cell == TANH else 3

    @property
    def state_per_unit(self) -> int:
        return 2 if self.cell == LSTM else 1

    @property
    def elems(self) -> int:
        """Newton-solved state elements B*T*H (LSTM counts units, not (c, h))."""
        return self.B * self.T * self.H

    def resized(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the method's hot path, named by what they are.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("gru_b1_t1024_in4_h8", GRU, B=1, T=1024, H=8, inp=4, seed=0,
                 tol=1e-6, max_iters=1024, bf16=False),
        Workload("gru_b16_t1048576_in2_h1", GRU, B=16, T=1 << 20, H=1, inp=2, seed=1,
                 tol=1e-6, max_iters=1 << 20, bf16=False),
        Workload("gru_b8_t4096_h2048_bf16", GRU, B=8, T=4096, H=2048, inp=2048, seed=2,
                 tol=0.0, max_iters=3, bf16=True, backward=True, residual=True,
                 w_dist="normal", w_var=1.0 / 2048, a_range=0.9, bias_var=0.1),
        Workload("lstm_b4_t8192_h1024_bf16", LSTM, B=4, T=8192, H=1024, inp=1024, seed=3,
                 tol=1e-5, max_iters=8192, bf16=True, backward=True,
                 w_dist="normal", w_var=1.0 / 1024, a_range=0.5, forget_bias=1.0),
        Workload("tanh_b16_t65536_in4_n8_deer", TANH, B=16, T=65536, H=8, inp=4, seed=4,
                 tol=1e-5, max_iters=65536, bf16=False),
        Workload("tanh_b16_t65536_in4_n8_quasi", TANH, B=16, T=65536, H=8, inp=4, seed=4,
                 tol=1e-5, max_iters=65536, bf16=False, quasi=True),
        Workload("tanh_b16_t65536_in4_n64_deer", TANH, B=16, T=65536, H=64, inp=4, seed=4,
                 tol=1e-5, max_iters=65536, bf16=False),
        Workload("tanh_b16_t65536_in4_n64_quasi", TANH, B=16, T=65536, H=64, inp=4, seed=4,
                 tol=1e-5, max_iters=65536, bf16=False, quasi=True),
    ]
}

BENCH_WORKLOAD = "gru_b16_t1048576_in2_h1"


def round_bf16(a: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 value (ties to even), returned as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of float32 values that are exactly bfloat16."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    assert not np.any(u & 0xFFFF), "values are not bf16-representable"
    return (u >> 16).astype(np.uint16)


def generate(w: Workload, with_grad: bool | None = None) -> dict:
    """Draw the inputs of workload ``w`` (see the module docstring for order/layout).

    Returns float32 arrays; bf16 inputs are float32 arrays holding bf16 values.
    Keys: x, W, bias, a, peep (LSTM), A (tanh), h0, g (when with_grad).
    """
    if with_grad is None:
        with_grad = w.backward
    rng = np.random.Generator(np.random.PCG64(w.seed))
    B, T, H, I, G = w.B, w.T, w.H, w.inp, w.G
    out = {}
    out["x"] = rng.standard_normal((B, T, I))
    if w.cell == TANH:
        W = None
    else:
        ws = []
        for _ in range(G):
            if w.w_dist == "normal":
                ws.append(rng.standard_normal((H, I)) * math.sqrt(w.w_var))
            else:
                bound = 1.0 / math.sqrt(I)
                ws.append(rng.uniform(-bound, bound, size=(H, I)))
        W = np.concatenate(ws, axis=0)
        out["a"] = np.stack([rng.uniform(-w.a_range, w.a_range, size=H) for _ in range(3)])
        if w.cell == LSTM:
            out["peep"] = np.stack([rng.uniform(-w.a_range, w.a_range, size=H) for _ in range(2)])
        if w.bias_var > 0:
            bias = np.concatenate([rng.standard_normal(H) * math.sqrt(w.bias_var) for _ in range(G)])
        else:
            bias = np.zeros(G * H)
        if w.cell == LSTM:
            bias[0:H] = w.forget_bias
        out["bias"] = bias
    if w.cell == TANH:
        out["A"] = rng.standard_normal((H, H)) * (0.9 / math.sqrt(H))
        bound = 1.0 / math.sqrt(I)
        W = rng.uniform(-bound, bound, size=(H, I))
        out["bias"] = np.zeros(H)
    out["W"] = W
    if w.cell == LSTM:
        out["h0"] = np.zeros((B, H, 2))
    else:
        out["h0"] = np.zeros((B, H))
    if with_grad:
        g = rng.standard_normal((B, T, H))
        if w.cell == LSTM:
            gg = np.zeros((B, T, H, 2))
            gg[..., 1] = g          # dL/dh drawn, dL/dc = 0
            g = gg
        out["g"] = g
    for k in list(out):
        out[k] = np.ascontiguousarray(out[k], dtype=np.float32)
    if w.bf16:
        out["x"] = round_bf16(out["x"])
        out["W"] = round_bf16(out["W"])
    return out
