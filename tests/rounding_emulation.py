"""CPU emulation of the CUDA path's rounding points, for tests only (not part of the oracle).

The oracle computes the layer in fp64 with no intermediate rounding.  The CUDA path rounds at
three places: the SwiGLU output h is rounded to bf16 (it is the down GEMM's operand), each
expert's output row is scaled by its fp32 router weight and kept in fp32, and the combine sums
a token's k rows plus the shared expert's row in fp32, in slot order, and rounds y to bf16 once.
This module applies exactly those roundings to fp64 products (the GPU's fp32 accumulation order
is the only thing left out), so the GPU's output should agree with it to about one bf16 ulp of y,
whatever the oracle-relative error of bf16 arithmetic on a given input is.
"""
from __future__ import annotations

import numpy as np

import moe_inputs as mi
import oracle


def bf16_round(a) -> np.ndarray:
    """fp64 -> nearest bf16 value (round to nearest even, through fp32), returned as fp64."""
    u = np.asarray(a, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _swiglu_rows(X, GU):
    F = GU.shape[0] // 2
    g = X @ GU[:F].T
    u = X @ GU[F:].T
    return g / (1.0 + np.exp(-g)) * u


def emulate_layer(x, wg, bias, gate_up, down, k, shared_gate_up=None, shared_down=None):
    """y [T, D] (fp64 holding bf16 values) with the CUDA path's roundings; bf16 inputs as uint16."""
    X = mi.bf16_to_f64(x)
    T, D = X.shape
    E = wg.shape[0]
    idx, p = oracle.router(x, wg, bias, k)
    p32 = p.astype(np.float32).astype(np.float64)
    GU, DN = mi.bf16_to_f64(gate_up), mi.bf16_to_f64(down)
    acc = np.zeros((T, k, D), np.float32)  # the fp32 pre-scaled expert rows, by slot
    for e in range(E):
        sel = np.argwhere(idx == e)
        if sel.size == 0:
            continue
        t, j = sel[:, 0], sel[:, 1]
        h = bf16_round(_swiglu_rows(X[t], GU[e]))
        o = (h @ DN[e].T).astype(np.float32)  # the GEMM's fp32 accumulator
        acc[t, j] = o * p32[t, j].astype(np.float32)[:, None]  # the epilogue's fp32 scale
    y = np.zeros((T, D), np.float32)
    for j in range(k):  # the combine: fp32 sums in slot order
        y = y + acc[:, j]
    if shared_gate_up is not None:
        hs = bf16_round(_swiglu_rows(X, mi.bf16_to_f64(shared_gate_up)))
        y = y + (hs @ mi.bf16_to_f64(shared_down).T).astype(np.float32)
    return bf16_round(y.astype(np.float64))
