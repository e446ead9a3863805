"""The router GEMM in front of the routing step, and its backward -- the oracle's plain
definitions (test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline use this module).

Article ("Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72"), lead and
§01: at every step a router decides anew which experts each token goes to, so in training
the router itself receives a gradient.  The pages give no formula for the router; the plain
reading is a bias-free linear layer whose outputs are the logits the routing step ranks.

Readings (the pages are silent; listed in the design notes):
* W_r is stored as [E, d], one row per expert (the layout of a linear layer's weight):
  logits[t, e] = sum_i x[t, i] * W_r[e, i].
* The forward operands are bf16 (x as the layer receives it, W_r given in bf16); the sum is
  exact here (fp64) and accumulated in fp32 on the device; the logits are fp32.
* Backward: the logits' gradient G (fp32, from the routing-weight backward) is rounded to
  bf16 (nearest, ties to even) as the operand of both backward GEMMs, as the forward's
  operands are bf16:  dx_r = bf16(G) . W_r  [T, d],  dW_r = bf16(G)^T . x  [E, d].
  dx_r is the router's share of the gradient of x (the expert path adds its own share).
"""
from __future__ import annotations

import numpy as np

from .layer import bf16_bits_to_f64, bf16_round


def router_logits_values(x: np.ndarray, wr: np.ndarray) -> np.ndarray:
    """logits [T, E] = x . W_r^T in fp64 for real-valued x [T, d], W_r [E, d]."""
    return np.asarray(x, np.float64) @ np.asarray(wr, np.float64).T


def router_logits(x_bits: np.ndarray, wr_bits: np.ndarray) -> np.ndarray:
    """logits [T, E] (fp64, exact) = x . W_r^T from bf16 bit patterns x [T, d], W_r [E, d]."""
    return router_logits_values(bf16_bits_to_f64(x_bits), bf16_bits_to_f64(wr_bits))


def router_backward(dlogits: np.ndarray, x_bits: np.ndarray, wr_bits: np.ndarray):
    """(dx_r [T, d], dW_r [E, d]) in fp64 from the logits' gradient [T, E].

    The gradient is rounded to bf16 first (reading above); the products are then exact.
    """
    g = bf16_round(np.asarray(dlogits, np.float64))
    return g @ bf16_bits_to_f64(wr_bits), g.T @ bf16_bits_to_f64(x_bits)


def router_logits_bruteforce(x_bits: np.ndarray, wr_bits: np.ndarray) -> np.ndarray:
    """Element-by-element loops of the same definition (small shapes only)."""
    x, w = bf16_bits_to_f64(x_bits), bf16_bits_to_f64(wr_bits)
    T, d = x.shape
    E = w.shape[0]
    out = np.zeros((T, E))
    for t in range(T):
        for e in range(E):
            s = 0.0
            for i in range(d):
                s += x[t, i] * w[e, i]
            out[t, e] = s
    return out


def router_backward_bruteforce(dlogits: np.ndarray, x_bits: np.ndarray, wr_bits: np.ndarray):
    """Loops over the chain rule of logits[t, e] = sum_i x[t, i] W_r[e, i] (small shapes)."""
    g = bf16_round(np.asarray(dlogits, np.float64))
    x, w = bf16_bits_to_f64(x_bits), bf16_bits_to_f64(wr_bits)
    T, d = x.shape
    E = w.shape[0]
    dx = np.zeros((T, d))
    dw = np.zeros((E, d))
    for t in range(T):
        for e in range(E):
            for i in range(d):
                dx[t, i] += g[t, e] * w[e, i]   # d logits[t, e] / d x[t, i] = W_r[e, i]
                dw[e, i] += g[t, e] * x[t, i]   # d logits[t, e] / d W_r[e, i] = x[t, i]
    return dx, dw
