"""MoE layer forward and backward on MX-quantised operands, fp64, one expert at a time.

Article ("Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72"):
* §01: dispatch sends each token to its experts; after the expert computation, combine
  returns each result to the token's original place; training adds two reverse
  communications in the backward pass.
* §02: the expert FFN is a grouped GEMM with SwiGLU; MXFP8 activations run through
  dispatch, the grouped GEMM and SwiGLU; forward = pull dispatch + push combine,
  backward = pull reverse-combine + push reverse-dispatch.
* §03: the benchmarked layer is scheduling, dispatch, expert FFN, combine and the final
  weighted merge.

Definitions used (the configuration fills what the pages leave open):
  forward, per assignment a = t*k + j routed to expert e:
    x^_t   = MX(x_t) along d (once per token)
    g_a    = x^_t . Wg^_e,   u_a = x^_t . Wu^_e   (Wg, Wu quantised along d per column)
    hpre_a = silu(g_a) * u_a,  silu(g) = g * sigmoid(g)
    h^_a   = MX(hpre_a) along f
    y_a    = h^_a . Wd^_e                          (Wd quantised along f per column)
    out_t  = sum_j w[t,j] * y_{t*k+j}
  backward (readings: the quantiser is a straight-through estimator; every backward
  GEMM operand is MX-quantised along that GEMM's K axis; the saved SwiGLU
  pre-activations g, u are kept in bf16; every weight-gradient operand is the
  token-direction requantisation of the dequantised MX operand the data path already
  holds -- x^, h^, w*dout^ and [dg|du]^):
    dout^_t   = MX(dOut_t) along d
    G_a       = dout^_t . Wd'_e^T          (Wd' = W_down quantised along d)
    dw[t,j]   = <G_a, h^_a>                (gradient w.r.t. the combine weight)
    dh_a      = w_a * G_a
    dg_a      = dh_a * u_a * s * (1 + g_a * (1 - s)),  du_a = dh_a * silu(g_a),  s = sigmoid(g_a)
    dxa_a     = [dg_a | du_a]^ . [Wg | Wu]'_e^T   (dgu quantised along 2f, [Wg|Wu] along 2f)
    dX_t      = sum_j dxa_{t*k+j}
    dWd_e     = H~_e^T . DY~_e,   dWg_e = X~_e^T . DG~_e,   dWu_e = X~_e^T . DU~_e
      where ~ is MX quantisation along the tokens of expert e's segment (blocks of 32
      rows in ascending-token order, zero-padded), H = h^, X = x^, DY = w * dout^ and
      [DG|DU] = [dg|du]^ (the operand of the dX GEMM).
"""
from __future__ import annotations

import numpy as np

from . import mxfp8 as mx
from . import routing as rt


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned as float64.

    Done on the exact value: the bf16 quantum of |v| is 2**(floor(log2|v|) - 7).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, e2 = np.frexp(a)
    e = np.maximum(e2.astype(np.int64) - 1, -126)
    q = np.ldexp(1.0, e - 7)
    return np.copysign(np.rint(a / q) * q, v)


def sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _fq(v, exact):
    """MX quantise-dequantise along the last axis (identity when ``exact``)."""
    return np.asarray(v, np.float64) if exact else mx.fake_quantize_mx(v)


def _bf(v, exact):
    return np.asarray(v, np.float64) if exact else bf16_round(v)


class ExpertWeights:
    """Quantised operand views of one expert's bf16 weights (float64 values)."""

    def __init__(self, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray, exact: bool = False):
        self.wg, self.wu, self.wd = wg, wu, wd           # [d,f], [d,f], [f,d]
        self.exact = exact
        self._cache = {}

    def fwd(self):
        """(Wg^T [f,d], Wu^T [f,d]) quantised along d; Wd^T [d,f] quantised along f."""
        if "fwd" not in self._cache:
            ex = self.exact
            self._cache["fwd"] = (_fq(self.wg.T, ex), _fq(self.wu.T, ex), _fq(self.wd.T, ex))
        return self._cache["fwd"]

    def bwd(self):
        """Wd [f,d] quantised along d; [Wg|Wu] [d,2f] quantised along 2f."""
        if "bwd" not in self._cache:
            ex = self.exact
            self._cache["bwd"] = (_fq(self.wd, ex),
                                  _fq(np.concatenate([self.wg, self.wu], axis=1), ex))
        return self._cache["bwd"]


def quantize_tokens(x_bits: np.ndarray):
    """MX codes/scales of bf16 token rows along the hidden axis, and their values."""
    x = bf16_bits_to_f64(x_bits)
    codes, scales = mx.quantize_mx(x)
    return codes, scales, mx.dequantize_mx(codes, scales)


def expert_forward(xhat_rows: np.ndarray, W: ExpertWeights):
    """One expert on its rows: returns g, u, hpre, (hq codes, hq scales), hhat, y."""
    wgq, wuq, wdq = W.fwd()
    g = xhat_rows @ wgq.T
    u = xhat_rows @ wuq.T
    hpre = g * sigmoid(g) * u
    hq, hs = mx.quantize_mx(hpre)
    hhat = hpre if W.exact else mx.dequantize_mx(hq, hs)
    y = hhat @ wdq.T
    return g, u, hpre, (hq, hs), hhat, y


def forward(x_bits, logits, k, score_fn, E, weights_fn, tokens=None, keep=False, exact=False):
    """Oracle forward of the layer.

    x_bits: bf16 bits [T,d]; logits: fp32 [T,E]; weights_fn(e) -> (Wg [d,f], Wu [d,f],
    Wd [f,d]) float64.  ``tokens``: optional sorted array of token ids; only their outputs
    are computed (rows of other tokens stay 0 and experts without a sampled token are
    skipped).  ``keep``: also return per-position intermediates (g, u, hq, hs, y) in the
    unpadded expert-contiguous order of ``perm``.  ``exact``: every quantiser becomes the
    identity (used to pin the structure against :func:`forward_exact`).
    """
    T, d = x_bits.shape
    idx, w = rt.route(logits, k, score_fn)
    counts, offsets, perm, inv = rt.layout(idx, E)
    xq, xs, xhat = quantize_tokens(x_bits)
    if exact:
        xhat = bf16_bits_to_f64(x_bits)
    out = np.zeros((T, d), np.float64)
    want = np.ones(T, bool) if tokens is None else np.isin(np.arange(T), tokens)
    res = dict(idx=idx, w=w, counts=counts, offsets=offsets, perm=perm, inv=inv,
               xq=xq, xs=xs, out=out)
    if keep:
        A = T * k
        f = None
    for e in range(E):
        rows = perm[offsets[e]:offsets[e + 1]]
        if rows.size == 0:
            continue
        sel = want[rows // k]
        if not sel.any():
            continue
        rows_s = rows[sel]
        t = rows_s // k
        W = ExpertWeights(*weights_fn(e), exact=exact)
        g, u, hpre, (hq, hs), hhat, y = expert_forward(xhat[t], W)
        np.add.at(out, t, w.reshape(-1)[rows_s][:, None] * y)
        if keep:
            if f is None:
                f = g.shape[1]
                for name, shape, dt in (("g", (A, f), np.float64), ("u", (A, f), np.float64),
                                        ("hq", (A, f), np.uint8), ("hs", (A, f // 32), np.uint8),
                                        ("y", (A, d), np.float64)):
                    res[name] = np.zeros(shape, dt)
            pos = inv[rows_s]
            res["g"][pos], res["u"][pos] = g, u
            res["hq"][pos], res["hs"][pos], res["y"][pos] = hq, hs, y
    return res


def forward_bf16(x_bits, logits, k, score_fn, E, weights_fn, round_h=True):
    """Oracle forward of the layer's BF16 variant (no MX quantisation).

    Reading (the pages report BF16 results beside MXFP8 ones and say nothing more): the
    same layer with bf16 operands throughout -- x and the expert weights as given (bf16
    values), each GEMM accumulated exactly here (fp32 on the device), and the SwiGLU output
    rounded to bf16, the operand dtype of the down GEMM:
        g = x Wg, u = x Wu, h = bf16(silu(g) * u), y = h Wd, out_t = sum_j w[t,j] y.
    ``round_h=False`` drops that rounding (the structure pin against forward_exact).
    Returns dict with idx, w and out [T,d] (fp64, before the final bf16 rounding).
    """
    T, d = x_bits.shape
    idx, w = rt.route(logits, k, score_fn)
    counts, offsets, perm, inv = rt.layout(idx, E)
    x = bf16_bits_to_f64(x_bits)
    out = np.zeros((T, d), np.float64)
    wflat = w.reshape(-1)
    for e in range(E):
        rows = perm[offsets[e]:offsets[e + 1]]
        if rows.size == 0:
            continue
        t = rows // k
        wg, wu, wd = weights_fn(e)
        g, u = x[t] @ wg, x[t] @ wu
        h = g * sigmoid(g) * u
        if round_h:
            h = bf16_round(h)
        np.add.at(out, t, wflat[rows][:, None] * (h @ wd))
    return dict(idx=idx, w=w, out=out)


def backward(x_bits, logits, dout_bits, k, score_fn, E, weights_fn, experts=None,
             want_dx=True, exact=False, prepared=None, plain=False):
    """Oracle backward (quantised reading, see module docstring).

    Returns dict with dx [T,d] (fp64, contributions of the processed experts only when
    ``experts`` is given), dw [T,k], and dW = {e: (dWg [d,f], dWu [d,f], dWd [f,d])} for
    the processed experts.  ``prepared``: optional {e: ExpertWeights} whose quantised
    weight views are reused (weight preparation done ahead of time).

    ``plain=True`` swaps in the textbook alternatives of the two readings, for comparison
    only: the incoming-gradient operands of the weight gradients are quantised along the
    tokens straight from their unquantised values (bf16 dg, du; w * dOut), and
    d(combine weight) = <dOut_t, y_a> with the forward's expert output y_a.
    """
    T, d = x_bits.shape
    idx, w = rt.route(logits, k, score_fn)
    counts, offsets, perm, inv = rt.layout(idx, E)
    _, _, xhat = quantize_tokens(x_bits)
    if exact:
        xhat = bf16_bits_to_f64(x_bits)
    dout = bf16_bits_to_f64(dout_bits)
    dhat = _fq(dout, exact)
    wflat = w.reshape(-1)
    dx = np.zeros((T, d), np.float64)
    dw = np.zeros(T * k, np.float64)
    dW = {}
    todo = range(E) if experts is None else experts
    for e in todo:
        rows = perm[offsets[e]:offsets[e + 1]]
        W = prepared[e] if prepared and e in prepared else ExpertWeights(*weights_fn(e),
                                                                        exact=exact)
        f = W.wg.shape[1]
        if rows.size == 0:
            dW[e] = (np.zeros((d, f)), np.zeros((d, f)), np.zeros((f, d)))
            continue
        t = rows // k
        g, u, _, _, hhat, _ = expert_forward(xhat[t], W)
        gb, ub = _bf(g, exact), _bf(u, exact)                 # saved pre-activations
        wd_k, wgu_k = W.bwd()
        G = dhat[t] @ wd_k.T                                  # [n, f]
        if plain:
            y = hhat @ W.fwd()[2].T
            dw[rows] = np.sum(dout[t] * y, axis=1)
        else:
            dw[rows] = np.sum(G * hhat, axis=1)
        dh = wflat[rows][:, None] * G
        s = sigmoid(gb)
        dg = dh * ub * s * (1.0 + gb * (1.0 - s))
        du = dh * gb * s
        dgu_hat = _fq(np.concatenate([dg, du], axis=1), exact)
        if want_dx:
            np.add.at(dx, t, dgu_hat @ wgu_k.T)
        # weight gradients: the data path's MX operands requantised along the tokens
        if plain:
            dy = wflat[rows][:, None] * dout[t]
            DGt, DUt = _tok_fake(_bf(dg, exact), exact), _tok_fake(_bf(du, exact), exact)
        else:
            dy = wflat[rows][:, None] * dhat[t]
            DGt, DUt = _tok_fake(dgu_hat[:, :f], exact), _tok_fake(dgu_hat[:, f:], exact)
        Ht, DYt = _tok_fake(hhat, exact), _tok_fake(dy, exact)
        Xt = _tok_fake(xhat[t], exact)
        dW[e] = (Xt.T @ DGt, Xt.T @ DUt, Ht.T @ DYt)
    return dict(idx=idx, w=w, counts=counts, offsets=offsets, perm=perm, inv=inv,
                dx=dx, dw=dw.reshape(T, k), dW=dW)


def _tok_fake(v: np.ndarray, exact: bool = False) -> np.ndarray:
    """Quantise-dequantise a segment along its rows (tokens) in blocks of 32 (zero-padded)."""
    if exact:
        return np.asarray(v, np.float64)
    codes, scales = mx.quantize_mx_axis0_segment(v)
    vals = mx.e4m3_decode(codes) * np.repeat(mx.e8m0_decode(scales), 32, axis=0)
    return vals


# ---------------------------------------------------------------------------------------
# unquantised reference (informational, and the subject of the finite-difference pin)
# ---------------------------------------------------------------------------------------

def forward_exact(x, idx, w, weights):
    """out_t = sum_j w[t,j] * (silu(x_t Wg_e) * (x_t Wu_e)) Wd_e, all fp64, no quantisation.

    weights: list over experts of (Wg [d,f], Wu [d,f], Wd [f,d]).
    """
    T, k = idx.shape
    out = np.zeros((T, weights[0][0].shape[0]), np.float64)
    for t in range(T):
        for j in range(k):
            Wg, Wu, Wd = weights[int(idx[t, j])]
            g, u = x[t] @ Wg, x[t] @ Wu
            out[t] += w[t, j] * ((g * sigmoid(g) * u) @ Wd)
    return out


def backward_exact(x, idx, w, weights, dout):
    """Exact gradients of sum(dout * forward_exact) w.r.t. x, w and the expert weights."""
    T, k = idx.shape
    dx = np.zeros_like(x)
    dw = np.zeros_like(w)
    dW = [tuple(np.zeros_like(m) for m in W) for W in weights]
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            Wg, Wu, Wd = weights[e]
            g, u = x[t] @ Wg, x[t] @ Wu
            s = sigmoid(g)
            h = g * s * u
            y = h @ Wd
            dw[t, j] = dout[t] @ y
            dy = w[t, j] * dout[t]
            dh = Wd @ dy
            dg = dh * u * s * (1.0 + g * (1.0 - s))
            du = dh * g * s
            dx[t] += Wg @ dg + Wu @ du
            dW[e][0][...] += np.outer(x[t], dg)
            dW[e][1][...] += np.outer(x[t], du)
            dW[e][2][...] += np.outer(h, dy)
    return dx, dw, dW
