"""Routing and per-expert layout -- the oracle's plain definitions.

Article ("Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72"):
* lead and §01: the router decides anew at every step which experts each token goes to;
  the configuration fixes the rule: top-k by logit, ties to the lower expert index.
* §01: the system must first count how many tokens each expert has, decide where each
  token is placed, and keep one expert's tokens contiguous (else the grouped GEMM has
  to reorder them again).
* §02 (pull dispatch): the consumer fetches the rows it needs by source and offset and
  lays them out by expert.

Readings (the pages are silent; listed in the design notes):
* slot j of a token is the rank of the expert in descending logit order (ties: lower id).
* selection is by logit, also for the sigmoid score function (sigmoid is monotone, so
  this equals selection by score in exact arithmetic and keeps the indices exact).
* within an expert's segment, rows are ordered by ascending token (a stable counting
  sort), which makes the layout unique; ``perm`` stores the assignment id a = t*k + j.
"""
from __future__ import annotations

import numpy as np

SCORE_SOFTMAX_TOPK = 0
SCORE_SIGMOID_RENORM = 1


def rank_keys(logits: np.ndarray, dtype=np.float32) -> np.ndarray:
    """The logits as ranking keys: a NaN logit ranks as -inf (the lowest key).

    Reading: the pages say nothing about invalid router outputs; a NaN must not be chosen
    ahead of any number, and when a row has fewer than k numbers the NaN experts are
    taken like -inf ones, lower index first.  The same keys feed the weights.
    """
    a = np.asarray(logits, dtype=dtype)
    return np.where(np.isnan(a), a.dtype.type(-np.inf), a)


def topk_select(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices [T, k] of the k largest logits per row, ties broken by the lower index.

    A stable ascending sort of -logit keeps equal keys in index order.
    """
    logits = rank_keys(logits)
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def topk_select_bruteforce(logits: np.ndarray, k: int) -> np.ndarray:
    """Per-token Python sort by the key (-logit, expert)."""
    out = []
    for row in rank_keys(logits):
        keyed = sorted(range(row.shape[0]), key=lambda e: (-float(row[e]), e))
        out.append(keyed[:k])
    return np.array(out, dtype=np.int32).reshape(len(out), k)


def routing_weights(logits: np.ndarray, idx: np.ndarray, score_fn: int) -> np.ndarray:
    """Combine weights [T, k] in fp64.

    softmax-top-k: softmax over the k selected logits (max subtracted).
    sigmoid-renorm: s = 1 / (1 + exp(-logit)) for the selected experts, w = s / sum(s).
    """
    sel = np.take_along_axis(rank_keys(logits, np.float64), idx.astype(np.int64), axis=1)
    if score_fn == SCORE_SOFTMAX_TOPK:
        z = np.exp(sel - sel.max(axis=1, keepdims=True))
        return z / z.sum(axis=1, keepdims=True)
    if score_fn == SCORE_SIGMOID_RENORM:
        s = 1.0 / (1.0 + np.exp(-sel))
        return s / s.sum(axis=1, keepdims=True)
    raise ValueError(score_fn)


def routing_weights_backward(logits: np.ndarray, idx: np.ndarray, dw: np.ndarray,
                             score_fn: int) -> np.ndarray:
    """d(loss)/d(logits) [T, E] in fp64 from d(loss)/d(combine weights) ``dw`` [T, k].

    The top-k selection is piecewise constant in the logits, so only the k selected
    logits of a token receive a gradient (the others get exactly zero); through the
    weights it is the chain rule of the two definitions above:
      softmax-top-k:  w = softmax(l_sel)         -> dl_i = w_i (dw_i - sum_j w_j dw_j)
      sigmoid-renorm: w = s / sum(s), s = sig(l) -> ds_i = (dw_i - sum_j w_j dw_j) / sum(s),
                                                     dl_i = ds_i s_i (1 - s_i)
    """
    logits = np.asarray(logits, np.float64)
    idx = idx.astype(np.int64)
    dw = np.asarray(dw, np.float64)
    w = routing_weights(logits, idx, score_fn)
    centred = dw - np.sum(w * dw, axis=1, keepdims=True)
    if score_fn == SCORE_SOFTMAX_TOPK:
        dsel = w * centred
    elif score_fn == SCORE_SIGMOID_RENORM:
        sel = np.take_along_axis(logits, idx, axis=1)
        s = 1.0 / (1.0 + np.exp(-sel))
        dsel = centred / s.sum(axis=1, keepdims=True) * s * (1.0 - s)
    else:
        raise ValueError(score_fn)
    out = np.zeros_like(logits)
    np.put_along_axis(out, idx, dsel, axis=1)
    return out


def route(logits: np.ndarray, k: int, score_fn: int):
    """Top-k indices [T,k] int32 and weights [T,k] float64."""
    idx = topk_select(logits, k)
    return idx, routing_weights(logits, idx, score_fn)


def layout(idx: np.ndarray, E: int):
    """counts [E], offsets [E+1], perm [A] (position -> assignment id), inv [A].

    counts[e] = #{a : idx[a] = e}; offsets is their exclusive prefix sum with
    offsets[E] = A; perm lists, expert by expert, the assignment ids in ascending
    token order; inv is the inverse permutation.
    """
    flat = np.asarray(idx, np.int64).ravel()
    A = flat.shape[0]
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv = np.empty(A, np.int32)
    inv[perm] = np.arange(A, dtype=np.int32)
    return counts, offsets, perm, inv


def layout_bruteforce(idx: np.ndarray, E: int):
    """Expert-by-expert, token-by-token loop building the same four arrays."""
    T, k = idx.shape
    counts = [0] * E
    perm = []
    offsets = [0]
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if int(idx[t, j]) == e:
                    perm.append(t * k + j)
                    counts[e] += 1
        offsets.append(len(perm))
    inv = [0] * len(perm)
    for p, a in enumerate(perm):
        inv[a] = p
    return (np.array(counts, np.int32), np.array(offsets, np.int32),
            np.array(perm, np.int32), np.array(inv, np.int32))


def padded_offsets(counts: np.ndarray, tile: int = 128) -> np.ndarray:
    """Exclusive prefix sum of the counts rounded up to a multiple of ``tile``.

    This is the expert-contiguous row layout of the permuted operand buffers in which
    every expert segment starts on a ``tile``-row boundary.
    """
    c = np.asarray(counts, np.int64)
    out = np.zeros(c.shape[0] + 1, np.int64)
    out[1:] = np.cumsum(-(-c // tile) * tile)
    return out.astype(np.int32)
