"""B200-native MoE layer hot path (route -> layout -> MXFP8 pull dispatch -> tcgen05 grouped
GEMM with SwiGLU -> push combine, and the backward pass).

This module is the thin Python binding over the C ABI of ``include/moe.h``: it allocates
device buffers with torch (memory and streams only) and passes raw pointers; every step of
the layer runs in the CUDA kernels of ``libmoe_b200.so``.  There is no CPU or PyTorch
fallback: if the library is missing, the calls raise.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field
from typing import Optional

from . import _lib
from ._lib import (MoeDims, MoeError, MoeSaved, MoeWeights, OP_BACKWARD, OP_FORWARD,
                   OP_FORWARD_BF16, OP_ROUTE, OP_ROUTER, SAVED_FIELDS, WEIGHT_FIELDS, WS_BUFFERS, check,
                   load)

SCORE_SOFTMAX_TOPK = 0
SCORE_SIGMOID_RENORM = 1

__all__ = ["Dims", "PreparedWeights", "Saved", "load", "MoeError", "workspace",
           "route_layout", "mxfp8_quantize", "prepare_weights", "forward", "backward",
           "grouped_gemm_mx", "grouped_gemm_bf16", "prepare_weights_bf16", "forward_bf16",
           "router_backward", "router_logits", "router_grads", "device_status", "padded_rows", "umma_scale_bytes",
           "min_tokens_for_waves", "workspace_view", "profile_enable", "profile_collect",
           "SCORE_SOFTMAX_TOPK", "SCORE_SIGMOID_RENORM"]


def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


@dataclass(frozen=True)
class Dims:
    T: int
    d: int
    f: int
    E: int
    k: int
    score_fn: int = SCORE_SOFTMAX_TOPK

    def c(self) -> MoeDims:
        return MoeDims(self.T, self.d, self.f, self.E, self.k, self.score_fn)

    @property
    def A(self) -> int:
        return self.T * self.k


def padded_rows(dims: Dims) -> int:
    v = load().moe_padded_rows(ctypes.byref(dims.c()))
    if v < 0:
        raise MoeError(2, "moe_padded_rows")
    return v


def umma_scale_bytes(rows: int, K: int) -> int:
    return load().moe_umma_scale_bytes(rows, K)


def min_tokens_for_waves(num_sms: int, waves: int, tile_m: int, tile_n: int, n_cols: int) -> int:
    return load().moe_min_tokens_for_waves(num_sms, waves, tile_m, tile_n, n_cols)


def workspace(dims: Dims, op: int, device="cuda"):
    """A zero-initialised workspace of moe_workspace_bytes(dims, op) bytes."""
    torch = _torch()
    n = load().moe_workspace_bytes(ctypes.byref(dims.c()), op)
    if n == 0:
        raise MoeError(2, "moe_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def workspace_view(ws, dims: Dims, op: int, name: str, nbytes: int):
    """A uint8 view of ``nbytes`` of an internal workspace buffer (moe_workspace_offset)."""
    off = load().moe_workspace_offset(ctypes.byref(dims.c()), op, WS_BUFFERS[name])
    if off < 0:
        raise MoeError(1, f"moe_workspace_offset({name})")
    return ws[off:off + nbytes]


def route_layout(logits, k: int, score_fn: int = SCORE_SOFTMAX_TOPK, ws=None, stream=None):
    """Routing and layout on the device.  Returns dict of idx, w, counts, offsets, perm, inv, pad_offsets."""
    torch = _torch()
    T, E = logits.shape
    dims = Dims(T, 256, 256, E, k, score_fn)
    dev = logits.device
    ws = workspace(dims, OP_ROUTE, dev) if ws is None else ws
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(idx=torch.empty((T, k), **i32), w=torch.empty((T, k), dtype=torch.float32,
                                                             device=dev),
               counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
               perm=torch.empty(T * k, **i32), inv=torch.empty(T * k, **i32),
               pad_offsets=torch.empty(E + 1, **i32))
    check(load().moe_route_layout(ctypes.byref(dims.c()), _ptr(logits.contiguous()),
                                  _ptr(out["idx"]), _ptr(out["w"]), _ptr(out["counts"]),
                                  _ptr(out["offsets"]), _ptr(out["perm"]), _ptr(out["inv"]),
                                  _ptr(out["pad_offsets"]), _ptr(ws), ws.numel(),
                                  _stream(stream)), "moe_route_layout")
    out["ws"] = ws
    return out


def mxfp8_quantize(x, scale_layout: int = 0, stream=None):
    """Rows of a bf16 matrix -> (E4M3 codes uint8 [rows, K], scale bytes)."""
    torch = _torch()
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, K = x.shape
    q = torch.empty((rows, K), dtype=torch.uint8, device=x.device)
    if scale_layout == 0:
        s = torch.empty((rows, K // 32), dtype=torch.uint8, device=x.device)
    else:
        s = torch.zeros(max(umma_scale_bytes(rows, K), 0), dtype=torch.uint8, device=x.device)
    check(load().mxfp8_quantize(_ptr(x), rows, K, x.stride(0), _ptr(q), _ptr(s), scale_layout,
                                _stream(stream)), "mxfp8_quantize")
    return q, s


@dataclass
class PreparedWeights:
    dims: Dims
    bufs: dict = field(default_factory=dict)

    def c(self) -> MoeWeights:
        return MoeWeights(*[_ptr(self.bufs.get(n)) for n in WEIGHT_FIELDS])


def prepare_weights(w_gate, w_up, w_down, dims: Dims, with_backward: bool = False, stream=None):
    """bf16 W_gate/W_up [E,d,f], W_down [E,f,d] -> MX weights in the grouped-GEMM layouts."""
    torch = _torch()
    lib = load()
    cd = dims.c()
    pw = PreparedWeights(dims)
    nfields = 8 if with_backward else 4
    for i in range(nfields):
        n = lib.moe_weights_bytes(ctypes.byref(cd), i)
        if n < 0:
            raise MoeError(2, "moe_weights_bytes")
        pw.bufs[WEIGHT_FIELDS[i]] = torch.empty(n, dtype=torch.uint8, device=w_gate.device)
    cw = pw.c()
    check(lib.moe_prepare_weights(ctypes.byref(cd), _ptr(w_gate.contiguous()),
                                  _ptr(w_up.contiguous()), _ptr(w_down.contiguous()),
                                  1 if with_backward else 0, ctypes.byref(cw), _stream(stream)),
          "moe_prepare_weights")
    return pw


@dataclass
class Saved:
    dims: Dims
    bufs: dict = field(default_factory=dict)

    def c(self) -> MoeSaved:
        return MoeSaved(*[_ptr(self.bufs[n]) for n in SAVED_FIELDS])


def alloc_saved(dims: Dims, device="cuda") -> Saved:
    torch = _torch()
    lib = load()
    cd = dims.c()
    sv = Saved(dims)
    dtypes = {"topk_idx": torch.int32, "topk_w": torch.float32, "counts": torch.int32,
              "offsets": torch.int32, "perm": torch.int32, "inv_perm": torch.int32,
              "pad_offsets": torch.int32, "gu": torch.bfloat16}
    for i, n in enumerate(SAVED_FIELDS):
        nbytes = lib.moe_saved_bytes(ctypes.byref(cd), i)
        dt = dtypes.get(n, torch.uint8)
        sv.bufs[n] = torch.empty(nbytes // torch.empty((), dtype=dt).element_size(), dtype=dt,
                                 device=device)
    return sv


def forward(x, logits, weights: PreparedWeights, save: bool = False, ws=None, out=None,
            saved: Optional[Saved] = None, stream=None):
    """The layer forward on the device.  Returns (out bf16 [T,d], Saved or None)."""
    torch = _torch()
    dims = weights.dims
    dev = x.device
    ws = workspace(dims, OP_FORWARD, dev) if ws is None else ws
    out = torch.empty((dims.T, dims.d), dtype=torch.bfloat16, device=dev) if out is None else out
    if save and saved is None:
        saved = alloc_saved(dims, dev)
    cw = weights.c()
    cs = saved.c() if saved is not None else None
    check(load().moe_forward(ctypes.byref(dims.c()), ctypes.byref(cw), _ptr(x), _ptr(logits),
                             _ptr(out), ctypes.byref(cs) if cs is not None else None, _ptr(ws),
                             ws.numel(), _stream(stream)), "moe_forward")
    return out, saved


def backward(dout, weights: PreparedWeights, saved: Saved, ws=None, stream=None, outs=None):
    """The layer backward.  Returns dict dx, dw_route, dWg, dWu, dWd."""
    torch = _torch()
    dims = weights.dims
    dev = dout.device
    ws = workspace(dims, OP_BACKWARD, dev) if ws is None else ws
    if outs is None:
        bf = dict(dtype=torch.bfloat16, device=dev)
        outs = dict(dx=torch.empty((dims.T, dims.d), **bf),
                    dw_route=torch.empty((dims.T, dims.k), dtype=torch.float32, device=dev),
                    dWg=torch.empty((dims.E, dims.d, dims.f), **bf),
                    dWu=torch.empty((dims.E, dims.d, dims.f), **bf),
                    dWd=torch.empty((dims.E, dims.f, dims.d), **bf))
    cw = weights.c()
    cs = saved.c()
    check(load().moe_backward(ctypes.byref(dims.c()), ctypes.byref(cw), ctypes.byref(cs),
                              _ptr(dout), _ptr(outs["dx"]), _ptr(outs["dw_route"]),
                              _ptr(outs["dWg"]), _ptr(outs["dWu"]), _ptr(outs["dWd"]), _ptr(ws),
                              ws.numel(), _stream(stream)), "moe_backward")
    return outs


def router_backward(logits, topk_idx, dw_route, score_fn: int = SCORE_SOFTMAX_TOPK,
                    status=None, stream=None):
    """d(loss)/d(logits) [T, E] fp32 from d(loss)/d(combine weights) [T, k]."""
    torch = _torch()
    T, E = logits.shape
    k = topk_idx.shape[1]
    dims = Dims(T, 256, 256, E, k, score_fn)
    dl = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    check(load().moe_router_backward(ctypes.byref(dims.c()), _ptr(logits.contiguous()),
                                     _ptr(topk_idx.contiguous()), _ptr(dw_route.contiguous()),
                                     _ptr(dl), _ptr(status), _stream(stream)),
          "moe_router_backward")
    return dl


def _router_dims(T: int, d: int, E: int) -> Dims:
    # the router calls read T, d and E; f, k and the score function only satisfy the rules
    return Dims(T, d, 256, E, 1, SCORE_SOFTMAX_TOPK)


def router_logits(x, wr, ws=None, out=None, stream=None):
    """logits [T, E] fp32 = x [T, d] bf16 . wr^T, wr [E, d] bf16 (one row per expert)."""
    torch = _torch()
    T, d = x.shape
    E = wr.shape[0]
    dims = _router_dims(T, d, E)
    ws = workspace(dims, OP_ROUTER, x.device) if ws is None else ws
    out = torch.empty((T, E), dtype=torch.float32, device=x.device) if out is None else out
    check(load().moe_router_logits(ctypes.byref(dims.c()), _ptr(x.contiguous()),
                                   _ptr(wr.contiguous()), _ptr(out), _ptr(ws), ws.numel(),
                                   _stream(stream)), "moe_router_logits")
    return out


def router_grads(dlogits, x, wr, ws=None, stream=None):
    """(dx_r [T, d] fp32, dwr [E, d] fp32) of logits = x . wr^T from d(loss)/d(logits),
    the gradient rounded to bf16 as the operand of both tensor-core products."""
    torch = _torch()
    T, d = x.shape
    E = wr.shape[0]
    dims = _router_dims(T, d, E)
    ws = workspace(dims, OP_ROUTER, x.device) if ws is None else ws
    dx = torch.empty((T, d), dtype=torch.float32, device=x.device)
    dw = torch.empty((E, d), dtype=torch.float32, device=x.device)
    check(load().moe_router_grads(ctypes.byref(dims.c()), _ptr(dlogits.contiguous()),
                                  _ptr(x.contiguous()), _ptr(wr.contiguous()), _ptr(dx),
                                  _ptr(dw), _ptr(ws), ws.numel(), _stream(stream)),
          "moe_router_grads")
    return dx, dw


@dataclass
class PreparedWeightsBf16:
    dims: Dims
    wgu_t: object = None     # [E*2f, d] bf16, gate/up interleaved in 128-row blocks
    wd_t: object = None      # [E*d, f] bf16


def prepare_weights_bf16(w_gate, w_up, w_down, dims: Dims, stream=None) -> PreparedWeightsBf16:
    """bf16 W_gate/W_up [E,d,f], W_down [E,f,d] -> the BF16 variant's GEMM layouts."""
    torch = _torch()
    dev = w_gate.device
    pw = PreparedWeightsBf16(dims)
    pw.wgu_t = torch.empty((dims.E * 2 * dims.f, dims.d), dtype=torch.bfloat16, device=dev)
    pw.wd_t = torch.empty((dims.E * dims.d, dims.f), dtype=torch.bfloat16, device=dev)
    check(load().moe_prepare_weights_bf16(ctypes.byref(dims.c()), _ptr(w_gate.contiguous()),
                                          _ptr(w_up.contiguous()), _ptr(w_down.contiguous()),
                                          _ptr(pw.wgu_t), _ptr(pw.wd_t), _stream(stream)),
          "moe_prepare_weights_bf16")
    return pw


def forward_bf16(x, logits, weights: PreparedWeightsBf16, ws=None, out=None, stream=None):
    """The layer's BF16 variant on the device.  Returns out bf16 [T,d]."""
    torch = _torch()
    dims = weights.dims
    ws = workspace(dims, OP_FORWARD_BF16, x.device) if ws is None else ws
    out = torch.empty((dims.T, dims.d), dtype=torch.bfloat16, device=x.device) if out is None \
        else out
    check(load().moe_forward_bf16(ctypes.byref(dims.c()), _ptr(weights.wgu_t),
                                  _ptr(weights.wd_t), _ptr(x), _ptr(logits), _ptr(out), _ptr(ws),
                                  ws.numel(), _stream(stream)), "moe_forward_bf16")
    return out


def grouped_gemm_bf16(mtile_prefix, a, b, N: int, rows_valid=None, ws=None, stream=None):
    """D[r, n] = sum_k A[r,k] B[g*N+n, k] with bf16 A [rows, K], B [G*N, K]; fp32 [rows, N]."""
    torch = _torch()
    G = mtile_prefix.numel() - 1
    rows, K = a.shape
    ws = torch.zeros(256, dtype=torch.uint8, device=a.device) if ws is None else ws
    d = torch.zeros((rows, N), dtype=torch.float32, device=a.device)
    check(load().moe_grouped_gemm_bf16(G, rows, N, K, _ptr(mtile_prefix), _ptr(rows_valid),
                                       _ptr(a), _ptr(b), _ptr(d), _ptr(ws), ws.numel(),
                                       _stream(stream)), "moe_grouped_gemm_bf16")
    return d


def grouped_gemm_mx(mtile_prefix, a_q, a_s, b_q, b_s, N: int, K: int, rows_valid=None,
                    ws=None, stream=None):
    """D[r, n] = sum_k A[r,k] B[g*N+n, k] over each group's 128-row tiles; fp32 [rows, N]."""
    torch = _torch()
    G = mtile_prefix.numel() - 1
    rows = a_q.shape[0]
    ws = torch.zeros(256, dtype=torch.uint8, device=a_q.device) if ws is None else ws
    d = torch.zeros((rows, N), dtype=torch.float32, device=a_q.device)
    check(load().moe_grouped_gemm_mx(G, rows, N, K, _ptr(mtile_prefix), _ptr(rows_valid),
                                     _ptr(a_q), _ptr(a_s), _ptr(b_q), _ptr(b_s), _ptr(d),
                                     _ptr(ws), ws.numel(), _stream(stream)),
          "moe_grouped_gemm_mx")
    return d


def profile_enable(on: bool = True) -> None:
    check(load().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def profile_collect() -> dict:
    """{stage: (total ms, launches)} of the stage launches recorded since the last collect."""
    n = len(_lib.STAGES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int32 * n)()
    check(load().moe_profile_collect(ms, cnt, n), "moe_profile_collect")
    return {name: (ms[i], cnt[i]) for i, name in enumerate(_lib.STAGES) if cnt[i]}


def device_status(ws, stream=None) -> int:
    """Synchronise and return (and clear) the status latched in a workspace."""
    code = ctypes.c_int32(0)
    check(load().moe_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(code)),
          "moe_get_device_status")
    return code.value
