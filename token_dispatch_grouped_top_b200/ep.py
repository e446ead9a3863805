"""Expert parallelism (argument marshalling for moe_ep_prepare / moe_ep_experts /
moe_ep_combine, and the peer table).

Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72", §01 and §02:
each rank owns E/G experts and routes its own tokens; the owner pulls the rows it needs
from the tokens' ranks, runs its grouped GEMMs and pushes the outputs back, where the
weighted merge runs.  A step is three phases, each started on every rank only once every
rank finished the previous one.

`forward_ranks` runs all ranks' phases on one GPU, in phase order (no kernel waits for
another: each phase's inputs are complete before it is launched); the peer table then
holds the other ranks' buffers on the same device.  On a multi-GPU node each rank runs
its own phases, the table's entries are peer mappings of the other GPUs' buffers (each
rank exports its buffers with CUDA IPC or allocates them in symmetric memory), gathered
with `gather_entries`, and a barrier separates the phases.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

from ._lib import EP_PEER_FIELDS, MoeEpPeer, OP_ROUTE, check, load


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


@dataclass
class RankState:
    """One rank's phase-1 outputs and its receive buffers for the pushed expert outputs."""
    T: int
    bufs: dict = field(default_factory=dict)

    def entry(self) -> dict:
        """This rank's peer-table entry: T and the device addresses of its buffers."""
        e = {"T": self.T}
        e.update({n: _ptr(self.bufs[n]) for n in EP_PEER_FIELDS})
        return e


def _alloc_state(dims, dev) -> RankState:
    torch = _torch()
    T, d, k, E = dims.T, dims.d, dims.k, dims.E
    i32 = dict(dtype=torch.int32, device=dev)
    st = RankState(T)
    b = st.bufs
    b["topk_idx"] = torch.empty((T, k), **i32)
    b["topk_w"] = torch.empty((T, k), dtype=torch.float32, device=dev)
    b["counts"] = torch.empty(E, **i32)
    b["offsets"] = torch.empty(E + 1, **i32)
    b["perm"] = torch.empty(max(T * k, 1), **i32)
    b["inv_perm"] = torch.empty(max(T * k, 1), **i32)
    b["xq"] = torch.empty((max(T, 1), d), dtype=torch.uint8, device=dev)
    b["xs"] = torch.empty((max(T, 1), d // 32), dtype=torch.uint8, device=dev)
    b["y"] = torch.empty((max(T * k, 1), d), dtype=torch.float16, device=dev)
    b["ys"] = torch.empty((max(T * k, 1), d // 32), dtype=torch.uint8, device=dev)
    return st


def prepare(dims, x, logits, ws=None, state=None, stream=None) -> RankState:
    """Phase 1 on this rank: route + layout of its T tokens and their MX quantisation.
    Allocates the rank's buffers (among them the [T*k, d] receive buffers the owners push
    into), or refills those of `state`."""
    from . import workspace
    dev = x.device
    ws = workspace(dims, OP_ROUTE, dev) if ws is None else ws
    st = _alloc_state(dims, dev) if state is None else state
    b = st.bufs
    check(load().moe_ep_prepare(ctypes.byref(dims.c()), _ptr(x), _ptr(logits),
                                _ptr(b["topk_idx"]), _ptr(b["topk_w"]), _ptr(b["counts"]),
                                _ptr(b["offsets"]), _ptr(b["perm"]), _ptr(b["inv_perm"]),
                                _ptr(b["xq"]), _ptr(b["xs"]), _ptr(ws), ws.numel(),
                                _stream(stream)), "moe_ep_prepare")
    return st


def peer_table(entries: list, device) -> object:
    """The moe_ep_peer array (one entry per rank, in rank order) as a device byte tensor."""
    torch = _torch()
    arr = (MoeEpPeer * len(entries))()
    for i, e in enumerate(entries):
        arr[i].T = int(e["T"])
        for n in EP_PEER_FIELDS:
            setattr(arr[i], n, int(e[n]) if e[n] else None)
    raw = bytes(arr)
    return torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(device)


def gather_entries(entry: dict, group=None, map_fn=None) -> list:
    """Every rank's entry, in rank order, through torch.distributed (any backend).

    map_fn(rank, entry) -> entry turns a remote rank's exported buffers into addresses this
    GPU can load from and store to (a peer mapping); None keeps the addresses as they are
    (ranks that share one device)."""
    import torch.distributed as dist
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, entry, group=group)
    me = dist.get_rank(group)
    if map_fn is not None:
        out = [e if r == me else map_fn(r, e) for r, e in enumerate(out)]
    return out


def workspace_bytes(dims_all, world: int) -> int:
    """moe_ep_experts workspace for dims_all (T = every rank's tokens together)."""
    return int(load().moe_ep_workspace_bytes(ctypes.byref(dims_all.c()), world))


def experts(dims_all, rank: int, world: int, table, weights_local, ws=None, stream=None):
    """Phase 2 on `rank`: pull its experts' rows from every rank, run its grouped GEMMs,
    push the outputs back.  weights_local: prepare_weights of its E/G experts."""
    torch = _torch()
    if ws is None:
        n = workspace_bytes(dims_all, world)
        if n == 0:
            check(2, "moe_ep_workspace_bytes")
        ws = torch.zeros(n, dtype=torch.uint8, device=table.device)
    cw = weights_local.c()
    check(load().moe_ep_experts(ctypes.byref(dims_all.c()), rank, world, _ptr(table),
                                ctypes.byref(cw), _ptr(ws), ws.numel(), _stream(stream)),
          "moe_ep_experts")
    return ws


def combine(dims, state: RankState, out=None, status=None, stream=None):
    """Phase 3 on this rank: out[t] = sum_j w[t,j] * y[t*k + j] (bf16)."""
    torch = _torch()
    b = state.bufs
    out = torch.empty((dims.T, dims.d), dtype=torch.bfloat16, device=b["y"].device) \
        if out is None else out
    check(load().moe_ep_combine(ctypes.byref(dims.c()), _ptr(b["topk_w"]), _ptr(b["y"]),
                                _ptr(b["ys"]), _ptr(out), _ptr(status), _stream(stream)),
          "moe_ep_combine")
    return out


def forward_ranks(xs: list, logits: list, weights_local: list, d: int, f: int, E: int, k: int,
                  score_fn: int, stream=None):
    """All ranks' three phases on one GPU, in phase order.  xs[r] [T_r, d] bf16, logits[r]
    [T_r, E] fp32, weights_local[r] the prepared weights of rank r's E/G experts.
    Returns (outs, states, workspaces)."""
    from . import Dims
    world = len(xs)
    dev = xs[0].device
    dims_r = [Dims(int(x.shape[0]), d, f, E, k, score_fn) for x in xs]
    states = [prepare(dims_r[r], xs[r], logits[r], stream=stream) for r in range(world)]
    table = peer_table([s.entry() for s in states], dev)
    dims_all = Dims(sum(int(x.shape[0]) for x in xs), d, f, E, k, score_fn)
    wss = [experts(dims_all, r, world, table, weights_local[r], stream=stream)
           for r in range(world)]
    outs = [combine(dims_r[r], states[r], stream=stream) for r in range(world)]
    return outs, states, wss
