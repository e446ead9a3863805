"""moe_route_layout_noalloc: routing and layout for callers that cannot allocate device
memory (a plugin whose host framework owns the device memory, a fixed memory budget, or a
path that must not pay cudaMalloc's device synchronisation).  Its scratch is a fixed array
inside the library, so it takes no workspace.

Checked through the C ABI against moe_route_layout on two calls in a row with different
inputs (the second call must not see the first call's scratch contents): indices, counts,
offsets and permutations equal, weights within the routing tolerance.  This file sorts
last so that a run stopping at the first failure has run every other test already.
"""
import ctypes

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, dims, logits_t):
    import torch
    T, E = logits_t.shape
    k = dims.k
    dev = logits_t.device
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(idx=torch.full((T, k), -1, **i32),
               w=torch.full((T, k), -1.0, dtype=torch.float32, device=dev),
               counts=torch.full((E,), -1, **i32), offsets=torch.full((E + 1,), -1, **i32),
               perm=torch.full((T * k,), -1, **i32), inv=torch.full((T * k,), -1, **i32),
               pad=torch.full((E + 1,), -1, **i32), status=torch.zeros(1, **i32))
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.moe_route_layout_noalloc(
        ctypes.byref(dims), logits_t.data_ptr(), out["idx"].data_ptr(), out["w"].data_ptr(),
        out["counts"].data_ptr(), out["offsets"].data_ptr(), out["perm"].data_ptr(),
        out["inv"].data_ptr(), out["pad"].data_ptr(), out["status"].data_ptr(), stream)
    assert rc == 0, rc
    return out


def test_noalloc_matches_workspace_route_twice():
    import torch

    import token_dispatch_grouped_top_b200 as moe
    lib = moe.load()
    cases = [synth.CONFIGS["imbalance"], synth.CONFIGS["tiny"]]
    for case in cases:                       # two calls in a row, different shapes and data
        logits = torch.from_numpy(synth.make_logits(case)).cuda()
        dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn).c()
        got = _call_noalloc(lib, dims, logits)
        ref = moe.route_layout(logits, case.k, case.score_fn)
        torch.cuda.synchronize()
        assert moe.device_status(ref["ws"]) == 0
        assert int(got["status"].item()) == 0
        for a, b in (("idx", "idx"), ("counts", "counts"), ("offsets", "offsets"),
                     ("perm", "perm"), ("inv", "inv"), ("pad", "pad_offsets")):
            assert torch.equal(got[a], ref[b]), a
        dw = (got["w"].double() - ref["w"].double()).abs().max().item()
        assert dw <= 2e-6


def test_noalloc_rejects_too_large_before_launch():
    import token_dispatch_grouped_top_b200 as moe
    lib = moe.load()
    dims = moe.Dims(200000, 256, 256, 256, 8, 0).c()      # scratch above the 8 MiB array
    rc = lib.moe_route_layout_noalloc(ctypes.byref(dims), 1, 1, 1, 1, 1, 1, 1, None, None,
                                      None)
    assert rc == 2
