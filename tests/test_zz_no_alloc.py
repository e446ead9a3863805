"""moe_route_layout_noalloc: routing and layout for callers that cannot allocate device
memory (a plugin whose host framework owns the device memory, a fixed memory budget, or a
path that must not pay cudaMalloc's device synchronisation).  Its scratch is a fixed array
inside the library, so it takes no workspace.

Checked through the C ABI against moe_route_layout and against the oracle on calls in a
row with different inputs (a later call must not see an earlier call's scratch contents):
indices, counts, offsets and permutations equal, weights within the routing tolerance.
Also: no tokens, a missing status word, and a problem whose scratch fills the 8 MiB array
exactly.  This file sorts last so that a run stopping at the first failure has run every
other test already.
"""
import ctypes

import numpy as np
import pytest

import synth
from oracle import routing as ort

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, dims, logits_t, with_status=True):
    import torch
    T, E = logits_t.shape
    k = dims.k
    dev = logits_t.device
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(idx=torch.full((max(T, 1), k), -1, **i32),
               w=torch.full((max(T, 1), k), -1.0, dtype=torch.float32, device=dev),
               counts=torch.full((E,), -1, **i32), offsets=torch.full((E + 1,), -1, **i32),
               perm=torch.full((max(T, 1) * k,), -1, **i32),
               inv=torch.full((max(T, 1) * k,), -1, **i32),
               pad=torch.full((E + 1,), -1, **i32), status=torch.zeros(1, **i32))
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.moe_route_layout_noalloc(
        ctypes.byref(dims), logits_t.data_ptr() if T else None, out["idx"].data_ptr(),
        out["w"].data_ptr(), out["counts"].data_ptr(), out["offsets"].data_ptr(),
        out["perm"].data_ptr(), out["inv"].data_ptr(), out["pad"].data_ptr(),
        out["status"].data_ptr() if with_status else None, stream)
    return rc, out


def _check_against_workspace_and_oracle(moe, got, logits_t, logits_np, case):
    import torch
    ref = moe.route_layout(logits_t, case.k, case.score_fn)
    torch.cuda.synchronize()
    assert moe.device_status(ref["ws"]) == 0
    assert int(got["status"].item()) == 0
    for a, b in (("idx", "idx"), ("counts", "counts"), ("offsets", "offsets"),
                 ("perm", "perm"), ("inv", "inv"), ("pad", "pad_offsets")):
        assert torch.equal(got[a], ref[b]), a
    dw = (got["w"].double() - ref["w"].double()).abs().max().item()
    assert dw <= 2e-6
    idx, w = ort.route(logits_np, case.k, case.score_fn)
    counts, offsets, perm, inv = ort.layout(idx, case.E)
    assert np.array_equal(got["idx"].cpu().numpy(), idx)
    assert np.max(np.abs(got["w"].cpu().numpy() - w)) <= 2e-6
    for key, want in (("counts", counts), ("offsets", offsets), ("perm", perm), ("inv", inv),
                      ("pad", ort.padded_offsets(counts))):
        assert np.array_equal(got[key].cpu().numpy(), want), key


def test_noalloc_matches_workspace_route_and_oracle_twice():
    import torch

    import token_dispatch_grouped_top_b200 as moe
    lib = moe.load()
    cases = [synth.CONFIGS["imbalance"], synth.CONFIGS["tiny"]]
    for case in cases:                       # two calls in a row, different shapes and data
        logits_np = synth.make_logits(case)
        logits = torch.from_numpy(logits_np).cuda()
        dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn).c()
        rc, got = _call_noalloc(lib, dims, logits)
        assert rc == 0, rc
        _check_against_workspace_and_oracle(moe, got, logits, logits_np, case)


def test_noalloc_at_the_scratch_limit():
    # E = 256, k = 8, T = 131024 needs exactly the 8 MiB of the array; one token more is
    # rejected before anything is launched
    import torch

    import token_dispatch_grouped_top_b200 as moe
    lib = moe.load()
    case = synth.MoeCase("limit", 131024, 256, 256, 256, 8, 1, "normal0.5", seed=21)
    logits_np = synth.make_logits(case)
    logits = torch.from_numpy(logits_np).cuda()
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn).c()
    rc, got = _call_noalloc(lib, dims, logits)
    assert rc == 0, rc
    _check_against_workspace_and_oracle(moe, got, logits, logits_np, case)
    big = moe.Dims(case.T + 1, case.d, case.f, case.E, case.k, case.score_fn).c()
    assert lib.moe_route_layout_noalloc(ctypes.byref(big), 1, 1, 1, 1, 1, 1, 1, None, 1,
                                        None) == 2


def test_noalloc_no_tokens_and_missing_status():
    import torch

    import token_dispatch_grouped_top_b200 as moe
    lib = moe.load()
    empty = torch.empty((0, 8), dtype=torch.float32, device="cuda")
    dims = moe.Dims(0, 256, 256, 8, 2, 0).c()
    rc, got = _call_noalloc(lib, dims, empty)
    torch.cuda.synchronize()
    assert rc == 0
    assert not torch.any(got["counts"]) and not torch.any(got["offsets"])
    assert not torch.any(got["pad"])
    case = synth.CONFIGS["tiny"]
    logits = torch.from_numpy(synth.make_logits(case)).cuda()
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn).c()
    rc, _ = _call_noalloc(lib, dims, logits, with_status=False)
    assert rc == 1                           # the status word is required when T > 0


def test_noalloc_rejects_too_large_before_launch():
    import token_dispatch_grouped_top_b200 as moe
    lib = moe.load()
    dims = moe.Dims(200000, 256, 256, 256, 8, 0).c()      # scratch above the 8 MiB array
    rc = lib.moe_route_layout_noalloc(ctypes.byref(dims), 1, 1, 1, 1, 1, 1, 1, None, None,
                                      None)
    assert rc == 2
