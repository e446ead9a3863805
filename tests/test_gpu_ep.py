"""Expert parallelism through the C ABI, its ranks run on one GPU in phase order:
each rank's buffers are separate allocations reached through the peer table, and every
phase is launched only after the previous phase of all ranks (no kernel waits for another).

* each rank's output equals the single-GPU layer (moe_forward on that rank's tokens with
  all experts) bit for bit: the same routing, the same MX operands and per-row arithmetic;
  only the rows' placement in the GEMM tiles differs;
* and is within the layer tolerance of the fp64 oracle;
* uneven ranks, a rank without tokens, experts without tokens, one rank;
* a corrupted count is caught: MOE_ERR_DEVICE_BOUNDS latched, nothing received, no fault.
"""
import numpy as np
import pytest

import synth
from oracle import layer as olayer
from tests.gpu_util import assert_close_out, bf16_tensor_f64, bits_to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _split(case, sizes):
    import torch
    assert sum(sizes) == case.T
    x_all = bits_to_bf16_tensor(synth.make_x(case), "cuda")
    lg_all = torch.from_numpy(synth.make_logits(case)).cuda()
    cuts = np.concatenate([[0], np.cumsum(sizes)])
    xs = [x_all[cuts[r]:cuts[r + 1]].contiguous() for r in range(len(sizes))]
    lgs = [lg_all[cuts[r]:cuts[r + 1]].contiguous() for r in range(len(sizes))]
    return xs, lgs, cuts


def _run(moe, case, sizes, world):
    import torch
    from token_dispatch_grouped_top_b200 import ep
    wg, wu, wd = synth.expert_weights_torch(case, "cuda")
    E_loc = case.E // world
    wl = []
    for r in range(world):
        sl = slice(r * E_loc, (r + 1) * E_loc)
        dl = moe.Dims(case.T, case.d, case.f, E_loc, min(case.k, E_loc), case.score_fn)
        wl.append(moe.prepare_weights(wg[sl].contiguous(), wu[sl].contiguous(),
                                      wd[sl].contiguous(), dl))
    full = moe.prepare_weights(wg, wu, wd, moe.Dims(case.T, case.d, case.f, case.E, case.k,
                                                   case.score_fn))
    del wg, wu, wd
    xs, lgs, cuts = _split(case, sizes)
    outs, states, wss = ep.forward_ranks(xs, lgs, wl, case.d, case.f, case.E, case.k,
                                         case.score_fn)
    torch.cuda.synchronize()
    for ws in wss:
        assert moe.device_status(ws) == 0
    for r in range(world):
        if sizes[r] == 0:
            assert outs[r].shape == (0, case.d)
            continue
        dims_r = moe.Dims(sizes[r], case.d, case.f, case.E, case.k, case.score_fn)
        full.dims = dims_r
        single, _ = moe.forward(xs[r], lgs[r], full)
        torch.cuda.synchronize()
        assert torch.equal(outs[r].view(torch.int16), single.view(torch.int16)), r
    return outs, cuts


@pytest.mark.parametrize("world,sizes", [(2, [256, 256]), (4, [100, 212, 0, 200]),
                                         (1, [512])])
def test_ep_tiny_matches_single_gpu_and_oracle(moe, world, sizes):
    case = synth.CONFIGS["tiny"]
    outs, cuts = _run(moe, case, sizes, world)
    got = np.concatenate([bf16_tensor_f64(o) for o in outs if o.shape[0]], axis=0)
    ref = olayer.forward(synth.make_x(case), synth.make_logits(case), case.k, case.score_fn,
                         case.E, lambda e: synth.expert_weights_f64(case, e))["out"]
    assert_close_out(got, ref)


def test_ep_skewed_uneven_ranks(moe):
    # skewed load: some experts receive nothing, some rows come from one rank only
    case = synth.MoeCase("ep_skew", 600, 256, 512, 12, 3, 0, "skew1.5", seed=17)
    _run(moe, case, [300, 0, 123, 177], 4)


def test_ep_mid_four_ranks(moe):
    case = synth.CONFIGS["mid"]
    _run(moe, case, [1000, 1100, 996, 1000], 4)


def test_ep_corrupted_count_latches_bounds(moe):
    import torch
    from token_dispatch_grouped_top_b200 import ep
    case = synth.CONFIGS["tiny"]
    world, E_loc = 2, case.E // 2
    wg, wu, wd = synth.expert_weights_torch(case, "cuda")
    dl = moe.Dims(case.T, case.d, case.f, E_loc, case.k, case.score_fn)
    wl = [moe.prepare_weights(wg[r * E_loc:(r + 1) * E_loc].contiguous(),
                              wu[r * E_loc:(r + 1) * E_loc].contiguous(),
                              wd[r * E_loc:(r + 1) * E_loc].contiguous(), dl)
          for r in range(world)]
    xs, lgs, _ = _split(case, [256, 256])
    dims_r = [moe.Dims(256, case.d, case.f, case.E, case.k, case.score_fn)] * world
    states = [ep.prepare(dims_r[r], xs[r], lgs[r]) for r in range(world)]
    states[1].bufs["counts"][0] = -5            # rank 1 claims a negative count for expert 0
    table = ep.peer_table([s.entry() for s in states], "cuda")
    dims_all = moe.Dims(512, case.d, case.f, case.E, case.k, case.score_fn)
    ws0 = ep.experts(dims_all, 0, world, table, wl[0])
    ws1 = ep.experts(dims_all, 1, world, table, wl[1])
    torch.cuda.synchronize()
    assert moe.device_status(ws0) == 7          # MOE_ERR_DEVICE_BOUNDS, rank 0 owns expert 0
    assert moe.device_status(ws1) == 0
