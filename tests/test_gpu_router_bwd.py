"""GPU parity of the router backward (d(logits) from d(combine weights)) against the oracle.

The unselected logits of a token must get exactly zero.  For the k selected ones the
device works in fp32 (expf, sums over k <= 32 terms), the oracle in fp64; the bound is
derived from the expression: each result is a weight-scaled difference of dw_i and the
weighted mean of dw, so its fp32 error is a few ulps of the magnitudes it is formed from,
|err_i| <= 1e-5 * c_i * (|dw_i| + sum_j w_j |dw_j|), with c_i = w_i (softmax over the
selected logits) or s_i (1 - s_i) / S (sigmoid scores renormalised).
"""
import numpy as np
import pytest

import synth
from oracle import routing as ort
from tests.gpu_util import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _check(moe, logits, k, score, seed):
    import torch
    lg = torch.from_numpy(logits).cuda()
    route = moe.route_layout(lg, k, score)
    idx = to_np(route["idx"]).astype(np.int64)
    rng = np.random.default_rng(seed)
    dw = rng.standard_normal(idx.shape).astype(np.float32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = to_np(moe.router_backward(lg, route["idx"], torch.from_numpy(dw).cuda(), score,
                                    status=status)).astype(np.float64)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = ort.routing_weights_backward(logits, idx, dw.astype(np.float64), score)
    sel = np.zeros(logits.shape, bool)
    np.put_along_axis(sel, idx, True, axis=1)
    assert np.all(got[~sel] == 0.0)                      # exactly zero off the selection
    w = ort.routing_weights(logits, idx, score)
    mag = np.abs(dw) + np.sum(w * np.abs(dw), axis=1, keepdims=True)
    if score == ort.SCORE_SOFTMAX_TOPK:
        c = w
    else:
        s = 1.0 / (1.0 + np.exp(-np.take_along_axis(logits.astype(np.float64), idx, axis=1)))
        c = s * (1 - s) / s.sum(axis=1, keepdims=True)
    bound = np.zeros(logits.shape)
    np.put_along_axis(bound, idx, 1e-5 * c * mag, axis=1)
    err = np.abs(got - ref)
    print(f"  max err / bound {np.max(err[sel] / bound[sel]):.3e}")
    assert np.all(err <= bound + 1e-30)


@pytest.mark.parametrize("name", ["tiny", "mid", "dsv3", "imbalance"])
def test_router_backward_configs(moe, name):
    case = synth.CONFIGS[name]
    _check(moe, synth.make_logits(case), case.k, case.score_fn, seed=5)


@pytest.mark.parametrize("T,E,k,score", [(1, 8, 1, 0), (1, 8, 1, 1), (77, 6, 6, 0),
                                         (77, 6, 6, 1), (300, 1024, 32, 1), (130, 33, 3, 0),
                                         (64, 10, 5, 1)])
def test_router_backward_edges(moe, T, E, k, score):
    rng = np.random.default_rng(T + 7 * E + k)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    _check(moe, logits, k, score, seed=T * E)


def test_router_backward_k1_is_zero_and_bad_index_latches(moe):
    import torch
    case = synth.CONFIGS["tiny"]
    lg = torch.from_numpy(synth.make_logits(case)).cuda()
    route = moe.route_layout(lg, 1, 0)
    dw = torch.ones((case.T, 1), dtype=torch.float32, device="cuda")
    dl = moe.router_backward(lg, route["idx"], dw, 0)
    torch.cuda.synchronize()
    assert not torch.any(dl != 0)                        # a single weight is constant 1
    bad = route["idx"].clone()
    bad[3, 0] = case.E + 2
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.router_backward(lg, bad, dw, 0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 7                       # MOE_ERR_DEVICE_BOUNDS, no fault
