"""The device-side tile scheduler: readiness signalling between the dispatch and the grouped
GEMM, and its failure detection, on the GPU through the C ABI.

* The dispatch publishes each minibatch of rows through a device-local count-down counter
  and the gate/up GEMM (launched while the dispatch still runs) waits for it.  With the
  test hook withholding one minibatch, the GEMM's bounded wait gives up after its limit
  (2 s), MOE_ERR_DEVICE_TIMEOUT (6) is latched and read back, and the next call, hook
  off, is correct again: the context stays usable, nothing faults or hangs.
* Results do not depend on the scheduling: runs agree bit for bit, and the weight
  gradients (handed out longest expert first) agree with the oracle in the backward tests.
"""
import numpy as np
import pytest

import synth
from oracle import routing as ort
from tests.gpu_util import assert_close_out, bf16_tensor_f64, bits_to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _setup(moe, case, backward=False):
    import torch
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    wg, wu, wd = synth.expert_weights_torch(case, "cuda")
    pw = moe.prepare_weights(wg, wu, wd, dims, with_backward=backward)
    x = bits_to_bf16_tensor(synth.make_x(case), "cuda")
    lg = torch.from_numpy(synth.make_logits(case)).cuda()
    return dims, pw, x, lg


@pytest.mark.parametrize("name,batch", [("tiny", 0), ("mid", 3)])
def test_withheld_minibatch_times_out_and_context_recovers(moe, name, batch):
    import torch
    case = synth.CONFIGS[name]
    dims, pw, x, lg = _setup(moe, case)
    ws = moe.workspace(dims, moe.OP_FORWARD)
    good, _ = moe.forward(x, lg, pw, ws=ws)
    good = good.clone()
    assert moe.device_status(ws) == 0
    # the minibatch exists: mid has several (two waves of 128 x 256 tiles each)
    counts = np.bincount(ort.topk_select(synth.make_logits(case), case.k).ravel(),
                         minlength=case.E)
    rows = int(ort.padded_offsets(counts)[-1])
    mb = -(-moe.min_tokens_for_waves(torch.cuda.get_device_properties(0).multi_processor_count,
                                     2, 128, 256, 2 * case.f) // 128) * 128
    assert batch * mb < rows
    lib = moe.load()
    assert lib.moe_debug_withhold_ready(batch) == 0
    try:
        moe.forward(x, lg, pw, ws=ws)
        torch.cuda.synchronize()
    finally:
        assert lib.moe_debug_withhold_ready(-1) == 0
    assert moe.device_status(ws) == 6                 # MOE_ERR_DEVICE_TIMEOUT, read back
    again, _ = moe.forward(x, lg, pw, ws=ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    assert torch.equal(again, good)


def test_withheld_minibatch_in_backward_times_out(moe):
    import torch
    case = synth.MoeCase("sched_b", 300, 256, 512, 8, 2, 0, "skew1.5", seed=51)
    dims, pw, x, lg = _setup(moe, case, backward=True)
    wsf = moe.workspace(dims, moe.OP_FORWARD)
    _, saved = moe.forward(x, lg, pw, save=True, ws=wsf)
    dout = bits_to_bf16_tensor(synth.make_dout(case), "cuda")
    wsb = moe.workspace(dims, moe.OP_BACKWARD)
    ref = {k: v.clone() for k, v in moe.backward(dout, pw, saved, ws=wsb).items()}
    assert moe.device_status(wsb) == 0
    lib = moe.load()
    assert lib.moe_debug_withhold_ready(0) == 0
    try:
        moe.backward(dout, pw, saved, ws=wsb)
        torch.cuda.synchronize()
    finally:
        assert lib.moe_debug_withhold_ready(-1) == 0
    assert moe.device_status(wsb) == 6
    grads = moe.backward(dout, pw, saved, ws=wsb)
    torch.cuda.synchronize()
    assert moe.device_status(wsb) == 0
    for k in ref:
        assert torch.equal(grads[k], ref[k]), k


def test_scheduling_is_deterministic_under_imbalance(moe):
    # the dynamic tile order differs from run to run; every tile's result does not
    import torch
    case = synth.CONFIGS["imbalance"].replace(T=2048, d=512, f=256, name="imb_small")
    dims, pw, x, lg = _setup(moe, case, backward=True)
    ws = moe.workspace(dims, moe.OP_FORWARD)
    wsb = moe.workspace(dims, moe.OP_BACKWARD)
    dout = bits_to_bf16_tensor(synth.make_dout(case), "cuda")
    outs = []
    for _ in range(3):
        o, saved = moe.forward(x, lg, pw, save=True, ws=ws)
        g = moe.backward(dout, pw, saved, ws=wsb)
        outs.append((o.clone(), {k: v.clone() for k, v in g.items()}))
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0 and moe.device_status(wsb) == 0
    for o, g in outs[1:]:
        assert torch.equal(o, outs[0][0])
        for k in g:
            assert torch.equal(g[k], outs[0][1][k]), k
    # the empty experts' gradients are zero, the hot ones' are not
    counts = to_counts(case)
    for e in np.flatnonzero(counts == 0)[:3]:
        assert not torch.any(outs[0][1]["dWd"][e].float() != 0)
    hot = int(np.argmax(counts))
    assert torch.any(outs[0][1]["dWd"][hot].float() != 0)


def to_counts(case):
    return np.bincount(ort.topk_select(synth.make_logits(case), case.k).ravel(),
                       minlength=case.E)


def test_forward_mid_matches_oracle_with_overlap(moe):
    # the gate/up GEMM runs while the dispatch writes rows; sampled tokens vs the oracle
    import torch
    from oracle import layer as olayer
    case = synth.CONFIGS["mid"]
    dims, pw, x, lg = _setup(moe, case)
    out, _ = moe.forward(x, lg, pw)
    torch.cuda.synchronize()
    toks = np.arange(0, case.T, 97)
    ref = olayer.forward(synth.make_x(case), synth.make_logits(case), case.k, case.score_fn,
                         case.E, lambda e: synth.expert_weights_f64(case, e), tokens=toks)
    assert_close_out(bf16_tensor_f64(out)[toks], ref["out"][toks])
