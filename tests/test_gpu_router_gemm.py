"""GPU parity of the router GEMM in front of the routing step (moe_router_logits) and its
backward (moe_router_grads), through the C ABI, against oracle.router.

* exact: small-integer operands keep every fp32 partial sum exact, so logits, dx_r and dW_r
  must equal the fp64 products bit for bit -- ragged T (swapped last tiles), E not a
  multiple of 256 (zero-padded N tiles, columns past E not stored), E < 128 in the weight
  gradient (a single partial M tile), several N tiles;
* random bf16 operands: every element within the fp32 summation bound
  2 K 2^-24 sum_i |a_i b_i| of the exact value (any summation order), and the relative
  Frobenius error below 1e-5;
* the route ranks the GPU's logits exactly as the oracle ranks them (indices bit-exact);
* the DeepSeek-V3 shape (T=8192, d=7168, E=256) in full.
"""
import numpy as np
import pytest

import synth
from oracle import router as orr
from oracle import routing as ort
from oracle.layer import bf16_bits_to_f64
from tests.gpu_util import bits_to_bf16_tensor, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _small_int_bits(rng, shape, lo=-8, hi=8):
    v = rng.integers(lo, hi + 1, shape).astype(np.float32)
    return synth.f32_to_bf16_bits(v)


def _abs_bound(a, b):
    """2 K 2^-24 (|a| @ |b|): the fp32 rounding bound of a K-term sum, any order."""
    return 2.0 * a.shape[1] * 2.0 ** -24 * (np.abs(a) @ np.abs(b)) + 1e-30


def _assert_within_sum_bound(got, ref, a, b):
    bound = _abs_bound(a, b)
    err = np.abs(got - ref)
    assert np.all(err <= bound), float(np.max(err / bound))
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert rel <= 1e-5, rel


SHAPES = [(1, 256, 8), (77, 512, 64), (300, 768, 256), (129, 2048, 24), (256, 256, 264),
          (640, 1024, 128)]


@pytest.mark.parametrize("T,d,E", SHAPES)
def test_router_logits_exact_small_integers(moe, T, d, E):
    import torch
    rng = np.random.default_rng(T + d + E)
    x, wr = _small_int_bits(rng, (T, d)), _small_int_bits(rng, (E, d))
    got = to_np(moe.router_logits(bits_to_bf16_tensor(x, "cuda"), bits_to_bf16_tensor(wr, "cuda")))
    torch.cuda.synchronize()
    assert np.array_equal(got.astype(np.float64), orr.router_logits(x, wr))


@pytest.mark.parametrize("T,d,E", SHAPES)
def test_router_grads_exact_small_integers(moe, T, d, E):
    import torch
    rng = np.random.default_rng(7 * T + d + E)
    x, wr = _small_int_bits(rng, (T, d)), _small_int_bits(rng, (E, d))
    g = rng.integers(-8, 9, (T, E)).astype(np.float32)
    dx, dw = moe.router_grads(torch.from_numpy(g).cuda(), bits_to_bf16_tensor(x, "cuda"),
                              bits_to_bf16_tensor(wr, "cuda"))
    torch.cuda.synchronize()
    rdx, rdw = orr.router_backward(g, x, wr)
    assert np.array_equal(to_np(dx).astype(np.float64), rdx)
    assert np.array_equal(to_np(dw).astype(np.float64), rdw)


def _random_case(moe, case):
    import torch
    x, wr = synth.make_x(case), synth.make_router_weight(case)
    xt, wt = bits_to_bf16_tensor(x, "cuda"), bits_to_bf16_tensor(wr, "cuda")
    logits = to_np(moe.router_logits(xt, wt))
    g = synth.make_dlogits(case)
    dx, dw = moe.router_grads(torch.from_numpy(g).cuda(), xt, wt)
    torch.cuda.synchronize()
    xf, wf = bf16_bits_to_f64(x), bf16_bits_to_f64(wr)
    _assert_within_sum_bound(logits.astype(np.float64), orr.router_logits(x, wr), xf, wf.T)
    rdx, rdw = orr.router_backward(g, x, wr)
    gb = orr.bf16_round(g.astype(np.float64))
    _assert_within_sum_bound(to_np(dx).astype(np.float64), rdx, gb, wf)
    _assert_within_sum_bound(to_np(dw).astype(np.float64), rdw, gb.T, xf)
    return logits


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_router_random_vs_oracle_and_route_chain(moe, name):
    import torch
    case = synth.CONFIGS[name]
    logits = _random_case(moe, case)
    # the route ranks the GPU's logits exactly as the oracle does
    r = moe.route_layout(torch.from_numpy(logits).cuda(), case.k, case.score_fn)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(r["idx"]), ort.topk_select(logits, case.k))


def test_router_dsv3_full(moe):
    _random_case(moe, synth.CONFIGS["dsv3"])


def test_router_grads_without_tokens(moe):
    import torch
    wr = bits_to_bf16_tensor(synth.make_router_weight(synth.CONFIGS["tiny"]), "cuda")
    x = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((0, 8), dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe._router_dims(0, 256, 8), moe.OP_ROUTER)
    dx, dw = moe.router_grads(g, x, wr, ws=ws)
    torch.cuda.synchronize()
    assert dx.shape == (0, 256) and not torch.any(dw != 0)
    assert moe.device_status(ws) == 0
