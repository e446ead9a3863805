"""GPU parity of routing + layout and of the MXFP8 quantiser, through the C ABI.

Routing indices, counts, offsets, perm and inv must equal the oracle bit for bit; routing
weights within 2e-6 (fp32 expf vs fp64 exp); quantised bytes and scales bit-exact.
"""
import numpy as np
import pytest

import synth
from oracle import mxfp8 as omx
from oracle import routing as ort
from tests.gpu_util import bits_to_bf16_tensor, to_np, umma_to_canonical

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _route_check(moe, logits, k, score_fn):
    import torch
    E = logits.shape[1]
    res = moe.route_layout(torch.from_numpy(logits).cuda(), k, score_fn)
    assert moe.device_status(res["ws"]) == 0
    idx, w = ort.route(logits, k, score_fn)
    counts, offsets, perm, inv = ort.layout(idx, E)
    assert np.array_equal(to_np(res["idx"]), idx)
    assert np.max(np.abs(to_np(res["w"]).astype(np.float64) - w)) <= 2e-6
    assert np.array_equal(to_np(res["counts"]), counts)
    assert np.array_equal(to_np(res["offsets"]), offsets)
    assert np.array_equal(to_np(res["perm"]), perm)
    assert np.array_equal(to_np(res["inv"]), inv)
    assert np.array_equal(to_np(res["pad_offsets"]), ort.padded_offsets(counts))
    return res


@pytest.mark.parametrize("name", ["tiny", "mid", "dsv3", "imbalance"])
def test_route_layout_configs(moe, name):
    case = synth.CONFIGS[name]
    _route_check(moe, synth.make_logits(case), case.k, case.score_fn)


@pytest.mark.parametrize("T,E,k,score", [(1, 8, 2, 0), (1, 4, 4, 1), (63, 8, 8, 0), (65, 5, 1, 1),
                                         (300, 1024, 32, 0), (200, 33, 3, 1), (130, 1, 1, 0)])
def test_route_layout_edges(moe, T, E, k, score):
    rng = np.random.default_rng(T * 31 + E)
    lg = rng.integers(-4, 5, (T, E)).astype(np.float32) * np.float32(0.25)   # many exact ties
    _route_check(moe, lg, k, score)


def test_route_signed_zero_ties(moe):
    # rows of -0, +0, 1, -1: -0 and +0 tie (lower index first) whichever sign comes first
    rng = np.random.default_rng(23)
    lg = rng.choice(np.array([-0.0, 0.0, 1.0, -1.0], np.float32), (700, 64))
    _route_check(moe, lg, 6, 0)


@pytest.mark.parametrize("T,E,k", [(20000, 96, 6), (9000, 256, 8), (17000, 1024, 4)])
def test_route_many_tiles(moe, T, E, k):
    # more than 128 tiles of 64 tokens: the lookback runs over several flag windows
    rng = np.random.default_rng(T + E)
    lg = (rng.normal(size=(T, E)) + np.linspace(0, 2, E)).astype(np.float32)
    _route_check(moe, lg, k, 1)


def test_route_all_tokens_one_expert_and_empty_batch(moe):
    import torch
    T, E = 500, 16
    lg = np.full((T, E), -1.0, np.float32)
    lg[:, 11] = 3.0
    _route_check(moe, lg, 1, 0)
    res = moe.route_layout(torch.zeros((0, E), device="cuda"), 2, 0)
    assert moe.device_status(res["ws"]) == 0
    assert not to_np(res["counts"]).any() and not to_np(res["offsets"]).any()


@pytest.mark.parametrize("score", [0, 1])
def test_route_nan_logits_rank_as_minus_infinity(moe, score):
    # Rows with a few NaN logits, rows with fewer than k numbers and all-NaN rows: every
    # index stays a valid expert (the oracle's reading: a NaN ranks as -inf) and no device
    # error is latched.  Weights of rows that had to take -inf experts may be NaN on both
    # sides (0/0); they must be NaN at the same places and close elsewhere.
    import torch
    T, E, k = 300, 40, 6
    rng = np.random.default_rng(17 + score)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[rng.random((T, E)) < 0.1] = np.nan
    lg[::7, 3:] = np.nan                    # only 3 numbers left in these rows
    lg[::11] = np.nan                       # nothing but NaN
    lg[5, :10] = -np.inf
    res = moe.route_layout(torch.from_numpy(lg).cuda(), k, score)
    assert moe.device_status(res["ws"]) == 0
    idx, w = ort.route(lg, k, score)
    counts, offsets, perm, inv = ort.layout(idx, E)
    assert np.array_equal(to_np(res["idx"]), idx)
    gw = to_np(res["w"]).astype(np.float64)
    assert np.array_equal(np.isnan(gw), np.isnan(w))
    ok = ~np.isnan(w)
    assert np.max(np.abs(gw[ok] - w[ok])) <= 2e-6
    for key, want in (("counts", counts), ("offsets", offsets), ("perm", perm), ("inv", inv)):
        assert np.array_equal(to_np(res[key]), want), key


def test_route_deterministic(moe):
    import torch
    case = synth.CONFIGS["imbalance"]
    lg = torch.from_numpy(synth.make_logits(case)).cuda()
    ref = moe.route_layout(lg, case.k, case.score_fn)
    for _ in range(5):
        again = moe.route_layout(lg, case.k, case.score_fn)
        for key in ("idx", "perm", "inv", "offsets"):
            assert torch.equal(again[key], ref[key])


def test_mxfp8_edge_codes(moe):
    """Every block holds 448 (scale 2^0), so each edge value is converted as is: ties to even,
    saturation, subnormals and the sign of values that round to zero."""
    vals = [0.0, -0.0, 1.0, -1.0, 448.0, 464.0, 480.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10,
            1.0625, 1.1875, 2.0 ** -6, -(2.0 ** -11), 255.0, 256.0, 510.0, -464.0, 15 * 2.0 ** -10,
            -(2.0 ** -10), 7 * 2.0 ** -9, -(3 * 2.0 ** -10)]
    x = np.zeros((len(vals), 32), np.float32)
    x[:, 0] = 448.0
    x[:, 1] = vals
    bits = synth.f32_to_bf16_bits(x)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), x)          # all exact in bf16
    q, s = moe.mxfp8_quantize(bits_to_bf16_tensor(bits, "cuda"), 0)
    rq, rs = omx.quantize_mx(x.astype(np.float64))
    assert np.all(rs == 127)
    assert np.array_equal(to_np(s), rs)
    got, ref = to_np(q)[:, 1], rq[:, 1]
    assert np.array_equal(got, ref), list(zip(vals, got.tolist(), ref.tolist()))


def test_mxfp8_extreme_scales(moe):
    """Huge and tiny blocks: the scale clamps (-127) and tiny elements flush to (signed) zero."""
    x = np.zeros((4, 64), np.float32)
    x[0, :3] = [3.0e38, 2.0 ** -130, -1.5e-38]
    x[1, :2] = [2.0 ** -130, -(2.0 ** -131)]
    x[2, 5] = 1.0e-20
    x[3, 32:40] = np.float32(-7.25e10)
    bits = synth.f32_to_bf16_bits(x)
    q, s = moe.mxfp8_quantize(bits_to_bf16_tensor(bits, "cuda"), 0)
    rq, rs = omx.quantize_mx(synth.bf16_bits_to_f32(bits).astype(np.float64))
    assert np.array_equal(to_np(s), rs)
    assert np.array_equal(to_np(q), rq)


@pytest.mark.parametrize("rows,K", [(1, 32), (37, 256), (130, 384), (256, 7168), (5, 96)])
def test_mxfp8_quantize_canonical(moe, rows, K):
    rng = np.random.default_rng(rows + K)
    x = rng.normal(0, 1, (rows, K)).astype(np.float32) * np.exp(
        rng.uniform(-8, 8, (rows, 1))).astype(np.float32)
    if K >= 64:
        x[0, 32:64] = 0.0                                    # an all-zero block
    bits = synth.f32_to_bf16_bits(x)
    q, s = moe.mxfp8_quantize(bits_to_bf16_tensor(bits, "cuda"), 0)
    rq, rs = omx.quantize_mx(synth.bf16_bits_to_f32(bits).astype(np.float64))
    assert np.array_equal(to_np(s), rs)
    assert np.array_equal(to_np(q), rq)


@pytest.mark.parametrize("rows,K", [(128, 128), (200, 512), (1, 256)])
def test_mxfp8_quantize_umma_layout(moe, rows, K):
    rng = np.random.default_rng(7 + rows)
    bits = synth.f32_to_bf16_bits(rng.normal(0, 3, (rows, K)).astype(np.float32))
    q, s = moe.mxfp8_quantize(bits_to_bf16_tensor(bits, "cuda"), 1)
    rq, rs = omx.quantize_mx(synth.bf16_bits_to_f32(bits).astype(np.float64))
    assert np.array_equal(to_np(q), rq)
    assert np.array_equal(umma_to_canonical(to_np(s), rows, K), rs)


def test_mxfp8_quantize_strided_rows(moe):
    import torch
    rng = np.random.default_rng(3)
    bits = synth.f32_to_bf16_bits(rng.normal(0, 1, (64, 512)).astype(np.float32))
    full = bits_to_bf16_tensor(bits, "cuda")
    view = full[:, 128:384]
    q, s = moe.mxfp8_quantize(view, 0)
    rq, rs = omx.quantize_mx(synth.bf16_bits_to_f32(bits[:, 128:384]).astype(np.float64))
    assert np.array_equal(to_np(q), rq) and np.array_equal(to_np(s), rs)
    del torch


def test_host_side_errors(moe):
    import torch
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.mxfp8_quantize(x, 0)          # K % 32 != 0
    assert ei.value.code == 2
