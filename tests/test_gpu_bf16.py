"""GPU parity of the layer's BF16 variant (tcgen05.mma kind::f16, no MX quantisation).

* exact GEMM: bf16 operands that are small integers keep every fp32 partial sum exact, so
  the kind::f16 grouped GEMM must equal np.matmul bit for bit, ragged groups (swapped
  last tiles) and empty groups included;
* weight preparation: a pure re-layout, bit-exact;
* forward: routing as in the MXFP8 path; the output within relative Frobenius 2e-3 and
  max-abs 3e-2*RMS of the fp64 oracle (oracle.layer.forward_bf16), which rounds h to bf16
  between the GEMMs as the device does (from fp64 there, fp32 here: a value on a rounding
  boundary may land one bf16 step apart, far inside the tolerance).
"""
import numpy as np
import pytest

import synth
from oracle import layer as olayer
from tests.gpu_util import assert_close_out, bf16_tensor_f64, bits_to_bf16_tensor, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _bf16(vals: np.ndarray):
    """Small integers are exact in bf16: their bits are the top half of the fp32 bits."""
    bits = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return bits_to_bf16_tensor(bits, "cuda")


@pytest.mark.parametrize("G,N,K,counts", [
    (1, 256, 64, [128]),
    (3, 256, 256, [5, 0, 300]),
    (4, 512, 1024, [129, 128, 1, 77]),
    (2, 768, 192, [256, 255]),
    (5, 256, 512, [16, 17, 112, 113, 127]),
])
def test_grouped_gemm_bf16_exact_small_integers(moe, G, N, K, counts):
    import torch
    rng = np.random.default_rng(G * 1000 + N + K + 7)
    counts = np.array(counts)
    mt = np.concatenate([[0], np.cumsum((counts + 127) // 128)]).astype(np.int32)
    R = int(mt[-1]) * 128 + 128
    a = rng.integers(-8, 9, (R, K)).astype(np.float64)
    b = rng.integers(-8, 9, (G * N, K)).astype(np.float64)
    D = to_np(moe.grouped_gemm_bf16(torch.from_numpy(mt).cuda(), _bf16(a), _bf16(b), N,
                                    rows_valid=torch.from_numpy(counts.astype(np.int32)).cuda()))
    torch.cuda.synchronize()
    for g in range(G):
        r0 = mt[g] * 128
        rows = slice(r0, r0 + counts[g])
        assert np.array_equal(D[rows].astype(np.float64), a[rows] @ b[g * N:(g + 1) * N].T), g


def test_prepare_weights_bf16_layout(moe):
    case = synth.MoeCase("pw16", 64, 512, 256, 3, 2, 0, "none", seed=9)
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    wg, wu, wd = synth.expert_weights_uploaded(case, "cuda")
    pw = moe.prepare_weights_bf16(wg, wu, wd, dims)
    import torch
    torch.cuda.synchronize()
    d, f = case.d, case.f
    wgu = to_np(pw.wgu_t.view(torch.int16)).view(np.uint16)
    wdt = to_np(pw.wd_t.view(torch.int16)).view(np.uint16)
    for e in range(case.E):
        g_bits, u_bits, d_bits = (synth.expert_weight_bits(case, e, m) for m in range(3))
        rows = np.arange(f)
        inter = e * 2 * f + (rows // 128) * 256 + rows % 128
        assert np.array_equal(wgu[inter], g_bits.T)
        assert np.array_equal(wgu[inter + 128], u_bits.T)
        assert np.array_equal(wdt[e * d:(e + 1) * d], d_bits.T)


def _forward_bf16_check(moe, case, tokens=None):
    import torch
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    x_bits, logits = synth.make_x(case), synth.make_logits(case)
    wg, wu, wd = synth.expert_weights_torch(case, "cuda")
    pw = moe.prepare_weights_bf16(wg, wu, wd, dims)
    del wg, wu, wd
    ws = moe.workspace(dims, moe.OP_FORWARD_BF16)
    out = moe.forward_bf16(bits_to_bf16_tensor(x_bits, "cuda"), torch.from_numpy(logits).cuda(),
                           pw, ws=ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    wcache = {}

    def wfn(e):
        if e not in wcache:
            wcache[e] = synth.expert_weights_f64(case, e)
        return wcache[e]
    if tokens is None:
        ref = olayer.forward_bf16(x_bits, logits, case.k, case.score_fn, case.E, wfn)["out"]
        rows = slice(None)
    else:
        # only the sampled tokens' expert rows (each expert streamed once)
        sub = olayer.forward_bf16(x_bits[tokens], logits[tokens], case.k, case.score_fn,
                                  case.E, wfn)["out"]
        ref = np.zeros((case.T, case.d))
        ref[tokens] = sub
        rows = tokens
    got = bf16_tensor_f64(out)
    return assert_close_out(got[rows], ref[rows])


def test_forward_bf16_tiny_and_edges(moe):
    _forward_bf16_check(moe, synth.CONFIGS["tiny"])
    for case in [synth.MoeCase("e1", 200, 256, 256, 1, 1, 0, "none", seed=3),
                 synth.MoeCase("kE", 77, 512, 256, 4, 4, 1, "normal0.5", seed=4),
                 synth.MoeCase("t1", 1, 256, 512, 8, 2, 0, "none", seed=5),
                 synth.MoeCase("skew", 333, 256, 768, 16, 3, 0, "skew1.5", seed=6)]:
        _forward_bf16_check(moe, case)


def test_forward_bf16_mid(moe):
    _forward_bf16_check(moe, synth.CONFIGS["mid"])


@pytest.mark.parametrize("name", ["dsv3", "imbalance"])
def test_forward_bf16_full_size_sampled(moe, name):
    case = synth.CONFIGS[name]
    rng = np.random.default_rng(1)
    _forward_bf16_check(moe, case, tokens=np.sort(rng.choice(case.T, 6, replace=False)))
