"""GPU parity of the grouped block-scaled GEMM, the weight preparation and the forward.

* exact GEMM: E4M3 operands that are small integers, with power-of-two block scales, keep
  every fp32 partial sum exact, so the tcgen05 grouped GEMM must equal np.matmul bit for
  bit -- including ragged groups (whose last tile runs with the operands swapped, as
  wide as its valid rows) and empty groups.
* weights: every MX byte and scale equals the oracle's quantisation of the same bf16 bits.
* forward: routing/layout and the permuted MX activations bit-exact; the requantised
  SwiGLU output equal except for values on a rounding boundary (one code apart, the
  oracle's value next to the midpoint of the two codes); the output within relative
  Frobenius 2e-3 and max-abs 3e-2*RMS of the fp64 oracle.  The full-size configurations
  are checked here on sampled tokens and, expert by expert, in test_gpu_stage_parity.py.
"""
import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import mxfp8 as omx
from oracle import routing as ort
from tests.gpu_util import (assert_close_out, assert_codes_near, bf16_tensor_f64,
                            bits_to_bf16_tensor, padded_rows_of, rel_fro, to_np,
                            umma_scale_offsets, umma_to_canonical)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _umma_pack(scales: np.ndarray) -> np.ndarray:
    rows, nkb = scales.shape
    K = nkb * 32
    out = np.zeros(((rows + 127) // 128 * 128) * nkb, np.uint8)
    out[umma_scale_offsets(rows, K)] = scales
    return out


@pytest.mark.parametrize("G,N,K,counts", [
    (1, 256, 128, [128]),
    (3, 256, 256, [5, 0, 300]),
    (4, 512, 1024, [129, 128, 1, 77]),
    (2, 768, 384, [256, 255]),
    (5, 256, 512, [16, 17, 112, 113, 127]),
])
def test_grouped_gemm_exact_small_integers(moe, G, N, K, counts):
    import torch
    rng = np.random.default_rng(G * 1000 + N + K)
    counts = np.array(counts)
    mt = np.concatenate([[0], np.cumsum((counts + 127) // 128)]).astype(np.int32)
    R = int(mt[-1]) * 128 + 128
    a_val = rng.integers(-8, 9, (R, K)).astype(np.float64)
    b_val = rng.integers(-8, 9, (G * N, K)).astype(np.float64)
    # scales 2^-1 .. 2^1: every partial sum is a multiple of 2^-2 below 2^18 -> exact in fp32
    a_sc = rng.integers(126, 129, (R, K // 32)).astype(np.uint8)
    b_sc = rng.integers(126, 129, (G * N, K // 32)).astype(np.uint8)
    a_q, b_q = omx.e4m3_encode(a_val), omx.e4m3_encode(b_val)
    A = a_val * np.repeat(np.ldexp(1.0, a_sc.astype(np.int64) - 127), 32, axis=1)
    B = b_val * np.repeat(np.ldexp(1.0, b_sc.astype(np.int64) - 127), 32, axis=1)
    dev = "cuda"
    D = moe.grouped_gemm_mx(torch.from_numpy(mt).to(dev), torch.from_numpy(a_q).to(dev),
                            torch.from_numpy(_umma_pack(a_sc)).to(dev),
                            torch.from_numpy(b_q).to(dev),
                            torch.from_numpy(_umma_pack(b_sc)).to(dev), N, K,
                            rows_valid=torch.from_numpy(counts.astype(np.int32)).to(dev))
    torch.cuda.synchronize()
    D = to_np(D)
    for g in range(G):
        r0 = mt[g] * 128
        rows = slice(r0, r0 + counts[g])
        ref = A[rows] @ B[g * N:(g + 1) * N].T
        assert np.array_equal(D[rows].astype(np.float64), ref), f"group {g}"


def _weights(case, device="cuda"):
    return synth.expert_weights_torch(case, device)


def test_prepare_weights_bit_exact(moe):
    case = synth.MoeCase("pw", 64, 512, 256, 3, 2, 0, "none", seed=2)
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    wg, wu, wd = _weights(case)
    pw = moe.prepare_weights(wg, wu, wd, dims, with_backward=True)
    import torch
    torch.cuda.synchronize()
    d, f, E = case.d, case.f, case.E
    wgu_q = to_np(pw.bufs["wgu_q"]).reshape(E * 2 * f, d)
    wgu_s = umma_to_canonical(to_np(pw.bufs["wgu_s"]), E * 2 * f, d)
    wd_q = to_np(pw.bufs["wd_q"]).reshape(E * d, f)
    wd_s = umma_to_canonical(to_np(pw.bufs["wd_s"]), E * d, f)
    wdT_q = to_np(pw.bufs["wdT_q"]).reshape(E * f, d)
    wdT_s = umma_to_canonical(to_np(pw.bufs["wdT_s"]), E * f, d)
    wguT_q = to_np(pw.bufs["wguT_q"]).reshape(E * d, 2 * f)
    wguT_s = umma_to_canonical(to_np(pw.bufs["wguT_s"]), E * d, 2 * f)
    for e in range(E):
        Wg, Wu, Wd = synth.expert_weights_f64(case, e)
        gq, gs = omx.quantize_mx(Wg.T)
        uq, us = omx.quantize_mx(Wu.T)
        rows = np.arange(f)
        inter = e * 2 * f + (rows // 128) * 256 + rows % 128
        assert np.array_equal(wgu_q[inter], gq) and np.array_equal(wgu_s[inter], gs)
        assert np.array_equal(wgu_q[inter + 128], uq) and np.array_equal(wgu_s[inter + 128], us)
        dq, ds = omx.quantize_mx(Wd.T)
        assert np.array_equal(wd_q[e * d:(e + 1) * d], dq)
        assert np.array_equal(wd_s[e * d:(e + 1) * d], ds)
        tq, ts = omx.quantize_mx(Wd)
        assert np.array_equal(wdT_q[e * f:(e + 1) * f], tq)
        assert np.array_equal(wdT_s[e * f:(e + 1) * f], ts)
        cq, cs = omx.quantize_mx(np.concatenate([Wg, Wu], axis=1))
        assert np.array_equal(wguT_q[e * d:(e + 1) * d], cq)
        assert np.array_equal(wguT_s[e * d:(e + 1) * d], cs)


def _forward_check(moe, case, tokens=None, hq_check=True):
    import torch
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    x_bits = synth.make_x(case)
    logits = synth.make_logits(case)
    wg, wu, wd = _weights(case)
    pw = moe.prepare_weights(wg, wu, wd, dims)
    del wg, wu, wd
    x = bits_to_bf16_tensor(x_bits, "cuda")
    lg = torch.from_numpy(logits).cuda()
    ws = moe.workspace(dims, moe.OP_FORWARD)
    out, saved = moe.forward(x, lg, pw, save=True, ws=ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    wcache = {}

    def wfn(e):
        if e not in wcache:
            wcache[e] = synth.expert_weights_f64(case, e)
        return wcache[e]
    ref = olayer.forward(x_bits, logits, case.k, case.score_fn, case.E, wfn, tokens=tokens,
                         keep=tokens is None)
    sb = {k: to_np(v) for k, v in saved.bufs.items() if k != "gu"}
    assert np.array_equal(sb["topk_idx"].reshape(case.T, case.k), ref["idx"])
    assert np.max(np.abs(sb["topk_w"].reshape(case.T, case.k) - ref["w"])) <= 2e-6
    for key, rk in (("counts", "counts"), ("offsets", "offsets"), ("perm", "perm"),
                    ("inv_perm", "inv")):
        assert np.array_equal(sb[key], ref[rk]), key
    pad = sb["pad_offsets"]
    assert np.array_equal(pad, ort.padded_offsets(ref["counts"]))
    prow = padded_rows_of(pad, ref["offsets"])
    R = moe.padded_rows(dims)
    xq = sb["xq"].reshape(R, case.d)
    xs = umma_to_canonical(sb["xs"], R, case.d)
    tok = ref["perm"] // case.k
    assert np.array_equal(xq[prow], ref["xq"][tok])
    assert np.array_equal(xs[prow], ref["xs"][tok])
    if tokens is None and hq_check:
        hq = sb["hq"].reshape(R, case.f)[prow]
        hs = umma_to_canonical(sb["hs"], R, case.f)[prow]
        hpre = ref["g"] * olayer.sigmoid(ref["g"]) * ref["u"]
        assert_codes_near(hq, hs, ref["hq"], ref["hs"], hpre, f"{case.name} h codes")
        gu = bf16_tensor_f64(saved.bufs["gu"]).reshape(R, 2 * case.f)[prow]
        assert rel_fro(gu[:, :case.f], ref["g"]) < 4e-3
        assert rel_fro(gu[:, case.f:], ref["u"]) < 4e-3
    got = bf16_tensor_f64(out)
    rows = slice(None) if tokens is None else tokens
    return assert_close_out(got[rows], ref["out"][rows])


def test_forward_tiny_full(moe):
    err, mx = _forward_check(moe, synth.CONFIGS["tiny"])
    print(f"tiny: rel_fro {err:.3e}, max/rms {mx:.3e}")


def test_forward_small_ragged_edge_cases(moe):
    # E=1 (dense), k = E, a single token, rows not a multiple of 128
    for case in [synth.MoeCase("e1", 200, 256, 256, 1, 1, 0, "none", seed=3),
                 synth.MoeCase("kE", 77, 512, 256, 4, 4, 1, "normal0.5", seed=4),
                 synth.MoeCase("t1", 1, 256, 512, 8, 2, 0, "none", seed=5),
                 synth.MoeCase("skew", 333, 256, 768, 16, 3, 0, "skew1.5", seed=6)]:
        _forward_check(moe, case)


def test_forward_mid_full(moe):
    err, mx = _forward_check(moe, synth.CONFIGS["mid"])
    print(f"mid: rel_fro {err:.3e}, max/rms {mx:.3e}")


@pytest.mark.parametrize("name,tokens", [("dsv3", [5, 4321]), ("imbalance", [0, 9999, 16383])])
def test_forward_full_size_sampled(moe, name, tokens):
    err, mx = _forward_check(moe, synth.CONFIGS[name], tokens=np.array(tokens))
    print(f"{name}: rel_fro {err:.3e}, max/rms {mx:.3e} on tokens {tokens}")


def test_forward_deterministic_and_status(moe):
    import torch
    case = synth.CONFIGS["tiny"]
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    wg, wu, wd = _weights(case)
    pw = moe.prepare_weights(wg, wu, wd, dims)
    x = bits_to_bf16_tensor(synth.make_x(case), "cuda")
    lg = torch.from_numpy(synth.make_logits(case)).cuda()
    ws = moe.workspace(dims, moe.OP_FORWARD)
    o1, _ = moe.forward(x, lg, pw, ws=ws)
    o1 = o1.clone()
    o2, _ = moe.forward(x, lg, pw, ws=ws)
    assert torch.equal(o1, o2)
    assert moe.device_status(ws) == 0
