"""Stage parity of the forward and backward on the GPU, at full size, through the C ABI.

Each stage is checked on the operands the device itself produced, so that a difference in
one place cannot hide in, or spread from, another:

* forward, full size (DeepSeek-V3 shape, load-imbalance stress): every row of the most
  loaded expert, of one whose last 128-row tile holds fewer than 16 rows, of one with a
  multiple of 128 rows and of an empty one (where the layout has them): the requantised
  SwiGLU output codes against the oracle (equal except on rounding boundaries, next to the
  midpoint), the expert outputs y against fp64 arithmetic on the device's own h codes
  (only the kernel's fp32 accumulation and the scaled-fp16 storage of y differ) and
  against the oracle end to end;
* backward: the token-direction MX operands of the weight gradients bit-exact against the
  oracle's quantiser applied to the device's data-path operands; the weight-gradient GEMM
  against fp64 matmul of those identical operands at the layer tolerance (relative
  Frobenius <= 2e-3, max-abs <= 3e-2*RMS beyond each element's own rounding to the bf16
  output); the dgrad GEMMs, d(combine weight) and the
  SwiGLU backward codes likewise on the device's own inputs; dX from the device's
  per-assignment rows.
"""
import numpy as np
import pytest

import synth
from oracle import layer as olayer
from oracle import mxfp8 as omx
from tests.gpu_util import (assert_close_out, assert_codes_near, assert_stage_close,
                            bf16_tensor_f64, bits_to_bf16_tensor, canonical_scales,
                            expert_rows, f16s_values, mx_values, pick_experts, rel_fro,
                            to_np)

pytestmark = pytest.mark.gpu

# Stage tolerances on identical operands.  The GEMMs accumulate in fp32 (~1e-7 relative
# here); their results y and dXa are then stored as scaled fp16, whose rounding moves
# each value by at most 2^-11 of itself (fp16 unit roundoff), so the relative Frobenius
# error of a stored result stays below 2^-11 + the accumulation's share.
STAGE_REL = 1e-5
STAGE_REL_F16S = 2.0 ** -11 + 2e-5


@pytest.fixture(scope="module")
def moe():
    import token_dispatch_grouped_top_b200 as m
    m.load()
    return m


def _rows_t(rows):
    import torch
    return torch.from_numpy(np.asarray(rows, np.int64)).cuda()


def _host_rows(buf, R, C, rows):
    """Rows of a [R, C] device buffer (any dtype view) copied to the host."""
    return to_np(buf.view(R, C).index_select(0, _rows_t(rows)))


# ---------------------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["dsv3", "imbalance"])
def test_forward_full_experts(moe, name):
    import torch
    case = synth.CONFIGS[name]
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    x_bits, logits = synth.make_x(case), synth.make_logits(case)
    wg, wu, wd = synth.expert_weights_torch(case, "cuda")
    pw = moe.prepare_weights(wg, wu, wd, dims)
    del wg, wu, wd
    ws = moe.workspace(dims, moe.OP_FORWARD)
    out, saved = moe.forward(bits_to_bf16_tensor(x_bits, "cuda"),
                             torch.from_numpy(logits).cuda(), pw, save=True, ws=ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    R, d, f, k = moe.padded_rows(dims), case.d, case.f, case.k
    counts, offsets = to_np(saved.bufs["counts"]), to_np(saved.bufs["offsets"])
    pad, perm = to_np(saved.bufs["pad_offsets"]), to_np(saved.bufs["perm"])
    hs_all = to_np(saved.bufs["hs"])
    y = moe.workspace_view(ws, dims, moe.OP_FORWARD, "y", 2 * R * d).view(torch.int16)
    ys = moe.workspace_view(ws, dims, moe.OP_FORWARD, "y_s", R * (d // 32))
    picks = pick_experts(counts)
    assert "short_last_tile" in picks
    if name == "imbalance":
        assert "empty" in picks
    _, _, xhat = olayer.quantize_tokens(x_bits)
    for label, e in picks.items():
        if counts[e] == 0:
            assert pad[e + 1] == pad[e]          # no rows, no tiles
            continue
        rows = expert_rows(pad, counts, e)
        t = perm[offsets[e]:offsets[e + 1]] // k
        W = olayer.ExpertWeights(*synth.expert_weights_f64(case, e))
        g, u, hpre, (hq_ref, hs_ref), _, y_ref = olayer.expert_forward(xhat[t], W)
        hq = _host_rows(saved.bufs["hq"], R, f, rows)
        hs = canonical_scales(hs_all, R, f, rows)
        what = f"{name} expert {e} ({label}, {counts[e]} rows)"
        assert_codes_near(hq, hs, hq_ref, hs_ref, hpre, what + " h codes")
        y_gpu = f16s_values(_host_rows(y, R, d, rows), _host_rows(ys, R, d // 32, rows))
        assert_stage_close(y_gpu, mx_values(hq, hs) @ W.fwd()[2].T, STAGE_REL_F16S, what + " y")
        # end to end (through the device's and the oracle's own h codes, which differ at
        # rounding boundaries): the relative Frobenius bound; an element of y moves by a
        # few percent of RMS where one of its h codes flipped, so the element-wise bound
        # is applied to the layer output (sampled tokens, test_gpu_gemm_forward.py)
        e2e = rel_fro(y_gpu, y_ref)
        print(f"  {what} y end to end: rel_fro {e2e:.3e}")
        assert e2e <= 2e-3
    del out


# ---------------------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------------------
def _transposed(codes_buf, canon_scales, C, R, col0, n32):
    """Columns [col0, col0 + n32) of a [C, R] token-direction operand as [n32, C] codes and
    [n32/32, C] scale bytes (``canon_scales``: the [C, R/32] scales of the whole matrix).
    The codes are stored in 128 x 128 tiles (token block major, then feature block; a
    tile's rows are features of 128 token bytes); col0 starts a 128-token block."""
    assert col0 % 128 == 0
    tb0, ntb = col0 // 128, -(-n32 // 128)
    tiles = codes_buf.view(R // 128, C // 128, 128, 128)[tb0:tb0 + ntb]
    cr = tiles.permute(1, 2, 0, 3).reshape(C, ntb * 128)     # [features, tokens of the blocks]
    codes = to_np(cr[:, :n32]).T
    sc = canon_scales[:, col0 // 32:(col0 + n32) // 32].T
    return np.ascontiguousarray(codes), np.ascontiguousarray(sc)


def _tok_values(codes, scales):
    return omx.e4m3_decode(codes) * np.repeat(omx.e8m0_decode(scales), 32, axis=0)


def _weights_rows(pw, name, scales_host, rows_total, K, rows):
    q = to_np(pw.bufs[name + "_q"].view(rows_total, K).index_select(0, _rows_t(rows)))
    return mx_values(q, canonical_scales(scales_host, rows_total, K, rows))


def _backward_stage_parity(moe, case, experts=None, dx_tokens=None):
    import torch
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    x_bits, logits, dout_bits = synth.make_x(case), synth.make_logits(case), synth.make_dout(case)
    wg, wu, wd = synth.expert_weights_torch(case, "cuda")
    pw = moe.prepare_weights(wg, wu, wd, dims, with_backward=True)
    del wg, wu, wd
    wsf = moe.workspace(dims, moe.OP_FORWARD)
    _, saved = moe.forward(bits_to_bf16_tensor(x_bits, "cuda"), torch.from_numpy(logits).cuda(),
                           pw, save=True, ws=wsf)
    del wsf
    wsb = moe.workspace(dims, moe.OP_BACKWARD)
    grads = moe.backward(bits_to_bf16_tensor(dout_bits, "cuda"), pw, saved, ws=wsb)
    torch.cuda.synchronize()
    assert moe.device_status(wsb) == 0
    R, d, f, E, k = moe.padded_rows(dims), case.d, case.f, case.E, case.k
    sb = {n: to_np(saved.bufs[n]) for n in ("counts", "offsets", "pad_offsets", "perm",
                                            "inv_perm", "topk_idx", "topk_w", "xs", "hs")}
    counts, offsets, pad = sb["counts"], sb["offsets"], sb["pad_offsets"]
    perm, w_all = sb["perm"], sb["topk_w"]

    def wsv(name, nbytes):
        return moe.workspace_view(wsb, dims, moe.OP_BACKWARD, name, nbytes)
    usb = moe.umma_scale_bytes
    dq_s = to_np(wsv("dout_s", usb(R, d)))
    dgu_s = to_np(wsv("dgu_s", usb(R, 2 * f)))
    G = wsv("g", 4 * R * f).view(torch.float32)
    dxa = wsv("dxa", 2 * R * d).view(torch.int16)
    dxas = wsv("dxa_s", R * (d // 32))
    tr = {nm: (wsv(nm + "_q", C * R),
               canonical_scales(to_np(wsv(nm + "_s", usb(C, R))), C, R, np.arange(C)), C)
          for nm, C in (("xt", d), ("ht", f), ("gt", 2 * f), ("yt", d))}
    wdT_s, wguT_s = to_np(pw.bufs["wdT_s"]), to_np(pw.bufs["wguT_s"])
    dw_gpu = to_np(grads["dw_route"]).reshape(-1).astype(np.float64)
    todo = [e for e in range(E)] if experts is None else experts
    for e in todo:
        n = int(counts[e])
        what = f"{case.name} expert {e} ({n} rows)"
        if n == 0:
            for nm in ("dWg", "dWu", "dWd"):
                assert not torch.any(grads[nm][e].float() != 0), what
            continue
        rows = expert_rows(pad, counts, e)
        asg = perm[offsets[e]:offsets[e + 1]]
        n32 = -(-n // 32) * 32
        # the data path's operands, as the device holds them
        X = mx_values(_host_rows(saved.bufs["xq"], R, d, rows), canonical_scales(sb["xs"], R, d, rows))
        H = mx_values(_host_rows(saved.bufs["hq"], R, f, rows), canonical_scales(sb["hs"], R, f, rows))
        dgu_q = _host_rows(wsv("dgu_q", R * 2 * f), R, 2 * f, rows)
        dgu_sc = canonical_scales(dgu_s, R, 2 * f, rows)
        DGU = mx_values(dgu_q, dgu_sc)
        dq = _host_rows(wsv("dout_q", R * d), R, d, rows)
        dsc = canonical_scales(dq_s, R, d, rows)
        # w * dout^ in fp32, as the kernel forms it: (2^s * w) first, then times the code
        mul = (omx.e8m0_decode(dsc).astype(np.float32) * w_all[asg][:, None].astype(np.float32))
        DY = (omx.e4m3_decode(dq).astype(np.float32) * np.repeat(mul, 32, axis=1)).astype(np.float64)
        # 1. token-direction operands: bit-exact
        vals = {}
        for nm, src in (("xt", X), ("ht", H), ("gt", DGU), ("yt", DY)):
            qb, sbuf, C = tr[nm]
            got_q, got_s = _transposed(qb, sbuf, C, R, int(pad[e]), n32)
            ref_q, ref_s = omx.quantize_mx_axis0_segment(src)
            assert np.array_equal(got_q, ref_q), f"{what}: {nm} codes"
            assert np.array_equal(got_s, ref_s), f"{what}: {nm} scales"
            vals[nm] = _tok_values(got_q, got_s)
        # 2. weight-gradient GEMM on those operands
        for nm, ref in (("dWg", vals["xt"].T @ vals["gt"][:, :f]),
                        ("dWu", vals["xt"].T @ vals["gt"][:, f:]),
                        ("dWd", vals["ht"].T @ vals["yt"])):
            print(f"  {what} {nm} stage:")
            assert_close_out(bf16_tensor_f64(grads[nm][e]), ref)
        # 3. dgrad of the down projection, d(combine weight), SwiGLU backward codes
        # from d = 6144 on G is stored only for the rows of an expert's partial last tile
        # (the full tiles run the SwiGLU backward in the GEMM epilogue), below it for every
        # row; the references take the fp64 G
        wdT = _weights_rows(pw, "wdT", wdT_s, E * f, d, e * f + np.arange(f))
        g_ref = mx_values(dq, dsc) @ wdT.T
        stored = np.arange(n) >= (n // 128) * 128 if d >= 6144 else np.ones(n, bool)
        if stored.any():
            g_gpu = _host_rows(G, R, f, rows[stored]).astype(np.float64)
            assert_stage_close(g_gpu, g_ref[stored], STAGE_REL, what + " G")
        assert_stage_close(dw_gpu[asg], np.sum(g_ref * H, axis=1), STAGE_REL,
                           what + " d(combine weight)")
        gu = bf16_tensor_f64(saved.bufs["gu"].view(R, 2 * f).index_select(0, _rows_t(rows)))
        gb, ub = gu[:, :f], gu[:, f:]
        s = olayer.sigmoid(gb)
        dh = w_all[asg][:, None].astype(np.float64) * g_ref
        dgdu = np.concatenate([dh * ub * s * (1 + gb * (1 - s)), dh * gb * s], axis=1)
        ref_q, ref_s = omx.quantize_mx(dgdu)
        assert_codes_near(dgu_q, dgu_sc, ref_q, ref_s, dgdu, what + " [dg|du] codes")
        # 4. dgrad of gate/up
        wguT = _weights_rows(pw, "wguT", wguT_s, E * d, 2 * f, e * d + np.arange(d))
        dxa_rows = f16s_values(_host_rows(dxa, R, d, rows), _host_rows(dxas, R, d // 32, rows))
        assert_stage_close(dxa_rows, DGU @ wguT.T, STAGE_REL_F16S, what + " dXa")
    # 5. dX = sum over the token's k rows of dXa
    toks = np.arange(case.T) if dx_tokens is None else np.asarray(dx_tokens)
    a = (toks[:, None] * k + np.arange(k)[None, :]).ravel()
    e_of = sb["topk_idx"][a]
    prow = pad[e_of] + (sb["inv_perm"][a] - offsets[e_of])
    rows_dxa = f16s_values(_host_rows(dxa, R, d, prow), _host_rows(dxas, R, d // 32, prow))
    rows_dxa = rows_dxa.reshape(toks.size, k, d)
    print(f"  {case.name} dX stage:")
    assert_close_out(bf16_tensor_f64(grads["dx"])[toks], rows_dxa.sum(axis=1))
    return counts


def test_backward_stage_parity_small(moe):
    _backward_stage_parity(moe, synth.MoeCase("sp_s", 300, 256, 512, 8, 2, 0, "skew1.5", seed=41))


def test_backward_stage_parity_empty_and_ragged(moe):
    _backward_stage_parity(moe, synth.MoeCase("sp_h", 200, 512, 256, 32, 4, 1, "hot4cold16",
                                              seed=42))


def test_backward_stage_parity_mid(moe):
    _backward_stage_parity(moe, synth.CONFIGS["mid"])


def test_backward_stage_parity_dsv3(moe):
    case = synth.CONFIGS["dsv3_bwd"]
    counts = np.bincount(np.argsort(-synth.make_logits(case), axis=1, kind="stable")[:, :case.k]
                         .ravel(), minlength=case.E)
    picks = pick_experts(counts)
    rng = np.random.default_rng(0)
    _backward_stage_parity(moe, case, experts=sorted(set(picks.values())),
                           dx_tokens=np.sort(rng.choice(case.T, 256, replace=False)))
