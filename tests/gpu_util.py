"""Test-side helpers for comparing the device path with the oracle (no layer arithmetic)."""
from __future__ import annotations

import numpy as np

import synth


def umma_scale_offsets(rows: int, K: int) -> np.ndarray:
    """Byte offset of every (row, 32-block) scale in the UMMA layout (as documented in moe.h)."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    kb = np.arange(K // 32, dtype=np.int64)[None, :]
    return ((((r >> 7) * (K // 128) + (kb >> 2)) << 9) + ((r & 31) << 4) + (((r & 127) >> 5) << 2)
            + (kb & 3))


def umma_to_canonical(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return np.asarray(buf, np.uint8)[umma_scale_offsets(rows, K)]


def to_np(t):
    return t.detach().cpu().numpy()


def bf16_tensor_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_bf16_tensor(bits: np.ndarray, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_tensor_f64(t) -> np.ndarray:
    with np.errstate(invalid="ignore"):     # padding rows of saved buffers hold garbage
        return synth.bf16_bits_to_f32(bf16_tensor_bits(t)).astype(np.float64)


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def bf16_floor_error(ref: np.ndarray) -> float:
    """Relative Frobenius error of rounding the exact result itself to bf16."""
    from oracle.layer import bf16_round
    return rel_fro(bf16_round(ref), ref)


# Largest relative error of rounding a value to bf16 (8 significant bits): half a unit in
# the last place, at most 2^-8 of the value.
BF16_HALF_ULP_REL = 2.0 ** -8


def assert_close_out(got: np.ndarray, ref: np.ndarray, rel=2e-3, maxabs_rms=3e-2,
                     out_bf16: bool = True):
    """The layer tolerance: relative Frobenius error <= rel, and element-wise
    |got - ref| <= maxabs_rms * RMS(ref), on top of (for results stored in bf16) the
    rounding of that element to bf16 itself, 2^-8 * |ref|: a bf16 result cannot be closer
    to the fp64 value than its own rounding, which for a heavy-tailed matrix (a weight
    gradient summed over a few tokens) exceeds 3e-2 * RMS at its largest elements."""
    err = rel_fro(got, ref)
    print(f"  rel_fro {err:.3e} (bf16 rounding of the exact result alone: "
          f"{bf16_floor_error(ref):.3e})")
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    dev = np.abs(got - ref)
    bound = maxabs_rms * rms + (BF16_HALF_ULP_REL * np.abs(ref) if out_bf16 else 0.0)
    worst = float(np.max(dev / np.maximum(bound, 1e-300))) if got.size else 0.0
    mx = float(np.max(dev)) if got.size else 0.0
    print(f"  max abs error {mx:.3e} = {mx / max(rms, 1e-300):.3e} * RMS; worst element "
          f"uses {worst:.3f} of its bound")
    assert err <= rel, f"relative Frobenius error {err:.3e} > {rel:.1e}"
    assert worst <= 1.0, f"max abs error beyond {maxabs_rms}*RMS (+ bf16 rounding): {worst:.3f}"
    return err, mx / max(rms, 1e-300)


def padded_rows_of(pad_offsets: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    """Row index in the padded operand buffers of every unpadded position p."""
    E = offsets.shape[0] - 1
    pos = np.arange(offsets[-1])
    e = np.searchsorted(offsets, pos, side="right") - 1
    e = np.minimum(e, E - 1)
    return pad_offsets[e] + (pos - offsets[e])


def canonical_scales(umma_buf, rows_total: int, K: int, rows) -> np.ndarray:
    """Canonical [len(rows), K/32] scale bytes of the given rows of a [rows_total, K]
    matrix whose scales are stored in the UMMA layout (documented in moe.h)."""
    r = np.asarray(rows, dtype=np.int64)[:, None]
    kb = np.arange(K // 32, dtype=np.int64)[None, :]
    off = ((((r >> 7) * (K // 128) + (kb >> 2)) << 9) + ((r & 31) << 4)
           + (((r & 127) >> 5) << 2) + (kb & 3))
    return np.asarray(umma_buf, np.uint8)[off]


def mx_values(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dequantised float64 values of MX codes [n, K] with canonical scales [n, K/32]."""
    from oracle import mxfp8 as omx
    return omx.e4m3_decode(codes) * np.repeat(omx.e8m0_decode(scales), 32, axis=1)


def f16s_values(q_rows, scale_rows) -> np.ndarray:
    """Scaled fp16 (moe.h): fp16 values [n, C] times 2^(b - 127) per 32-column block."""
    q = np.asarray(q_rows).view(np.float16).astype(np.float64)
    s = np.ldexp(1.0, np.asarray(scale_rows, np.int64) - 127)
    return q * np.repeat(s, 32, axis=1)


def expert_rows(pad_offsets: np.ndarray, counts: np.ndarray, e: int) -> np.ndarray:
    """Padded-buffer row indices of expert e's assignments (in segment order)."""
    return int(pad_offsets[e]) + np.arange(int(counts[e]))


def pick_experts(counts: np.ndarray) -> dict:
    """Experts whose rows exercise the tile edge cases: the most loaded one, one whose last
    128-row tile holds fewer than 16 rows, one with a multiple of 128 rows, an empty one
    (each only when the layout has one)."""
    counts = np.asarray(counts)
    out = {"hottest": int(np.argmax(counts))}
    tail = [e for e in range(counts.size) if counts[e] % 128 and counts[e] % 128 < 16]
    if tail:
        out["short_last_tile"] = tail[0]
    full = [e for e in range(counts.size) if counts[e] and counts[e] % 128 == 0]
    if full:
        out["multiple_of_128"] = full[0]
    empty = [e for e in range(counts.size) if counts[e] == 0]
    if empty:
        out["empty"] = empty[0]
    return out


def assert_stage_close(got: np.ndarray, ref: np.ndarray, rel: float, what: str):
    """Stage parity on identical operands: only the kernel's own fp32 arithmetic differs."""
    err = rel_fro(got, ref)
    print(f"  {what}: rel_fro {err:.3e}")
    assert err <= rel, f"{what}: relative Frobenius error {err:.3e} > {rel:.1e}"


def assert_codes_near(got_q, got_s, ref_q, ref_s, ref_vals, what: str, max_frac=1e-3):
    """MX codes computed from fp32 (device) and fp64 (oracle) values of the same quantity:
    equal except where the value sits on a rounding boundary.  At most ``max_frac`` of the
    elements may differ; a differing code under an equal scale must be the neighbour of the
    oracle's, and the oracle's value must lie within 5% of one E4M3 step of the midpoint of
    the two codes' values (a systematic error -- a wrong rounding rule, a wrong scale --
    would put it anywhere up to half a step away; the device's fp32 GEMM accumulation over
    thousands of products moves values by up to ~1e-3 relative, a few percent of a step).
    A pair +0 / -0 is the zero boundary itself: the value rounds to zero either way, its
    sign decided by a rounding far below the smallest step."""
    from oracle import mxfp8 as omx
    got_q, ref_q = np.asarray(got_q), np.asarray(ref_q)
    scale_eq = np.repeat(np.asarray(got_s) == np.asarray(ref_s), 32, axis=1)
    bad = ~((got_q == ref_q) & scale_eq)
    frac = bad.mean() if bad.size else 0.0
    print(f"  {what}: {int(bad.sum())} of {bad.size} codes differ")
    assert frac <= max_frac, f"{what}: {frac:.2e} of the codes differ"
    sel = bad & scale_eq
    if sel.any():
        g, r = got_q[sel].astype(np.int64), ref_q[sel].astype(np.int64)
        assert np.all(np.abs((g & 0x7F) - (r & 0x7F)) <= 1), what
        sc = np.repeat(omx.e8m0_decode(np.asarray(ref_s)), 32, axis=1)[sel]
        v = np.asarray(ref_vals)[sel] / sc
        gv, rv = omx.e4m3_decode(got_q[sel]), omx.e4m3_decode(ref_q[sel])
        zero = (gv == 0) & (rv == 0)            # +0 against -0
        assert np.all(np.abs(v[zero]) <= 2.0 ** -10), what   # rounds to zero either way
        step = np.abs(gv - rv)[~zero]
        if step.size:
            off = np.abs(np.abs(v[~zero]) - np.abs(0.5 * (gv + rv)[~zero])) / step
            print(f"  {what}: differing codes sit within {off.max():.2e} of a step of the "
                  f"midpoint ({int(zero.sum())} signed zeros)")
            assert np.all(off <= 0.05), what
