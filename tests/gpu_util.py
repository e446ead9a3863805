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


def assert_close_out(got: np.ndarray, ref: np.ndarray, rel=2e-3, maxabs_rms=3e-2):
    """The layer tolerance: relative Frobenius error and max-abs error relative to RMS."""
    err = rel_fro(got, ref)
    print(f"  rel_fro {err:.3e} (bf16 rounding of the exact result alone: "
          f"{bf16_floor_error(ref):.3e})")
    rms = float(np.sqrt(np.mean(ref ** 2)))
    mx = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert err <= rel, f"relative Frobenius error {err:.3e} > {rel:.1e}"
    assert mx <= maxabs_rms * rms, f"max abs error {mx:.3e} > {maxabs_rms}*RMS ({rms:.3e})"
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
    oracle's and the oracle's value must lie next to the midpoint of the two codes' values
    (within 1e-4 relative: the fp32 evaluation's error is ~1e-6)."""
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
        mid = 0.5 * (omx.e4m3_decode(got_q[sel]) + omx.e4m3_decode(ref_q[sel]))
        assert np.all(np.abs(np.abs(v) - np.abs(mid)) <= 1e-4 * np.abs(v) + 1e-30), what
