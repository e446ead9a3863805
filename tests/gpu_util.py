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
