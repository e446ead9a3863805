"""Seeded synthetic inputs for the MoE layer: shared by the CPU oracle and the GPU path.

This module only *draws* inputs. It holds none of the layer's arithmetic (no routing,
no quantisation, no GEMM). Both sides import it so that they see identical input bits:

* ``x`` and ``dout`` are drawn in fp32 from NumPy ``default_rng`` streams and rounded
  (round-to-nearest-even) to bf16; they are returned as raw bf16 bit patterns (uint16).
* router ``logits`` are materialised once in fp32 on the host (noise + per-expert bias,
  added in fp32), so both sides route on the same bits.
* expert weights are too large to draw on the host for the big shapes (the
  DeepSeek-V3-shaped layer holds 11.3e9 weights), so they come from a counter-based
  generator that NumPy (CPU, one expert at a time) and torch (GPU, all experts) evaluate
  to the same bits: a 32-bit integer hash of (seed, expert, matrix, element index) picks
  one of 65536 fp32 normal quantiles, which is scaled by 1/sqrt(fan_in) in fp32 and
  rounded to bf16.  Integer hashing and one IEEE fp32 multiply are exact on both sides.

The workloads are the five synthetic configurations of the MoE layer (tiny, mid,
DeepSeek-V3-shaped, load-imbalance stress, and the backward of the DeepSeek-V3 shape);
the pages describing the method run no public benchmark or dataset, so nothing here
stands in for one.
"""
from __future__ import annotations

import dataclasses
import functools

import numpy as np

SCORE_SOFTMAX_TOPK = 0
SCORE_SIGMOID_RENORM = 1

# stream ids for SeedSequence spawning (fixed so that every input has its own stream)
_STREAM_X, _STREAM_LOGITS, _STREAM_BIAS, _STREAM_DOUT, _STREAM_EXPERT_PICK = 1, 2, 3, 4, 5
_STREAM_ROUTER, _STREAM_DLOGITS = 6, 7
_WG, _WU, _WD = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class MoeCase:
    """Shape and input recipe of one MoE-layer workload."""
    name: str
    T: int          # tokens
    d: int          # hidden size
    f: int          # expert FFN intermediate size
    E: int          # experts
    k: int          # experts per token
    score_fn: int   # SCORE_SOFTMAX_TOPK or SCORE_SIGMOID_RENORM
    bias: str       # "none" | "skew1.5" | "normal0.5" | "hot4cold16"
    seed: int = 0
    backward: bool = False

    @property
    def A(self) -> int:
        return self.T * self.k

    def replace(self, **kw) -> "MoeCase":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": MoeCase("tiny", 512, 256, 512, 8, 2, SCORE_SOFTMAX_TOPK, "none"),
    "mid": MoeCase("mid", 4096, 2048, 1536, 64, 6, SCORE_SOFTMAX_TOPK, "skew1.5"),
    "dsv3": MoeCase("dsv3", 8192, 7168, 2048, 256, 8, SCORE_SIGMOID_RENORM, "normal0.5"),
    "imbalance": MoeCase("imbalance", 16384, 4096, 1536, 128, 8, SCORE_SOFTMAX_TOPK,
                         "hot4cold16"),
    "dsv3_bwd": MoeCase("dsv3_bwd", 8192, 7168, 2048, 256, 8, SCORE_SIGMOID_RENORM,
                        "normal0.5", backward=True),
}
CONFIG_ORDER = ["tiny", "mid", "dsv3", "imbalance", "dsv3_bwd"]


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, stream]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_x(case: MoeCase) -> np.ndarray:
    """Token activations x [T, d]: bf16 bits of N(0, 1) draws."""
    z = _rng(case.seed, _STREAM_X).standard_normal((case.T, case.d), dtype=np.float32)
    return f32_to_bf16_bits(z)


def make_dout(case: MoeCase) -> np.ndarray:
    """Upstream gradient dOut [T, d]: bf16 bits of N(0, 1) draws."""
    z = _rng(case.seed, _STREAM_DOUT).standard_normal((case.T, case.d), dtype=np.float32)
    return f32_to_bf16_bits(z)


def expert_bias(case: MoeCase) -> np.ndarray:
    """Per-expert fp32 logit bias for the configuration's load pattern."""
    E = case.E
    if case.bias == "none":
        return np.zeros(E, np.float32)
    if case.bias == "skew1.5":      # b_e = 1.5 * z_e, z_e ~ N(0,1): skewed, Zipf-like load
        z = _rng(case.seed, _STREAM_BIAS).standard_normal(E, dtype=np.float32)
        return (np.float32(1.5) * z).astype(np.float32)
    if case.bias == "normal0.5":    # per-expert bias ~ N(0, 0.5) (0.5 = standard deviation)
        z = _rng(case.seed, _STREAM_BIAS).standard_normal(E, dtype=np.float32)
        return (np.float32(0.5) * z).astype(np.float32)
    if case.bias == "hot4cold16":   # 4 hot experts (+4.0), 16 experts never chosen (-1e4)
        b = np.zeros(E, np.float32)
        pick = _rng(case.seed, _STREAM_EXPERT_PICK).permutation(E)
        b[pick[:4]] = np.float32(4.0)
        b[pick[4:20]] = np.float32(-1e4)
        return b
    raise ValueError(case.bias)


def make_logits(case: MoeCase) -> np.ndarray:
    """Router logits [T, E] fp32: N(0,1) noise plus the per-expert bias, added in fp32."""
    noise = _rng(case.seed, _STREAM_LOGITS).standard_normal((case.T, case.E), dtype=np.float32)
    return (noise + expert_bias(case)[None, :]).astype(np.float32)


def make_router_weight(case: MoeCase) -> np.ndarray:
    """Router weight W_r [E, d] (one row per expert): bf16 bits of N(0, 1/sqrt(d)) draws, so
    that x . W_r^T has the unit scale of the configurations' logits."""
    z = _rng(case.seed, _STREAM_ROUTER).standard_normal((case.E, case.d), dtype=np.float32)
    return f32_to_bf16_bits(z * np.float32(1.0 / np.sqrt(float(case.d))))


def make_dlogits(case: MoeCase) -> np.ndarray:
    """A gradient of the logits [T, E] fp32: N(0, 1) draws."""
    return _rng(case.seed, _STREAM_DLOGITS).standard_normal((case.T, case.E), dtype=np.float32)


# ---------------------------------------------------------------------------------------
# counter-based expert weights
# ---------------------------------------------------------------------------------------

@functools.lru_cache(maxsize=1)
def normal_quantile_table() -> np.ndarray:
    """65536 fp32 quantiles of N(0,1) at probabilities (u + 0.5) / 65536."""
    from scipy.special import ndtri
    u = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
    return ndtri(u).astype(np.float32)


_M1, _M2 = 0x7FEB352D, 0x846CA68B   # "lowbias32" integer hash multipliers (public domain)


def _mix32_np(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.uint32, copy=True)
    x ^= x >> np.uint32(16)
    x *= np.uint32(_M1)
    x ^= x >> np.uint32(15)
    x *= np.uint32(_M2)
    x ^= x >> np.uint32(16)
    return x


def _keys(seed: int, expert: int, which: int) -> tuple[int, int]:
    s = np.array([(seed * 0x9E3779B1 + 0x632BE5AB) & 0xFFFFFFFF], np.uint32)
    k1 = _mix32_np(_mix32_np(s) ^ np.uint32(((expert * 4 + which + 1) * 0x85EBCA77) & 0xFFFFFFFF))
    k2 = _mix32_np(k1 + np.uint32(0x27D4EB2F))
    return int(k1[0]), int(k2[0])


def _weight_std(case: MoeCase, which: int) -> np.float32:
    fan_in = case.d if which in (_WG, _WU) else case.f
    return np.float32(1.0 / np.sqrt(float(fan_in)))


def _weight_shape(case: MoeCase, which: int) -> tuple[int, int]:
    return (case.d, case.f) if which in (_WG, _WU) else (case.f, case.d)


def expert_weight_bits(case: MoeCase, expert: int, which: int) -> np.ndarray:
    """bf16 bits of one expert matrix: which = 0 W_gate [d,f], 1 W_up [d,f], 2 W_down [f,d]."""
    shape = _weight_shape(case, which)
    n = shape[0] * shape[1]
    assert n < 2 ** 32
    k1, k2 = _keys(case.seed, expert, which)
    idx = np.arange(n, dtype=np.uint32)
    h = _mix32_np(_mix32_np(idx ^ np.uint32(k1)) + np.uint32(k2)) >> np.uint32(16)
    z = normal_quantile_table()[h]
    v = (z * _weight_std(case, which)).astype(np.float32)
    return f32_to_bf16_bits(v).reshape(shape)


def expert_weights_f64(case: MoeCase, expert: int):
    """(W_gate [d,f], W_up [d,f], W_down [f,d]) of one expert as float64 arrays of bf16 values."""
    return tuple(bf16_bits_to_f32(expert_weight_bits(case, expert, w)).astype(np.float64)
                 for w in (_WG, _WU, _WD))


def _mul32_torch(x, c: int):
    """(x * c) mod 2**32 for int64 tensors holding values < 2**32, with no int64 overflow."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & 0xFFFFFFFF


def _mix32_torch(x):
    x = x ^ (x >> 16)
    x = _mul32_torch(x, _M1)
    x = x ^ (x >> 15)
    x = _mul32_torch(x, _M2)
    return x ^ (x >> 16)


def expert_weights_torch(case: MoeCase, device, experts=None):
    """All experts' bf16 weights generated on ``device`` with torch integer ops.

    Returns (W_gate [E,d,f], W_up [E,d,f], W_down [E,f,d]) as torch.bfloat16 tensors whose
    bits equal :func:`expert_weight_bits` for every expert.
    """
    import torch
    experts = range(case.E) if experts is None else experts
    table = torch.from_numpy(normal_quantile_table()).to(device)
    outs = []
    for which in (_WG, _WU, _WD):
        shape = _weight_shape(case, which)
        n = shape[0] * shape[1]
        std = torch.tensor(float(_weight_std(case, which)), dtype=torch.float32, device=device)
        w = torch.empty((len(experts),) + shape, dtype=torch.bfloat16, device=device)
        idx = torch.arange(n, dtype=torch.int64, device=device)
        for i, e in enumerate(experts):
            k1, k2 = _keys(case.seed, e, which)
            h = _mix32_torch((_mix32_torch(idx ^ k1) + k2) & 0xFFFFFFFF) >> 16
            v = table[h] * std                      # one IEEE fp32 multiply
            w[i] = v.to(torch.bfloat16).view(shape)  # round-to-nearest-even
            del h, v
        outs.append(w)
    return tuple(outs)


def expert_weights_uploaded(case: MoeCase, device):
    """The same weights as :func:`expert_weights_torch`, drawn on the host with NumPy and
    uploaded with one copy per matrix (for small cases: no device-side generator kernels)."""
    import torch
    outs = []
    for which in (_WG, _WU, _WD):
        bits = np.stack([expert_weight_bits(case, e, which) for e in range(case.E)])
        outs.append(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device))
    return tuple(outs)


def case_by_name(name: str, **overrides) -> MoeCase:
    return CONFIGS[name].replace(**overrides) if overrides else CONFIGS[name]
