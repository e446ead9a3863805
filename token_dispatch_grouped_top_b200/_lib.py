"""ctypes view of the C ABI declared in include/moe.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

c_i32, c_i64, c_sz, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "misaligned pointer",
          4: "workspace too small", 5: "CUDA runtime error", 6: "device-side wait timed out",
          7: "device-side index out of bounds", 8: "no sm_100 device"}

OP_ROUTE, OP_FORWARD, OP_BACKWARD, OP_FORWARD_BF16, OP_ROUTER = 0, 1, 2, 3, 4

# internal workspace buffers that moe_workspace_offset locates (moe_ws_buffer)
WS_BUFFERS = {"mtile": 0, "y": 1, "dout_q": 2, "dout_s": 3, "g": 4, "dgu_q": 5, "dgu_s": 6,
              "dxa": 7, "xt_q": 8, "xt_s": 9, "ht_q": 10, "ht_s": 11, "gt_q": 12, "gt_s": 13,
              "yt_q": 14, "yt_s": 15, "counts": 16, "y_s": 17, "dxa_s": 19}

STAGES = ["route", "permute", "gateup", "down", "combine", "bwd_dout", "bwd_dgrad_down",
          "bwd_dgrad_gateup", "bwd_dx", "bwd_transpose", "bwd_wgrad", "bwd_swiglu", "ep_pull",
          "ep_push"]


class MoeDims(ctypes.Structure):
    _fields_ = [("T", c_i64), ("d", c_i32), ("f", c_i32), ("E", c_i32), ("k", c_i32),
                ("score_fn", c_i32)]


WEIGHT_FIELDS = ["wgu_q", "wgu_s", "wd_q", "wd_s", "wdT_q", "wdT_s", "wguT_q", "wguT_s"]
SAVED_FIELDS = ["topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm", "pad_offsets",
                "xq", "xs", "hq", "hs", "gu"]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in WEIGHT_FIELDS]


class MoeSaved(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in SAVED_FIELDS]


EP_PEER_FIELDS = ["counts", "offsets", "perm", "xq", "xs", "y", "ys"]


class MoeEpPeer(ctypes.Structure):
    """One rank's entry of the expert-parallel peer table (moe_ep_peer)."""
    _fields_ = [("T", c_i64)] + [(n, c_vp) for n in EP_PEER_FIELDS]


# name -> (restype, argtypes)
SIGNATURES = {
    "moe_padded_rows": (c_i64, [ctypes.POINTER(MoeDims)]),
    "moe_umma_scale_bytes": (c_i64, [c_i64, c_i64]),
    "moe_weights_bytes": (c_i64, [ctypes.POINTER(MoeDims), c_i32]),
    "moe_saved_bytes": (c_i64, [ctypes.POINTER(MoeDims), c_i32]),
    "moe_workspace_bytes": (c_sz, [ctypes.POINTER(MoeDims), c_i32]),
    "moe_min_tokens_for_waves": (c_i64, [c_i32, c_i32, c_i32, c_i32, c_i64]),
    "moe_workspace_offset": (c_i64, [ctypes.POINTER(MoeDims), c_i32, c_i32]),
    "moe_status_string": (ctypes.c_char_p, [c_i32]),
    "moe_route_layout": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                 c_vp, c_vp, c_vp, c_sz, c_vp]),
    "moe_route_layout_noalloc": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_vp,
                                         c_vp, c_vp, c_vp, c_vp, c_vp]),
    "mxfp8_quantize": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_vp, c_i32, c_vp]),
    "moe_prepare_weights": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_i32,
                                    ctypes.POINTER(MoeWeights), c_vp]),
    "moe_forward": (c_i32, [ctypes.POINTER(MoeDims), ctypes.POINTER(MoeWeights), c_vp, c_vp,
                            c_vp, ctypes.POINTER(MoeSaved), c_vp, c_sz, c_vp]),
    "moe_backward": (c_i32, [ctypes.POINTER(MoeDims), ctypes.POINTER(MoeWeights),
                             ctypes.POINTER(MoeSaved), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                             c_vp, c_sz, c_vp]),
    "moe_grouped_gemm_mx": (c_i32, [c_i32, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                    c_vp, c_vp, c_vp, c_sz, c_vp]),
    "moe_get_device_status": (c_i32, [c_vp, c_vp, ctypes.POINTER(c_i32)]),
    "moe_grouped_gemm_bf16": (c_i32, [c_i32, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                      c_vp, c_sz, c_vp]),
    "moe_prepare_weights_bf16": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_vp,
                                         c_vp]),
    "moe_forward_bf16": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                 c_sz, c_vp]),
    "moe_router_backward": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "moe_router_logits": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "moe_router_grads": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                 c_sz, c_vp]),
    "moe_ep_prepare": (c_i32, [ctypes.POINTER(MoeDims)] + [c_vp] * 11 + [c_sz, c_vp]),
    "moe_ep_workspace_bytes": (c_sz, [ctypes.POINTER(MoeDims), c_i32]),
    "moe_ep_experts": (c_i32, [ctypes.POINTER(MoeDims), c_i32, c_i32, c_vp,
                               ctypes.POINTER(MoeWeights), c_vp, c_sz, c_vp]),
    "moe_ep_combine": (c_i32, [ctypes.POINTER(MoeDims), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "moe_profile_enable": (c_i32, [c_i32]),
    "moe_debug_withhold_ready": (c_i32, [c_i32]),
    "moe_profile_collect": (c_i32, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_i32),
                                    c_i32]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load the in-tree library; raise loudly when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m token_dispatch_grouped_top_b200"
                f".build` (or __graft_entry__.build()); there is no fallback implementation")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")
        self.code = code


def check(code: int, where: str) -> None:
    if code != 0:
        raise MoeError(code, where)
