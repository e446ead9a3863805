"""The C-ABI library loads without a GPU, exports every function include/moe.h declares,
and its host-side logic (sizes, argument checks, the wave rule) behaves as documented.
No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from token_dispatch_grouped_top_b200 import build
    build.build()
    from token_dispatch_grouped_top_b200 import _lib
    return _lib.load()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while", "sizeof")))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "moe_forward" in names and "mxfp8_quantize" in names and len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    from token_dispatch_grouped_top_b200 import _lib
    assert set(_lib.SIGNATURES) == set(names)


def _dims(T=8192, d=7168, f=2048, E=256, k=8, s=1):
    from token_dispatch_grouped_top_b200._lib import MoeDims
    return MoeDims(T, d, f, E, k, s)


def test_sizes(lib):
    D = _dims()
    R = lib.moe_padded_rows(ctypes.byref(D))
    assert R % 128 == 0 and R >= 8192 * 8 + 256 * 127
    assert lib.moe_umma_scale_bytes(200, 512) == 256 * 16
    assert lib.moe_umma_scale_bytes(200, 100) == -1
    assert lib.moe_weights_bytes(ctypes.byref(D), 0) == 256 * 4096 * 7168
    assert lib.moe_weights_bytes(ctypes.byref(D), 3) == 256 * 7168 * 2048 // 32
    assert lib.moe_weights_bytes(ctypes.byref(D), 8) == -1
    # permuted MX codes (1 byte) + scaled-fp16 expert outputs (2 bytes) per padded row element
    assert lib.moe_workspace_bytes(ctypes.byref(D), 1) > R * 7168 * 3
    assert lib.moe_workspace_bytes(ctypes.byref(D), 7) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(d=200), 2), (dict(f=384), 2), (dict(k=33, E=64), 2), (dict(E=1025), 2),
    (dict(k=9, E=8), 2), (dict(T=-1), 1), (dict(s=3), 1), (dict(E=0), 1),
    # T*k below 2^31 but the padded row count (T*k + 127*E, rounded up) is not
    (dict(T=(2**31 - 1024 * 127) // 2, k=2, E=1024), 2)])
def test_dims_rejected_before_any_launch(lib, bad, code):
    args = dict(T=16, d=256, f=256, E=8, k=2, s=0)
    args.update(bad)
    D = _dims(**args)
    assert lib.moe_workspace_bytes(ctypes.byref(D), 0) == 0
    rc = lib.moe_route_layout(ctypes.byref(D), None, None, None, None, None, None, None, None,
                              None, 0, None)
    assert rc == code
    # the workspace-free routing entry point applies the same rules, first
    rc = lib.moe_route_layout_noalloc(ctypes.byref(D), None, None, None, None, None, None,
                                      None, None, None, None)
    assert rc == code


def test_noalloc_scratch_limit_is_host_logic(lib):
    # E = 256, k = 8: 131024 tokens fill the 8 MiB scratch array exactly; one more token
    # is rejected before any CUDA call (so this holds without a GPU)
    D = _dims(T=131025, d=256, f=256, E=256, k=8, s=1)
    assert lib.moe_route_layout_noalloc(ctypes.byref(D), 16, 16, 16, 16, 16, 16, 16, None, 16,
                                        None) == 2
    # T > 0 without a status word (checked before the device is touched)
    D = _dims(T=64, d=256, f=256, E=8, k=2, s=0)
    assert lib.moe_route_layout_noalloc(ctypes.byref(D), 16, 16, 16, 16, 16, 16, 16, None,
                                        None, None) == 1


def _noalloc_fits(lib, T, E, k):
    # With no status word a call that passed the scratch check stops at the null-pointer
    # check (1) before touching the device; one over the limit stops at the shape check (2)
    D = _dims(T=T, d=256, f=256, E=E, k=k, s=0)
    rc = lib.moe_route_layout_noalloc(ctypes.byref(D), 16, 16, 16, 16, 16, 16, 16, None,
                                      None, None)
    assert rc in (1, 2), rc
    return rc == 1


@pytest.mark.parametrize("E,k", [(256, 8), (64, 6), (1024, 4), (8, 2), (33, 3)])
def test_noalloc_scratch_formula(lib, E, k):
    # the largest T the 8 MiB array takes equals the header's formula:
    # 256 + 8*nt*E + 4*T*k + 4*(E+1) bytes, each term rounded up to 256, nt = ceil(T/64)
    def up(x):
        return (x + 255) // 256 * 256

    def need(T):
        nt = (T + 63) // 64
        return 256 + up(4 * nt * E) + up(4 * nt * E) + up(4 * T * k) + up(4 * (E + 1))

    lo, hi = 1, 1 << 24
    while lo < hi:                      # largest T with need(T) <= 8 MiB
        mid = (lo + hi + 1) // 2
        lo, hi = (mid, hi) if need(mid) <= 8 << 20 else (lo, mid - 1)
    assert _noalloc_fits(lib, lo, E, k)
    assert not _noalloc_fits(lib, lo + 1, E, k)
    if (E, k) == (256, 8):
        assert lo == 131024


def test_null_and_workspace_checks(lib):
    D = _dims(T=16, d=256, f=256, E=8, k=2, s=0)
    rc = lib.moe_route_layout(ctypes.byref(D), None, None, None, None, None, None, None, None,
                              None, 0, None)
    assert rc == 1
    assert lib.mxfp8_quantize(None, 4, 48, 48, None, None, 0, None) == 2
    assert lib.mxfp8_quantize(None, 4, 64, 64, None, None, 2, None) == 1
    assert lib.moe_grouped_gemm_mx(2, 128, 200, 128, None, None, None, None, None, None, None,
                                   None, 0, None) == 2


def test_status_strings(lib):
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(6) == b"device-side wait timed out"


def test_wave_rule_reproduces_minibatch_figure(lib):
    """Two full waves of 128x256 tiles on 148 SMs for the gate/up GEMM (N = 2*2048) need
    2368 tokens -- the article's minimum minibatch at hidden 7168 / intermediate 2048
    (the printed value and its citation: tests/golden/minibatch_waves.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "minibatch_waves.txt")
    g = dict(line.strip().split("=") for line in open(path)
             if line.strip() and not line.startswith("#"))
    g = {key: int(v) for key, v in g.items()}
    assert lib.moe_min_tokens_for_waves(g["sms"], g["waves"], g["tile_m"], g["tile_n"],
                                        2 * g["intermediate"]) == g["min_tokens"]
    assert lib.moe_min_tokens_for_waves(148, 1, 128, 256, 2 * 2048) == 1184
    assert lib.moe_min_tokens_for_waves(0, 1, 128, 256, 4096) == -1


def test_workspace_offsets(lib):
    # every internal buffer lies inside its operation's workspace, 256-byte aligned; the
    # ones an operation does not have are -1
    D = _dims(T=4096, d=2048, f=1536, E=64, k=6, s=0)
    from token_dispatch_grouped_top_b200._lib import WS_BUFFERS
    R = lib.moe_padded_rows(ctypes.byref(D))
    for op, names in ((1, ("mtile", "y", "counts")),
                      (2, ("mtile", "dout_q", "dout_s", "g", "dgu_q", "dgu_s", "dxa", "xt_q",
                           "xt_s", "ht_q", "ht_s", "gt_q", "gt_s", "yt_q", "yt_s")),
                      (3, ("mtile", "y", "counts"))):
        total = lib.moe_workspace_bytes(ctypes.byref(D), op)
        for n in names:
            off = lib.moe_workspace_offset(ctypes.byref(D), op, WS_BUFFERS[n])
            assert 0 < off < total and off % 256 == 0, (op, n)
    assert lib.moe_workspace_offset(ctypes.byref(D), 1, WS_BUFFERS["dxa"]) == -1
    assert lib.moe_workspace_offset(ctypes.byref(D), 2, WS_BUFFERS["y"]) == -1
    assert lib.moe_workspace_offset(ctypes.byref(D), 4, 0) == -1
    # the forward's expert outputs: R rows of d scaled-fp16 values, then their scale bytes
    y = lib.moe_workspace_offset(ctypes.byref(D), 1, WS_BUFFERS["y"])
    ys = lib.moe_workspace_offset(ctypes.byref(D), 1, WS_BUFFERS["y_s"])
    assert y + 2 * R * 2048 <= ys
    assert ys + R * 2048 // 32 <= lib.moe_workspace_bytes(ctypes.byref(D), 1)


def test_bf16_variant_and_router_backward_checks(lib):
    D = _dims(T=16, d=256, f=256, E=8, k=2, s=0)
    assert lib.moe_forward_bf16(ctypes.byref(D), None, None, None, None, None, None, 0,
                                None) == 1
    assert lib.moe_prepare_weights_bf16(ctypes.byref(D), None, None, None, None, None,
                                        None) == 1
    # K must be a multiple of 64 bf16 elements (one 128-byte swizzled row)
    assert lib.moe_grouped_gemm_bf16(2, 128, 256, 96, None, None, None, None, None, None, 0,
                                     None) == 2
    assert lib.moe_router_backward(ctypes.byref(D), None, None, None, None, None, None) == 1
    bad = _dims(T=16, d=256, f=256, E=8, k=9, s=0)
    assert lib.moe_router_backward(ctypes.byref(bad), None, None, None, None, None, None) == 2
    assert lib.moe_workspace_bytes(ctypes.byref(D), 3) > 0
    assert lib.moe_debug_withhold_ready(-1) == 0


def test_router_gemm_checks(lib):
    # host-side checks only: every failing call returns before any device work
    vp = ctypes.c_void_p
    D = _dims(T=100, d=512, f=256, E=16, k=2, s=0)
    n = lib.moe_workspace_bytes(ctypes.byref(D), 4)
    # header + W_r padded to 256 rows + bf16(G) [128, 64] + its transpose [128, 128]
    # + W_r^T [512, 64] + x^T [512, 128]
    assert n >= 256 + 256 * 512 * 2 + 128 * 64 * 2 + 128 * 128 * 2 + 512 * 64 * 2 + 512 * 128 * 2
    a, ws = vp(1 << 20), vp(1 << 24)
    E12 = _dims(T=100, d=512, f=256, E=12, k=2, s=0)
    assert lib.moe_router_logits(ctypes.byref(E12), a, a, a, ws, 1 << 30, None) == 2
    assert lib.moe_router_logits(ctypes.byref(D), None, a, a, ws, n, None) == 1
    assert lib.moe_router_logits(ctypes.byref(D), vp((1 << 20) + 8), a, a, ws, n, None) == 3
    assert lib.moe_router_logits(ctypes.byref(D), a, a, a, vp((1 << 24) + 16), n, None) == 3
    assert lib.moe_router_logits(ctypes.byref(D), a, a, a, ws, n - 1, None) == 4
    assert lib.moe_router_grads(ctypes.byref(D), a, a, a, a, None, ws, n, None) == 1
    assert lib.moe_router_grads(ctypes.byref(E12), a, a, a, a, a, ws, 1 << 30, None) == 2
    assert lib.moe_router_grads(ctypes.byref(D), a, a, a, a, a, ws, n - 1, None) == 4
    big = _dims()
    assert lib.moe_workspace_bytes(ctypes.byref(big), 4) >= 7168 * 8192 * 2


def test_expert_parallel_checks(lib):
    vp = ctypes.c_void_p
    D = _dims(T=4096, d=512, f=256, E=16, k=4, s=0)
    n4 = lib.moe_ep_workspace_bytes(ctypes.byref(D), 4)
    # receive rows: T * min(k, E/G) + E/G * 127, rounded to 128 -> codes, h, y (2 bytes)
    rows = -(-(4096 * 4 + 4 * 127) // 128) * 128
    assert n4 >= rows * (512 + 256 + 2 * 512)
    assert lib.moe_ep_workspace_bytes(ctypes.byref(D), 3) == 0      # E % world != 0
    assert lib.moe_ep_workspace_bytes(ctypes.byref(D), 0) == 0
    assert lib.moe_ep_workspace_bytes(ctypes.byref(D), 65) == 0
    D16 = _dims(T=4096, d=512, f=256, E=16, k=4, s=0)
    assert lib.moe_ep_workspace_bytes(ctypes.byref(D16), 16) < n4  # min(k, E/G) = 1 row
    a, ws = vp(1 << 20), vp(1 << 24)
    from token_dispatch_grouped_top_b200._lib import MoeWeights
    W = MoeWeights(*([1 << 20] * 8))
    assert lib.moe_ep_experts(ctypes.byref(D), 0, 3, a, ctypes.byref(W), ws, n4, None) == 2
    assert lib.moe_ep_experts(ctypes.byref(D), 4, 4, a, ctypes.byref(W), ws, n4, None) == 1
    assert lib.moe_ep_experts(ctypes.byref(D), 0, 4, None, ctypes.byref(W), ws, n4, None) == 1
    assert lib.moe_ep_experts(ctypes.byref(D), 0, 4, vp((1 << 20) + 8), ctypes.byref(W), ws,
                              n4, None) == 3
    assert lib.moe_ep_experts(ctypes.byref(D), 0, 4, a, ctypes.byref(W), ws, n4 - 1, None) == 4
    assert lib.moe_ep_combine(ctypes.byref(D), None, a, a, a, None, None) == 1
    assert lib.moe_ep_prepare(ctypes.byref(D), None, a, a, a, a, a, a, a, a, a, ws, 1 << 30,
                              None) == 1
