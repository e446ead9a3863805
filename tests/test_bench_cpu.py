"""The benchmark's reference arm (the CPU oracle on a bounded sample) and its JSON line.

Runs on the host only: `bench.py --impl reference` never touches a GPU.  Checks the keys
the line must carry, that the sample is bounded, and the sweep's command construction.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=240):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                       capture_output=True, text=True, timeout=timeout, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("pass_", ["fwd", "fwdbwd"])
def test_reference_arm_line(pass_):
    d = _run("--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1",
             "--pass", pass_)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["unit"] == "tokens/s" and d["value"] > 0
    assert d["warmup"] >= 3 and d["steps"] == 2
    assert d["config"]["workload"].startswith("tiny")
    assert d["config"]["pass"] == ("forward+backward" if pass_ == "fwdbwd" else "forward")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "experts" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_oracle_sample_is_bounded():
    sys.path.insert(0, ROOT)
    import bench
    import synth
    case = synth.CONFIGS["dsv3"]
    # the sample's expert choice only needs the routing, not the weights: check it on the
    # routing alone (preparing DeepSeek-V3-sized weights takes ~20 s per expert)
    import numpy as np
    from oracle import routing as rt
    idx, _ = rt.route(synth.make_logits(case), case.k, case.score_fn)
    counts = np.bincount(idx.ravel(), minlength=case.E)
    chosen = [e for e in range(case.E) if 128 <= counts[e] <= 512][:2]
    assert len(chosen) == 2
    assert sum(counts[e] for e in chosen) <= 1024      # a pass stays a few seconds
    assert hasattr(bench, "OracleSample") and hasattr(bench, "cpu_baseline")


def test_layer_summary_closed_form():
    sys.path.insert(0, ROOT)
    import bench
    import synth
    case = synth.CONFIGS["dsv3"]
    A = case.T * case.k
    peaks = {"bf16": 1000.0, "hbm": 5000.0}          # 2 PFLOP/s MXFP8, 5 TB/s
    fwd_stages = {"route": 0.05, "permute": 0.2, "gateup": 2.0, "down": 1.5, "combine": 0.3}
    r = bench.layer_summary(case, fwd_stages, 4.05, peaks, bwd=False)
    assert r["flops"] == pytest.approx(6.0 * A * case.d * case.f)
    weights = 3 * case.E * case.d * case.f * (1 + 1 / 32)
    assert r["bytes"] > weights                       # weights read once, plus activations
    t_fl, t_by = r["flops"] / 2e15, r["bytes"] / 5e12
    assert r["t_roof_ms"] == pytest.approx(1e3 * max(t_fl, t_by))
    assert r["bound"] == ("tensor" if t_fl >= t_by else "hbm")
    assert r["tensor_frac"] == pytest.approx(r["flops"] / 4.05e-3 / 2e15)
    assert r["frac_of_roof"] == pytest.approx(r["t_roof_ms"] / 4.05)
    # the method's per-unit bytes: logits + idx/w + perm/inv; x + permuted MX rows; bf16
    # expert outputs + out
    mv = (4 * case.T * case.E + 16 * A) + (2 * case.T * case.d + A * case.d * (1 + 1 / 32)) + \
        (2 * A * case.d + 2 * case.T * case.d)
    assert r["data_movement_hbm_frac"] == pytest.approx(mv / 0.55e-3 / 5e12)
    assert r["route_permute_combine_hbm_frac"] == pytest.approx(mv / 0.55e-3 / 5e12)
    impl = bench.implementation_bytes(case, True, rows_used=A + 1000, rows_out=A + 500)
    alg = bench.algorithmic_bytes(case, True)
    # scaled fp16 rows (2 bytes + a scale byte per 32) instead of bf16
    assert impl["combine"] - alg["combine"] == pytest.approx(A * case.d / 32)
    assert impl["bwd_transpose"] > alg["bwd_transpose"]           # padded rows
    bwd_stages = dict(fwd_stages, bwd_dout=0.2, bwd_dgrad_down=1.3, bwd_swiglu=0.4,
                      bwd_dgrad_gateup=2.7, bwd_dx=0.3, bwd_transpose=1.0, bwd_wgrad=6.2)
    rb = bench.layer_summary(case, bwd_stages, 16.6, peaks, bwd=True)
    assert rb["flops"] == pytest.approx(18.0 * A * case.d * case.f)
    # the weight gradients' bf16 output alone: 2 bytes x E x 3 x d x f
    assert rb["bytes"] - r["bytes"] > 2 * case.E * 3 * case.d * case.f
    assert rb["bound"] == "hbm"


@pytest.mark.parametrize("tail", [0, 1000, 65536])
def test_fused_swiglu_byte_split(tail):
    # Fusing the SwiGLU backward into the dgrad epilogue moves the full rows' SwiGLU bytes
    # into the GEMM's stage and drops exactly their G round trip (2 bytes written and 2
    # read per element, counted in bf16) for the d(w) partial sums (4 bytes per
    # row and 128 features); every other stage keeps its bytes.
    sys.path.insert(0, ROOT)
    import bench
    import synth
    case = synth.CONFIGS["dsv3_bwd"]
    A, f = case.T * case.k, case.f
    plain = bench.algorithmic_bytes(case, True)
    fused = bench.algorithmic_bytes(case, True, tail_rows=tail)
    pair = ("bwd_dgrad_down", "bwd_swiglu")
    saved = sum(plain[s] for s in pair) - sum(fused[s] for s in pair)
    assert saved == pytest.approx((A - tail) * f * 4 - A * (f // 128) * 4)
    assert {s: v for s, v in plain.items() if s not in pair} == \
        {s: v for s, v in fused.items() if s not in pair}


@pytest.mark.parametrize("with_bwd", [False, True])
def test_cpu_baseline_fields(with_bwd):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    r = bench.cpu_baseline(synth.CONFIGS["tiny"], budget_s=0.2, with_bwd=with_bwd)
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["value"] > 0
    assert r["cores"] >= 1 and r["host_cores_visible"] >= 1 and r["host_cpu"]
    assert ("backward" in r["sample"]) == with_bwd
