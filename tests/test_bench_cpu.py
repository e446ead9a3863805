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
