"""Benchmark of the MoE layer hot path on B200: one JSON line on rank 0.

A step is one pass of the whole hot path over one synthetic batch of the DeepSeek-V3-shaped
configuration (T=8192 tokens, d=7168, f=2048, E=256 experts, top-8 sigmoid-renormalised
routing, MXFP8 expert GEMMs): route -> layout -> MXFP8 pull dispatch -> grouped GEMM
gate/up + SwiGLU + requantisation -> grouped GEMM down -> weighted combine (forward), then
the backward pass on the same batch (--pass fwd times the forward alone).  Inputs are resident in HBM when
the timed region starts; the weights (11.6 GB of MXFP8) exceed the 126 MB L2, so every
step streams them from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs an independent replica on its own batch (the layer
on one GPU does not shard; data-parallel replicas only), value = all ranks' tokens over
the max-over-ranks device time.  --impl reference times the CPU oracle (rank 0 only) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd/bwd tokens/s at 1 B200; % of MXFP8 tensor peak and HBM BW"
CONFIG_NAME = "dsv3"


# Pure-write HBM stream measured on this machine's B200s with TMA stores of 32-row x 128-byte
# boxes into a 4 GiB [rows, 4096-byte] matrix (the weight-gradient epilogue's pattern; plain
# coalesced 16-byte stores reach ~6300 GB/s): the ceiling of an output-dominated kernel.
WRITE_ONLY_GBS = 5959.0
# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the kernels the roofline
# reports, from ncu captures of the mid configuration (profiles/wgrad_mid_full.md,
# profiles/grouped_gemm_mid_full.md), as a ratio to the same launches' algorithmic bytes;
# a full-size launch's traffic is that ratio times its own algorithmic bytes (its operand
# and output bytes both grow with the shape).  Lines still dirty in L2 when a launch ends
# are not counted by the capture.
WGRAD_TRAFFIC_RATIO = (752.110592 + 153.921536 + 349.786368 + 107.617280) / 1428.553728
GATEUP_TRAFFIC_RATIO = (413.373440 + 168.876032) / 657.063936


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def _workload(case, pass_):
    score = "sigmoid-renorm" if case.score_fn == 1 else "softmax-top-k"
    return (f"{case.name} {pass_} (MoE layer: T={case.T}, d={case.d}, f={case.f}, E={case.E}, "
            f"top-{case.k} {score}, bias {case.bias}, MXFP8 E4M3/E8M0, fp32 accumulate, "
            f"bf16 out)")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        load = [s for s in sm if s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


def max_over_ranks(ms: float, device, world: int) -> float:
    """The slowest rank's time: every rank contributes its own device-timed milliseconds
    (one all-reduce MAX over the process group; a no-op on one rank)."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, steps: int, ms: float) -> float:
    """Whole-job throughput: the tokens every rank processed over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms * 1e-3)


def algorithmic_bytes(case, bwd: bool, tail_rows=None) -> dict:
    """Bytes each stage must move by the method (the per-unit figures of the method times the
    units of one step): MX bytes include the 1/32 scale overhead, activations count the
    A = T*k assignments (no tile padding), expert outputs and input gradients per
    assignment are bf16, weights are read once.

    tail_rows (backward; given when the library fuses, i.e. for d >= 6144): the rows of
    the experts' partial last tiles.  The dgrad GEMM of the down projection then runs the
    SwiGLU backward in its epilogue for every other row, so G is not stored for them:
    those rows' SwiGLU bytes (g|u and h^ read, [dg|du]^ written) count in that GEMM's
    stage, and the SwiGLU stage keeps the tail rows (G written and read) and the per-row
    partial sums of d(w) (f/128 fp32 each).  None: G for every row, as unfused."""
    T, d, f, E, k = case.T, case.d, case.f, case.E, case.k
    A = T * k
    mx = 1 + 1 / 32
    by = {
        "route": 4 * T * E + 8 * A + 8 * A,
        "permute": 2 * T * d + A * d * mx,
        "gateup": 2 * E * f * d * mx + A * d * mx + A * f * mx + (4 * A * f if bwd else 0),
        "down": E * d * f * mx + A * f * mx + 2 * A * d,
        "combine": 2 * A * d + 2 * T * d,
    }
    if bwd:
        by.update({
            "bwd_dout": 2 * T * d + A * d * mx,
            "bwd_dgrad_down": E * f * d * mx + A * d * mx + 2 * A * f,
            # G and the saved g|u read, h^ read, [dg|du]^ written, per assignment row
            "bwd_swiglu": A * f * (2 + 4 + 3 * mx),
            "bwd_dgrad_gateup": 2 * E * d * f * mx + 2 * A * f * mx + 2 * A * d,
            "bwd_dx": 2 * A * d + 2 * T * d,
            "bwd_transpose": 2 * A * (2 * d + 3 * f) * mx,
            "bwd_wgrad": 2 * E * 3 * d * f + A * (2 * d + 3 * f) * mx,
        })
        if tail_rows is not None:
            full = A - tail_rows
            by["bwd_dgrad_down"] = (E * f * d * mx + A * d * mx + full * f * (4 + 3 * mx) +
                                    tail_rows * 2 * f)
            by["bwd_swiglu"] = tail_rows * f * (2 + 4 + 3 * mx) + A * (f // 128) * 4
    return by


# Bytes per element of the intermediates y and dXa: scaled fp16 (2-byte values plus one
# scale byte per 32); G stays fp32.
F16S = 2 + 1 / 32


def implementation_bytes(case, bwd: bool, rows_used: int, rows_out: int, tail_rows=None) -> dict:
    """Bytes the kernels actually move where they differ from the algorithmic count:
    scaled-fp16 expert outputs and input gradients, fp32 G, and the tile-padded rows (``rows_used``:
    rows inside some expert segment; ``rows_out``: rows a GEMM with such an output
    writes)."""
    T, d, f, k = case.T, case.d, case.f, case.k
    A = T * k
    mx = 1 + 1 / 32
    alg = algorithmic_bytes(case, bwd, tail_rows)
    impl = dict(alg)
    impl["down"] = alg["down"] - 2 * A * d + F16S * rows_out * d
    impl["combine"] = F16S * A * d + 2 * T * d
    if bwd:
        if tail_rows is None:
            impl["bwd_dgrad_down"] = alg["bwd_dgrad_down"] - 2 * A * f + 4 * rows_out * f
            impl["bwd_swiglu"] = A * f * (4 + 4 + 3 * mx)
        else:  # G (fp32) stored and read for the tail rows only
            impl["bwd_dgrad_down"] = alg["bwd_dgrad_down"] + 2 * tail_rows * f
            impl["bwd_swiglu"] = alg["bwd_swiglu"] + 2 * tail_rows * f
        impl["bwd_dgrad_gateup"] = alg["bwd_dgrad_gateup"] - 2 * A * d + F16S * rows_out * d
        impl["bwd_dx"] = F16S * A * d + 2 * T * d
        impl["bwd_transpose"] = 2 * rows_used * (2 * d + 3 * f) * mx
        impl["bwd_wgrad"] = 2 * case.E * 3 * d * f + rows_used * (2 * d + 3 * f) * mx
    return impl


def layer_flops(case, bwd: bool) -> dict:
    A, d, f = case.T * case.k, case.d, case.f
    fl = {"gateup": 4.0 * A * d * f, "down": 2.0 * A * d * f}
    if bwd:
        fl.update({"bwd_dgrad_down": 2.0 * A * d * f, "bwd_dgrad_gateup": 4.0 * A * d * f,
                   "bwd_wgrad": 6.0 * A * d * f})
    return fl


DATA_MOVEMENT = ("route", "permute", "combine", "bwd_dout", "bwd_dx")


def layer_summary(case, stage_ms: dict, ms_step: float, peaks: dict, bwd: bool,
                  tail_rows=None) -> dict:
    """Whole-layer roofline of one step: algorithmic FLOPs and HBM bytes
    (:func:`algorithmic_bytes`), t_roof = max(FLOPs / P_mxfp8, bytes / BW_copy), and the
    fraction of each resource the measured step reaches.  Also the aggregate HBM fraction
    (sum of bytes over sum of times) of the data-movement kernels: routing, dispatch and
    combine (forward) and, with the backward, its dispatch and combine twins."""
    by, fl = algorithmic_bytes(case, bwd, tail_rows), layer_flops(case, bwd)
    flops, nbytes = sum(fl.values()), sum(by.values())
    p_mx, bw = 2.0 * peaks["bf16"] * 1e12, peaks["hbm"] * 1e9
    t_roof = max(flops / p_mx, nbytes / bw)
    sec = ms_step * 1e-3

    def agg(names):
        ms = sum(stage_ms.get(n, 0.0) for n in names)
        b = sum(by[n] for n in names if n in stage_ms)
        return (b / (ms * 1e-3) / bw) if ms > 0 else None
    fwd_moves = [n for n in DATA_MOVEMENT if not n.startswith("bwd") and n in by]
    moves = [n for n in DATA_MOVEMENT if n in by]
    return {"flops": flops, "bytes": nbytes, "t_roof_ms": t_roof * 1e3,
            "bound": "tensor" if flops / p_mx >= nbytes / bw else "hbm",
            "frac_of_roof": t_roof / sec, "tensor_frac": flops / sec / p_mx,
            "hbm_frac": nbytes / sec / bw,
            "route_permute_combine_hbm_frac": agg(fwd_moves),
            "data_movement_hbm_frac": agg(moves), "data_movement_kernels": moves}


def _safe_layer_summary(case, stage_info, ms_step, peaks, bwd, tail_rows=None):
    try:
        return layer_summary(case, {n: v["ms_per_launch"] for n, v in stage_info.items()},
                             ms_step, peaks, bwd, tail_rows)
    except Exception as e:  # reporting only: never lose the benchmark line over it
        return {"error": repr(e)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class OracleSample:
    """A bounded sample of the workload for timing the CPU oracle as it stands.

    The sample is the assignments of a few experts (the first ones, in index order, holding
    between 128 and 512 rows, i.e. near the mean load T*k/E of the DeepSeek-V3 shape, else
    the first non-empty ones): routing/layout of the whole batch is timed once and charged pro rata;
    per pass, the sampled tokens are quantised and the sampled experts' FFNs run (and, with
    ``with_bwd``, the oracle backward of the same experts on the same tokens).  Weight
    preparation (quantising each expert's weights, ~10-20 s per expert in fp64 NumPy) is
    done once, untimed, as on the GPU."""

    def __init__(self, case, with_bwd: bool, n_experts: int = 2):
        import numpy as np

        import synth
        from oracle import layer as L
        from oracle import routing as rt
        self.case, self.with_bwd, self.L, self.np = case, with_bwd, L, np
        self.x_bits, self.logits = synth.make_x(case), synth.make_logits(case)
        self.dout_bits = synth.make_dout(case) if with_bwd else None
        t0 = time.perf_counter()
        idx, w = rt.route(self.logits, case.k, case.score_fn)
        counts, offsets, perm, inv = rt.layout(idx, case.E)
        self.t_route = time.perf_counter() - t0
        self.wflat = w.reshape(-1)
        self.experts, self.rows, self.prepared = [], {}, {}
        sizes = np.diff(offsets)
        chosen = [e for e in range(case.E) if 128 <= sizes[e] <= 512][:n_experts]
        if len(chosen) < n_experts:
            chosen = [e for e in range(case.E) if sizes[e] > 0][:n_experts]
        for e in chosen:
            rows = perm[offsets[e]:offsets[e + 1]]
            W = L.ExpertWeights(*synth.expert_weights_f64(case, e))
            W.fwd()
            if with_bwd:
                W.bwd()
            self.experts.append(e)
            self.rows[e] = rows
            self.prepared[e] = W
        self.n_rows = sum(r.size for r in self.rows.values())
        self.frac = self.n_rows / (case.T * case.k)

    def run(self) -> float:
        """One timed pass over the sample; seconds including the pro-rata routing share."""
        np, L, case = self.np, self.L, self.case
        t0 = time.perf_counter()
        for e in self.experts:
            rows = self.rows[e]
            t = rows // case.k
            _, _, xhat = L.quantize_tokens(self.x_bits[t])
            y = L.expert_forward(xhat, self.prepared[e])[-1]
            out = np.zeros((t.size, case.d))
            np.add.at(out, np.arange(t.size), self.wflat[rows][:, None] * y)
            if self.with_bwd:
                ts = np.unique(t)
                L.backward(self.x_bits[ts], self.logits[ts], self.dout_bits[ts], case.k,
                           case.score_fn, case.E, lambda g: None, experts=[e],
                           prepared={e: self.prepared[e]})
        return time.perf_counter() - t0 + self.frac * self.t_route

    def describe(self, seconds: float, passes: int) -> str:
        what = "forward + backward" if self.with_bwd else "forward"
        return (f"fp64 NumPy oracle {what} of experts {self.experts} ({self.n_rows} of "
                f"{self.case.T * self.case.k} assignments; their tokens quantised, routing of "
                f"all {self.case.T} tokens charged pro rata; weights prepared untimed), "
                f"{passes} pass(es), {seconds:.1f} s timed")


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def cpu_baseline(case, budget_s: float = 15.0, with_bwd: bool = False):
    """The oracle on a bounded sample (see OracleSample), repeated until ``budget_s`` of
    timed work; tokens/s = sampled assignments / k per timed second."""
    sample = OracleSample(case, with_bwd)
    total, passes = 0.0, 0
    while passes == 0 or total < budget_s:
        total += sample.run()
        passes += 1
    value = (sample.n_rows / case.k) * passes / total
    return {"value": value, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
            "sample": sample.describe(total, passes),
            "host_cores_visible": len(os.sched_getaffinity(0)), "host_cpu": _cpu_model()}


def run_reference(args, case):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    peaks = _peaks()
    del peaks
    bwd = args.pass_ == "fwdbwd"
    sample = OracleSample(case, bwd)            # weight preparation: once, untimed
    for _ in range(args.warmup):
        sample.run()
    vals, secs = [], 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):                 # one step = one timed pass over the sample
        s = sample.run()
        secs += s
        vals.append((sample.n_rows / case.k) / s)
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    info = {"cores": _threads(), "sample": sample.describe(secs, args.steps),
            "host_cpu": _cpu_model()}
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * case.T / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": _workload(case, "forward+backward" if bwd else "forward"),
                       "pass": "forward+backward" if bwd else "forward",
                       "T": case.T, "d": case.d, "f": case.f, "E": case.E, "k": case.k},
            "impl": "reference",
            "cpu_baseline": {"kind": "oracle", "cores": info["cores"], "sample": info["sample"],
                             "value": value, "unit": "tokens/s", "host_cpu": info["host_cpu"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": wall}
    print(json.dumps(line), flush=True)


# kernels launched per stage (route: routing + scatter; permute / bwd_dout: scheduling
# tables + per-token quantisation + pull gather; transposes: 4; wgrad: 2 GEMMs)
KERNELS_PER_STAGE = {"route": 2, "permute": 3, "gateup": 1, "down": 1, "combine": 1,
                     "bwd_dout": 3, "bwd_dgrad_down": 1, "bwd_dgrad_gateup": 1, "bwd_dx": 1,
                     "bwd_transpose": 4, "bwd_wgrad": 2, "bwd_swiglu": 1}


def run_ours(args, case):
    import ctypes

    import numpy as np
    import torch

    import synth
    import token_dispatch_grouped_top_b200 as moe

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    bwd = args.pass_ == "fwdbwd"
    # each rank draws its own batch (seed offset by rank); weights are shared by seed
    rcase = case.replace(seed=case.seed + 1000 * rank) if rank else case
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    x_bits, logits_np = synth.make_x(rcase), synth.make_logits(rcase)
    dout_bits = synth.make_dout(rcase) if bwd else None
    wg, wu, wd = synth.expert_weights_torch(case, dev)
    pw = moe.prepare_weights(wg, wu, wd, dims, with_backward=bwd)
    torch.cuda.synchronize()
    del wg, wu, wd
    torch.cuda.empty_cache()
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    logits = torch.from_numpy(logits_np).to(dev)
    ws = moe.workspace(dims, moe.OP_FORWARD, dev)
    out = torch.empty((case.T, case.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    saved = moe.alloc_saved(dims, dev) if bwd else None
    if bwd:
        dout = torch.from_numpy(dout_bits.view(np.int16)).view(torch.bfloat16).to(dev)
        wsb = moe.workspace(dims, moe.OP_BACKWARD, dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        grads = dict(dx=torch.empty((case.T, case.d), **bf),
                     dw_route=torch.empty((case.T, case.k), dtype=torch.float32, device=dev),
                     dWg=torch.empty((case.E, case.d, case.f), **bf),
                     dWu=torch.empty((case.E, case.d, case.f), **bf),
                     dWd=torch.empty((case.E, case.f, case.d), **bf))

    def step(xx=None, ll=None, dd=None, oo=None, gg=None):
        moe.forward(x if xx is None else xx, logits if ll is None else ll, pw, ws=ws,
                    out=out if oo is None else oo, saved=saved)
        if bwd:
            moe.backward(dout if dd is None else dd, pw, saved, ws=wsb,
                         outs=grads if gg is None else gg)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if moe.device_status(ws) != 0 or (bwd and moe.device_status(wsb) != 0):
        raise RuntimeError("device status latched during warm-up")

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    # The timed region: no per-stage events inside it (an event recorded between the
    # dispatch and the GEMM launched as its programmatic dependent would serialise them).
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        barrier()
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, dev, world)
    # The per-stage breakdown: the same steps again, each stage bracketed by events (stages
    # run back to back here, so their sum is at least the overlapped step time above).
    moe.profile_collect()
    moe.profile_enable(True)
    for _ in range(args.steps):
        step()
    barrier()
    moe.profile_enable(False)
    stages = moe.profile_collect()
    status = moe.device_status(ws) | (moe.device_status(wsb) if bwd else 0)

    # end to end through the public API with host buffers: every step copies its inputs
    # host -> device (pinned) and its results device -> host.  The copies run on two copy
    # streams with double-buffered device inputs and outputs, so step i+1's inputs and step
    # i's results cross PCIe while step i computes (as a training loop prefetches); the
    # timed region runs from the first input copy to the last result copy.
    x_h = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    lg_h = torch.from_numpy(logits_np).pin_memory()
    out_h = torch.empty((case.T, case.d), dtype=torch.bfloat16).pin_memory()
    nb = 2
    x_d = [torch.empty_like(x) for _ in range(nb)]
    lg_d = [torch.empty_like(logits) for _ in range(nb)]
    out_d = [out] + [torch.empty_like(out) for _ in range(nb - 1)]
    h2d = 2 * case.T * case.d + 4 * case.T * case.E
    d2h = 2 * case.T * case.d
    if bwd:
        do_h = torch.from_numpy(dout_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        dx_h = torch.empty((case.T, case.d), dtype=torch.bfloat16).pin_memory()
        dw_h = torch.empty((case.T, case.k), dtype=torch.float32).pin_memory()
        do_d = [torch.empty_like(dout) for _ in range(nb)]
        g_d = [grads] + [dict(grads, dx=torch.empty_like(grads["dx"]),
                              dw_route=torch.empty_like(grads["dw_route"]))
                         for _ in range(nb - 1)]
        h2d += 2 * case.T * case.d
        d2h += 2 * case.T * case.d + 4 * case.T * case.k
    h2s, d2s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d_done, comp_done, d2h_done = ([ev() for _ in range(nb)] for _ in range(3))

    def e2e_run(n):
        for i in range(n):
            b = i % nb
            if i >= nb:
                h2s.wait_event(comp_done[b])     # step i-nb has read input buffer b
            with torch.cuda.stream(h2s):
                x_d[b].copy_(x_h, non_blocking=True)
                lg_d[b].copy_(lg_h, non_blocking=True)
                if bwd:
                    do_d[b].copy_(do_h, non_blocking=True)
            h2d_done[b].record(h2s)
            stream.wait_event(h2d_done[b])
            if i >= nb:
                stream.wait_event(d2h_done[b])   # step i-nb's results have left buffer b
            step(x_d[b], lg_d[b], do_d[b] if bwd else None, out_d[b], g_d[b] if bwd else None)
            comp_done[b].record(stream)
            d2s.wait_event(comp_done[b])
            with torch.cuda.stream(d2s):
                out_h.copy_(out_d[b], non_blocking=True)
                if bwd:
                    dx_h.copy_(g_d[b]["dx"], non_blocking=True)
                    dw_h.copy_(g_d[b]["dw_route"], non_blocking=True)
            d2h_done[b].record(d2s)
        stream.wait_stream(d2s)
        stream.wait_stream(h2s)

    e2e_run(2)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2s)
    e2e_run(args.steps)
    e1.record(stream)
    barrier()
    ms_e2e = e0.elapsed_time(e1)
    ms_e2e = max_over_ranks(ms_e2e, dev, world)

    # the forward alone (inference: nothing saved for a backward), timed on its own
    fwd_only = None
    if bwd:
        for _ in range(args.warmup):
            moe.forward(x, logits, pw, ws=ws, out=out)
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            moe.forward(x, logits, pw, ws=ws, out=out)
        f1.record(stream)
        barrier()
        fwd_ms = max_over_ranks(f0.elapsed_time(f1), dev, world)
        moe.profile_collect()
        moe.profile_enable(True)
        for _ in range(args.steps):
            moe.forward(x, logits, pw, ws=ws, out=out)
        barrier()
        moe.profile_enable(False)
        fwd_stages = moe.profile_collect()
        status |= moe.device_status(ws)
        fwd_only = {"ms_per_step": fwd_ms / args.steps,
                    "tokens_per_s": job_tokens_per_s(world, case.T, args.steps, fwd_ms),
                    "stages_ms": {n: t / max(c, 1) for n, (t, c) in fwd_stages.items()}}

    peaks = _peaks()
    A = case.T * case.k
    mx_peak = 2.0 * peaks["bf16"]                      # MXFP8 dense = 2 x bf16 (nominal ratio)
    fl = layer_flops(case, True)
    cd = dims.c()
    lib = moe.load()
    w_bytes = sum(lib.moe_weights_bytes(ctypes.byref(cd), i) for i in range(4))
    # rows the kernels touch beyond the A assignments (tile padding), from the layout
    counts_h = (saved.bufs["counts"] if bwd else moe.workspace_view(
        ws, dims, moe.OP_FORWARD, "counts", 4 * case.E).view(torch.int32)).cpu().numpy()
    r_used = int(((counts_h + 127) // 128 * 128).sum())
    r_out = int((counts_h // 128 * 128 + (counts_h % 128 + 31) // 32 * 32).sum())
    # rows of the experts' partial last tiles; the SwiGLU backward runs in the dgrad GEMM's
    # epilogue for the other rows from d = 6144 on (the library's rule, include/moe.h)
    tail = int((counts_h % 128).sum()) if case.d >= 6144 else None
    alg_bytes = algorithmic_bytes(case, bwd, tail)
    impl_bytes = implementation_bytes(case, bwd, r_used, r_out, tail)
    stage_info = {}
    for name, (tot_ms, n) in stages.items():
        s = {"ms_per_launch": tot_ms / max(n, 1), "launches": n}
        if name in alg_bytes:
            s["alg_bytes"] = alg_bytes[name]
            s["gbs"] = alg_bytes[name] / (s["ms_per_launch"] * 1e-3) / 1e9
            s["frac_hbm"] = s["gbs"] / peaks["hbm"]
            s["overhead_bytes"] = impl_bytes[name] - alg_bytes[name]
        if name in fl:
            s["flops"] = fl[name]
            s["tflops"] = fl[name] / (s["ms_per_launch"] * 1e-3) / 1e12
            s["frac_mxfp8"] = s["tflops"] / mx_peak
        stage_info[name] = s
    g = stage_info.get("gateup", {"ms_per_launch": float("nan"), "tflops": float("nan")})
    roof_gateup = {"bound": "tensor", "kernel": "grouped_gemm_kernel<GATEUP_SWIGLU>",
                   "achieved": g["tflops"], "peak": mx_peak, "unit": "TFLOP/s",
                   "frac": g["tflops"] / mx_peak,
                   "traffic": GATEUP_TRAFFIC_RATIO * g["alg_bytes"] if "alg_bytes" in g else None,
                   "traffic_note": "DRAM bytes per launch, scaled from the mid-shape ncu capture",
                   "peak_note": f"2 x {peaks['src']} bf16 burst ({peaks['bf16']} TFLOP/s), "
                                f"MXFP8:bf16 nominal ratio 2"}
    roofline = roof_gateup
    if bwd and "bwd_wgrad" in stage_info:
        # the dominant kernel of a forward+backward step: the weight-gradient GEMM, whose
        # bf16 output (22.5 GB at this shape) makes it an HBM-write-bound launch pair
        w = stage_info["bwd_wgrad"]
        roofline = {"bound": "hbm", "kernel": "grouped_gemm_kernel<WGRAD_BF16> (2 launches)",
                    "achieved": w["gbs"], "peak": peaks["hbm"], "unit": "GB/s",
                    "frac": w["gbs"] / peaks["hbm"],
                    "traffic": WGRAD_TRAFFIC_RATIO * w["alg_bytes"],
                    "traffic_note": "DRAM bytes of the launch pair, scaled from the mid-shape "
                                    "ncu capture (ratio to algorithmic bytes 0.954)",
                    "peak_note": f"{peaks['src']} copy bandwidth (read+write); pure-write "
                                 f"streams on this pool measured {WRITE_ONLY_GBS:.0f} GB/s",
                    "frac_of_write_only": w["gbs"] / WRITE_ONLY_GBS}
    if fwd_only is not None:
        fwd_only["frac_mxfp8"] = (fl["gateup"] + fl["down"]) / (
            fwd_only["ms_per_step"] * 1e-3) / 1e12 / mx_peak
        fwd_only["layer_roofline"] = _safe_layer_summary(
            case, {n: {"ms_per_launch": v} for n, v in fwd_only["stages_ms"].items()},
            fwd_only["ms_per_step"], peaks, False)
    ms_step = ms / args.steps
    value = job_tokens_per_s(world, case.T, args.steps, ms)
    # the forward's own time: the forward-only leg when there is one (forward+backward),
    # else the timed step itself; the backward's from its stages
    fwd_ms = fwd_only["ms_per_step"] if fwd_only is not None else ms_step
    bwd_ms = sum(v["ms_per_launch"] for k, v in stage_info.items() if k.startswith("bwd"))
    step_flops = sum(fl[k] for k in fl if bwd or not k.startswith("bwd"))
    # kernels of the timed region: per step, those of the profiled steps' stages
    launches = sum(KERNELS_PER_STAGE[k] * v["launches"] for k, v in stage_info.items())
    pass_name = "forward+backward" if bwd else "forward"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "mxfp8 (e4m3 x e4m3, e8m0 scales, fp32 accumulate)", "data": "synthetic",
        "config": {"workload": _workload(case, pass_name), "pass": pass_name, "T": case.T,
                   "d": case.d, "f": case.f, "E": case.E, "k": case.k,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "no flush: every step streams 11.6 GB of MXFP8 weights (> 126 MB L2)"},
        "roofline": roofline,
        "roofline_gateup": roof_gateup,
        "fwd_tokens_per_s": world * case.T / (fwd_ms * 1e-3),
        "bwd_tokens_per_s": world * case.T / (bwd_ms * 1e-3) if bwd else None,
        "layer_tflops": step_flops / (ms_step * 1e-3) / 1e12,
        "layer_roofline": _safe_layer_summary(case, stage_info, ms_step, peaks, bwd, tail),
        "layer_frac_mxfp8": step_flops / (ms_step * 1e-3) / 1e12 / mx_peak,
        "fwd_frac_mxfp8": (fl["gateup"] + fl["down"]) / (fwd_ms * 1e-3) / 1e12 / mx_peak,
        "forward_only": fwd_only,
        "weights_gbs_fwd": w_bytes / (fwd_ms * 1e-3) / 1e9,
        "stages": stage_info,
        "gpu_launches": launches,
        "device_status": status,
        "e2e": {"value": job_tokens_per_s(world, case.T, args.steps, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "per step: x, logits" + (", dOut" if bwd else "") + " copied in from "
                        "pinned host memory; out" + (", dX, d(router weights)" if bwd else "") +
                        " copied back" + ("; the weight gradients stay on the device (an "
                                          "optimizer step consumes them there)" if bwd else "") +
                        "; copies of step i+1 / i overlap step i's compute on two copy streams"},
        "clocks": clk.summary(),
        "padded_rows": moe.padded_rows(dims),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, budget_s=args.cpu_budget, with_bwd=bwd)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ep(args, case):
    """Expert-parallel forward (moe_ep_prepare / moe_ep_experts / moe_ep_combine) with G
    ranks run on this one GPU in phase order, each rank's buffers separate and reached
    through the peer table: one JSON line (not the default line) with the step time, the
    per-stage times of the pull dispatch and the push combine and their bytes, and the
    single-GPU forward over the same tokens on the same GPU.  One GPU does every rank's
    work, so the line measures the expert-parallel kernels and the per-rank overhead, not
    multi-GPU scaling."""
    import numpy as np
    import torch

    import synth
    import token_dispatch_grouped_top_b200 as moe
    from token_dispatch_grouped_top_b200 import ep

    G = args.ep_ranks
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    E_loc, k = case.E // G, case.k
    wg, wu, wd = synth.expert_weights_torch(case, dev)
    dl = moe.Dims(case.T, case.d, case.f, E_loc, min(k, E_loc), case.score_fn)
    wl = [moe.prepare_weights(wg[r * E_loc:(r + 1) * E_loc].contiguous(),
                              wu[r * E_loc:(r + 1) * E_loc].contiguous(),
                              wd[r * E_loc:(r + 1) * E_loc].contiguous(), dl) for r in range(G)]
    dims = moe.Dims(case.T, case.d, case.f, case.E, k, case.score_fn)
    full = moe.prepare_weights(wg, wu, wd, dims)
    del wg, wu, wd
    torch.cuda.empty_cache()
    x = torch.from_numpy(synth.make_x(case).view(np.int16)).view(torch.bfloat16).to(dev)
    lg = torch.from_numpy(synth.make_logits(case)).to(dev)
    cuts = np.linspace(0, case.T, G + 1).astype(int)
    xs = [x[cuts[r]:cuts[r + 1]].contiguous() for r in range(G)]
    lgs = [lg[cuts[r]:cuts[r + 1]].contiguous() for r in range(G)]
    dims_r = [moe.Dims(int(cuts[r + 1] - cuts[r]), case.d, case.f, case.E, k, case.score_fn)
              for r in range(G)]
    dims_all = moe.Dims(case.T, case.d, case.f, case.E, k, case.score_fn)
    rws = [moe.workspace(dims_r[r], moe.OP_ROUTE, dev) for r in range(G)]
    states = [ep.prepare(dims_r[r], xs[r], lgs[r], ws=rws[r]) for r in range(G)]
    table = ep.peer_table([s.entry() for s in states], dev)
    wss = [ep.experts(dims_all, r, G, table, wl[r]) for r in range(G)]
    outs = [ep.combine(dims_r[r], states[r]) for r in range(G)]

    def step():
        for r in range(G):
            ep.prepare(dims_r[r], xs[r], lgs[r], ws=rws[r], state=states[r])
        for r in range(G):
            ep.experts(dims_all, r, G, table, wl[r], ws=wss[r])
        for r in range(G):
            ep.combine(dims_r[r], states[r], out=outs[r])

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    for _ in range(args.warmup):
        step()
    ms = timed(step, args.steps)
    ws1 = moe.workspace(dims, moe.OP_FORWARD, dev)
    out1 = torch.empty((case.T, case.d), dtype=torch.bfloat16, device=dev)
    for _ in range(args.warmup):
        moe.forward(x, lg, full, ws=ws1, out=out1)
    ms1 = timed(lambda: moe.forward(x, lg, full, ws=ws1, out=out1), args.steps)
    moe.profile_enable(True)
    moe.profile_collect()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    stages = moe.profile_collect()
    moe.profile_enable(False)
    status = max(moe.device_status(w) for w in wss)
    A = case.T * k
    pull_b = A * (case.d + case.d // 32) * 2          # token rows read from the sources, written
    push_b = A * (2 * case.d + case.d // 32) * 2      # output rows read, written to the sources
    st = {}
    for name, (tot, n) in stages.items():
        per = tot / max(n, 1)
        st[name] = {"ms_per_launch": per, "launches": n}
        if name in ("ep_pull", "ep_push"):
            bts = (pull_b if name == "ep_pull" else push_b) / G   # per rank launch
            st[name]["alg_bytes"] = bts
            st[name]["gbs"] = bts / (per * 1e-3) / 1e9
    line = {"metric": "expert-parallel forward, ranks emulated on one GPU", "ranks": G,
            "value": case.T * args.steps / (ms * args.steps * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "single_gpu_forward_ms": ms1, "steps": args.steps,
            "warmup": args.warmup, "stages": st, "device_status": status,
            "config": {"workload": case.name, "T": case.T, "d": case.d, "f": case.f,
                       "E": case.E, "k": k, "E_per_rank": E_loc}}
    print(json.dumps(line), flush=True)


def run_variants(args, case):
    """The layer's BF16 variant (forward, bf16 operands on tcgen05 kind::f16) beside the
    MXFP8 forward, and the router GEMM (logits = x . W_r^T, and its backward), timed on one
    GPU with CUDA events: one JSON line (not the default line)."""
    import numpy as np
    import torch

    import synth
    import token_dispatch_grouped_top_b200 as moe

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dims = moe.Dims(case.T, case.d, case.f, case.E, case.k, case.score_fn)
    x = torch.from_numpy(synth.make_x(case).view(np.int16)).view(torch.bfloat16).to(dev)
    lg = torch.from_numpy(synth.make_logits(case)).to(dev)
    peaks = _peaks()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    def stages(fn):
        moe.profile_collect()
        moe.profile_enable(True)
        for _ in range(args.steps):
            fn()
        torch.cuda.synchronize()
        moe.profile_enable(False)
        return {n: t / max(c, 1) for n, (t, c) in moe.profile_collect().items()}

    A = case.T * case.k
    gu_fl, dn_fl = 4.0 * A * case.d * case.f, 2.0 * A * case.d * case.f
    out = torch.empty((case.T, case.d), dtype=torch.bfloat16, device=dev)
    # MXFP8 forward (the layer as benchmarked), then the BF16 variant on the same inputs
    wg, wu, wd = synth.expert_weights_torch(case, dev)
    pw = moe.prepare_weights(wg, wu, wd, dims)
    ws = moe.workspace(dims, moe.OP_FORWARD, dev)
    ms_mx = timed(lambda: moe.forward(x, lg, pw, ws=ws, out=out))
    del pw, ws
    pw16 = moe.prepare_weights_bf16(wg, wu, wd, dims)
    del wg, wu, wd
    torch.cuda.empty_cache()
    ws16 = moe.workspace(dims, moe.OP_FORWARD_BF16, dev)
    f16 = lambda: moe.forward_bf16(x, lg, pw16, ws=ws16, out=out)   # noqa: E731
    ms_16 = timed(f16)
    st16 = stages(f16)
    status = moe.device_status(ws16)
    del pw16, ws16
    torch.cuda.empty_cache()
    bf16 = {"ms_per_step": ms_16, "tokens_per_s": case.T / (ms_16 * 1e-3),
            "stages_ms": st16, "mxfp8_forward_ms": ms_mx,
            "bf16_over_mxfp8_time": ms_16 / ms_mx}
    for name, fl in (("gateup", gu_fl), ("down", dn_fl)):
        if name in st16:
            tf = fl / (st16[name] * 1e-3) / 1e12
            bf16[name + "_tflops"] = tf
            bf16[name + "_frac_bf16"] = tf / peaks["bf16"]
    # router GEMM and its backward
    wr = torch.from_numpy(synth.make_router_weight(case).view(np.int16)).view(
        torch.bfloat16).to(dev)
    g = torch.from_numpy(synth.make_dlogits(case)).to(dev)
    wsr = moe.workspace(moe._router_dims(case.T, case.d, case.E), moe.OP_ROUTER, dev)
    logits = torch.empty((case.T, case.E), dtype=torch.float32, device=dev)
    ms_rf = timed(lambda: moe.router_logits(x, wr, ws=wsr, out=logits))
    ms_rb = timed(lambda: moe.router_grads(g, x, wr, ws=wsr))
    status = max(status, moe.device_status(wsr))
    rfl = 2.0 * case.T * case.d * case.E
    router = {"forward_ms": ms_rf, "forward_tflops": rfl / (ms_rf * 1e-3) / 1e12,
              "backward_ms": ms_rb, "backward_tflops": 2 * rfl / (ms_rb * 1e-3) / 1e12,
              "note": "backward includes the bf16 copies of G, G^T, W_r^T and x^T"}
    line = {"metric": "BF16 variant forward and router GEMM, one GPU", "steps": args.steps,
            "warmup": args.warmup, "bf16_variant": bf16, "router": router,
            "peak_bf16_tflops": peaks["bf16"], "peak_src": peaks["src"],
            "device_status": status,
            "config": {"workload": case.name, "T": case.T, "d": case.d, "f": case.f,
                       "E": case.E, "k": case.k}}
    print(json.dumps(line), flush=True)


def sweep(args):
    """One JSON line per synthetic configuration and pass (forward, forward+backward).
    Not the default line: a table for the design notes."""
    import subprocess as sp
    for name in ("tiny", "mid", "dsv3", "imbalance"):
        for pass_ in ("fwd", "fwdbwd"):
            cmd = [sys.executable, os.path.abspath(__file__), "--config", name, "--steps",
                   str(args.steps), "--warmup", str(args.warmup), "--no-cpu-baseline",
                   "--pass", pass_]
            r = sp.run(cmd, capture_output=True, text=True)
            line = r.stdout.strip().splitlines()[-1] if r.stdout.strip() else json.dumps(
                {"config": name, "pass": pass_, "error": r.stderr[-500:]})
            print(line, flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=CONFIG_NAME)
    ap.add_argument("--pass", dest="pass_", default="fwdbwd", choices=["fwd", "fwdbwd"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--sweep", action="store_true", help="every synthetic config, one line each")
    ap.add_argument("--variants", action="store_true",
                    help="the BF16 layer variant and the router GEMM, one JSON line")
    ap.add_argument("--ep-ranks", type=int, default=0,
                    help="expert-parallel forward with this many ranks emulated on one GPU")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    import synth
    case = synth.CONFIGS[args.config]
    if args.sweep:
        sweep(args)
        return
    if args.ep_ranks:
        run_ep(args, case)
        return
    if args.variants:
        run_variants(args, case)
        return
    if args.impl == "reference":
        run_reference(args, case)
    else:
        run_ours(args, case)


if __name__ == "__main__":
    main()
