"""Benchmark of one windowed RIB attention + CLA gate layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload full] [--impl ours|reference]

A step is one pass of the whole hot path over the workload's input resident
in HBM: the content projections (rib_qkv_project), the CLA gate (cla_gate:
depthwise 3x3 then pointwise + sigmoid) and the fused windowed RIB attention
with the gate multiply and window reverse (rib_window_attention). The
position features are computed once per window size before timing (they are
a cache, reported once as pos_encode_ms).

The default workload is the 640x360 layer (230,400 tokens, C=180, 6 heads,
R=16, window 64). value = algorithmic TFLOP/s of the layer (attention
2N^2(dh+R)+2N^2 dh per window-head plus the projection, depthwise and
pointwise convs), summed over ranks and divided by the slowest rank's time.
Between timed steps a 256 MB buffer is written to flush the 126 MB L2; only
the steps are inside the CUDA-event windows.

Multi-GPU: every rank runs its own independent layer (windows and images are
independent units; no data-path collective), so scaling is weak; the only
collectives are the timing barrier and the max over ranks.

--impl reference times the fp64 oracle on the host cores on a bounded sample
of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "windowed RIB attention ms/layer & TFLOP/s at 640×360 tokens, % of BF16 peak"
UNIT = "TFLOP/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="full")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-windows", type=int, default=24, help="windows of the oracle's bounded CPU sample")
    ap.add_argument("--window", type=int, default=0, help="override the workload's window (lite: 16, 32 or 64)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads' sub-records (train, lite windows, stack) of the default run")
    ap.add_argument("--extra-steps", type=int, default=10, help="timed steps of each sub-record")
    return ap.parse_args()


def env_rank():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (ms) over the process group:
    a multi-GPU step is as slow as its slowest rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_tflops(world: int, flops_per_rank_step: float, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank processes its own copy of the workload
    (weak scaling), so the job does world * flops per step in the slowest
    rank's time."""
    return world * flops_per_rank_step * steps / (ms / 1e3) / 1e12


def layer_flops(s) -> dict:
    T = s.B * s.H * s.W
    f = {
        "attention": s.attention_flops(),
        "projection": 2.0 * T * s.C * 3 * s.C,
        "pointwise": 2.0 * T * s.C * s.C,
        "depthwise": 2.0 * 9 * T * s.C,
    }
    f["layer"] = sum(f.values())
    return f


def measured_peaks():
    """The measured HBM copy and bf16 GEMM peaks of this GPU model when the
    peaks file is present and readable, else the fallback figures."""
    fallback = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            with open(p) as fh:
                d = json.load(fh)
            out = {k: float(d[k]) for k in fallback if k in d}
            if "bf16_tflops" in out and out["bf16_tflops"] > 0:
                return {**fallback, **out}, "measured"
        except (OSError, ValueError, TypeError):
            pass
    return fallback, "fallback"


def source_code_hash(path: str) -> str:
    """First 16 hex digits of the sha256 of a C/CUDA source with its comments
    removed and its whitespace collapsed: a record taken on one version of a
    kernel stays valid across edits of its comments, and only those."""
    with open(path) as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"\s+", " ", text).strip()
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def kernel_traffic(kernel_src: str, workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current code of the kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    e = d.get(workload)
    if not e or e.get("source_code_sha256_16") != source_code_hash(kernel_src):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of this GPU's SM clock and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax = max(smax, float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline(wl_name: str, n_windows: int):
    """The oracle, as it stands, on a bounded sample of the workload's windows."""
    import numpy as np
    import oracle
    from windowed_attention_b200.workloads import WORKLOADS, make_inputs
    wl = WORKLOADS[wl_name]
    s = wl.layer
    inp = make_inputs(wl_name)
    nw = s.n_windows
    ids = sorted(set(int(i) for i in np.linspace(0, nw - 1, min(n_windows, nw))))
    cores = oracle.oracle_cores()
    t0 = time.perf_counter()
    oracle.rib_layer_forward_windows(inp["X"], inp, s.heads, s.R, s.L, s.window, ids, threads=cores)
    dt = time.perf_counter() - t0
    f = layer_flops(s)
    flops = f["layer"] * len(ids) / nw
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(ids)} of {nw} windows (all {s.heads} heads, projections and gate of those windows), "
                      f"{dt:.1f} s wall, fp64 NumPy, threads over (window, head)"}


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return
    import numpy as np
    import oracle
    from windowed_attention_b200.workloads import WORKLOADS, make_inputs
    wl = WORKLOADS[args.workload]
    s = wl.layer
    inp = make_inputs(args.workload)
    cores = oracle.oracle_cores()
    nw = s.n_windows
    f = layer_flops(s)
    per_window = f["layer"] / nw

    def step(i):
        oracle.rib_layer_forward_windows(inp["X"], inp, s.heads, s.R, s.L, s.window, [i % nw], threads=cores)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = per_window * args.steps / dt / 1e12
    sample = f"one window of {nw} (all {s.heads} heads) per step, fp64 NumPy oracle, {cores} threads"
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": wl.description, "name": args.workload,
                                         "tokens": s.B * s.H * s.W, "window": s.window,
                                         "flops_per_step": per_window, "sample_per_step": "1 window",
                                         "parallelism": "the fp64 oracle on rank 0's host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


class Case:
    """One workload prepared on the device: its timed parts (each a callable
    that launches this library's kernels on the current stream), the FLOPs of
    a step and the number of launches a step makes."""

    def __init__(self, name, shape, parts, flops, launches, **extra):
        self.name, self.shape, self.parts, self.flops, self.launches = name, shape, parts, flops, launches
        self.__dict__.update(extra)


def build_case(name, dev, window=0):
    """Device buffers and step functions of a workload: 'full' (640x360
    layer), 'lite' (320x180, one window), 'train' (forward + backward chain at
    16 x 96x96, window 96) or 'stack' (six blocks, windows 16,32,64,16,32,64)."""
    import torch
    from dataclasses import replace
    from windowed_attention_b200 import _lib
    from windowed_attention_b200.layer import RibLayer, RibStack
    from windowed_attention_b200.workloads import WORKLOADS, ffn_hidden, make_inputs

    wl = WORKLOADS[name]
    s = wl.layer if not window else replace(wl.layer, window=window)
    inp = make_inputs(name, layer=s, with_grad=wl.backward)
    t0 = time.perf_counter()
    if wl.blocks > 1:
        stack = RibStack(s, inp["blocks"], wl.windows, dev, ffns=inp.get("ffns"))
        layer = stack.layers[0]
    else:
        stack = None
        layer = RibLayer(s, inp, dev)
    torch.cuda.synchronize()
    pos_ms = (time.perf_counter() - t0) * 1e3
    X = inp["X"].to(dev, torch.bfloat16).contiguous()
    dh = s.C // s.heads
    qp, kp = layer.pos_cache(s.window)
    desc = _lib.attn_desc(s.B, s.H, s.W, s.C, s.heads, s.R, s.window, 1.0)
    f = layer_flops(s)

    # the training step keeps the gate's depthwise output for the backward
    gate_ws = layer.ws if wl.backward else None

    def proj_and_gate(Xd=X):
        _lib.rib_qkv_project(Xd, s.B, s.H, s.W, s.C, s.heads, s.window, layer.Wq, layer.Wk, layer.Wv,
                             1.0 / math.sqrt(dh), layer.Qc, layer.Kc, layer.V)
        _lib.cla_gate(Xd, s.B, s.H, s.W, s.C, layer.Wdw, layer.bdw, layer.Wpw, layer.bpw, layer.gate, gate_ws)

    def attention(Y=None):
        _lib.rib_window_attention(desc, layer.Qc, layer.Kc, layer.V, qp, kp, layer.gate, None,
                                  layer.Y if Y is None else Y)

    common = dict(wl=wl, layer=layer, stack=stack, X=X, desc=desc, qp=qp, kp=kp, pos_ms=pos_ms,
                  proj_and_gate=proj_and_gate, attention=attention, windows=(s.window,))
    if stack is not None:
        per = [layer_flops(replace(s, window=w)) for w in wl.windows]
        flops = {"attention": sum(x["attention"] for x in per), "layer": sum(x["layer"] for x in per)}
        common["windows"] = tuple(wl.windows)
        # per block: LayerNorm 1, projection 1, gate 1, attention 1; plus the
        # widening of the bf16 input into the fp32 residual stream
        launches = 4 * len(wl.windows) + 1
        if wl.ffn:
            # ConvFFN per block: 2 T C hidden flops each linear map, 9 taps of
            # the depthwise conv on the hidden features; launches: LayerNorm,
            # the first map, the fused depthwise + second map
            T = s.B * s.H * s.W
            hid = ffn_hidden(s.C)
            flops["ffn"] = len(wl.windows) * (2.0 * T * s.C * hid * 2 + 2.0 * 9 * T * hid)
            flops["layer"] += flops["ffn"]
            launches += 3 * len(wl.windows)
        return Case(name, s, [("stack", lambda: stack.forward(X))], flops, launches, **common)
    if not wl.backward:
        # projection 1, gate 1 (fused depthwise + pointwise), attention 1
        return Case(name, s, [("projection_and_gate", proj_and_gate), ("attention", attention)], f, 3, **common)

    # training step: forward saving lse and O, then the backward chain
    dY = inp["dY"].to(dev, torch.bfloat16).contiguous()
    T = s.B * s.H * s.W
    Tp = s.B * s.Hp * s.Wp
    e = torch.empty
    tb = {k: e(Tp * s.heads * 32, dtype=torch.float32, device=dev) for k in ("dQc", "dKc", "dV")}
    tb["dO"] = e(Tp * s.heads * 32, dtype=_lib.v_dtype(), device=dev)
    tb["Dsum"] = e(s.B * s.heads * s.Hp * s.Wp, dtype=torch.float32, device=dev)
    tb["lse"] = torch.empty_like(tb["Dsum"])
    tb["O"] = e(T * s.heads * layer.DP, dtype=torch.bfloat16, device=dev)
    tb["dG"] = e(s.B, s.H, s.W, s.C, dtype=torch.bfloat16, device=dev)
    for k in ("dQp", "dKp"):
        tb[k] = e(s.heads * s.window * s.window * s.R, dtype=torch.float32, device=dev)
    tb["ws"] = e(_lib.rib_window_attention_bwd_workspace_size(desc) // 4, dtype=torch.float32, device=dev)
    tb["dWh"] = e(s.enc_dim, s.hidden, dtype=torch.float32, device=dev)
    tb["dbh"] = e(s.hidden, dtype=torch.float32, device=dev)
    tb["dWpq"] = e(s.hidden, s.heads * s.R, dtype=torch.float32, device=dev)
    tb["dWpk"] = torch.empty_like(tb["dWpq"])
    tb["pws"] = e(_lib.rib_pos_encode_bwd_workspace_size(layer.mlp, s.window) // 4, dtype=torch.float32, device=dev)
    tb["dX"] = e(s.B, s.H, s.W, s.C, dtype=torch.float32, device=dev)
    for k in ("dWq", "dWk", "dWv", "dWpw"):
        tb[k] = e(s.C, s.C, dtype=torch.float32, device=dev)
    tb["dWdw"] = e(s.C, 3, 3, dtype=torch.float32, device=dev)
    tb["dbdw"] = e(s.C, dtype=torch.float32, device=dev)
    tb["dbpw"] = e(s.C, dtype=torch.float32, device=dev)
    tb["gws"] = e(_lib.cla_gate_bwd_workspace_size(s.B, s.H, s.W, s.C) // 4, dtype=torch.float32, device=dev)
    tb["qws"] = e(_lib.rib_qkv_project_bwd_workspace_size(s.B, s.H, s.W, s.C, s.heads), dtype=torch.uint8, device=dev)

    def attn_fwd():
        _lib.rib_window_attention(desc, layer.Qc, layer.Kc, layer.V, qp, kp, layer.gate, None, layer.Y,
                                  tb["lse"], tb["O"])

    def bwd_prep():
        _lib.rib_attention_bwd_prep(desc, dY, layer.gate, tb["O"], tb["dO"], tb["Dsum"], tb["dG"])

    def attn_bwd():
        _lib.rib_window_attention_bwd(desc, layer.Qc, layer.Kc, layer.V, qp, kp, tb["lse"], tb["dO"], tb["Dsum"],
                                      tb["dQc"], tb["dKc"], tb["dV"], tb["dQp"], tb["dKp"], tb["ws"])

    def mlp_bwd():
        _lib.rib_pos_encode_bwd(layer.mlp, s.window, tb["dQp"], tb["dKp"], tb["dWh"], tb["dbh"], tb["dWpq"],
                                tb["dWpk"], tb["pws"])

    def proj_bwd():
        _lib.rib_qkv_project_bwd(X, s.B, s.H, s.W, s.C, s.heads, s.window, layer.Wq, layer.Wk, layer.Wv,
                                 1.0 / math.sqrt(dh), tb["dQc"], tb["dKc"], tb["dV"], tb["dX"], tb["dWq"],
                                 tb["dWk"], tb["dWv"], tb["qws"])

    def gate_bwd():
        _lib.cla_gate_bwd(X, s.B, s.H, s.W, s.C, layer.Wdw, layer.Wpw, layer.ws, tb["dG"], tb["dX"], tb["dWdw"],
                          tb["dbdw"], tb["dWpw"], tb["dbpw"], tb["gws"])

    f = dict(f)
    f["attention_bwd"] = s.attention_bwd_flops()
    f["layer"] += f["attention_bwd"]
    parts = [("projection_and_gate", proj_and_gate), ("attention_fwd", attn_fwd), ("bwd_prep", bwd_prep),
             ("attention_bwd", attn_bwd), ("mlp_bwd", mlp_bwd), ("projection_bwd", proj_bwd),
             ("gate_bwd", gate_bwd)]
    return Case(name, s, parts, f, _lib.LAUNCHES["train_step"], tb=tb, dY=dY, **common)


def time_case(case, steps, flush, stream):
    """Run `steps` steps of the case with a flush of L2 between them (outside
    the event windows); returns per-part lists of CUDA-event milliseconds."""
    import torch
    n = len(case.parts)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        for k, (_, fn) in enumerate(case.parts):
            fn()
            ev[i][k + 1].record(stream)
    torch.cuda.synchronize()
    per = {label: [ev[i][k].elapsed_time(ev[i][k + 1]) for i in range(steps)]
           for k, (label, _) in enumerate(case.parts)}
    per["step"] = [ev[i][0].elapsed_time(ev[i][n]) for i in range(steps)]
    return per


def roofline_entry(flops, ms, peak, peak_src, kernel, traffic=None):
    achieved = flops / (ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic, "kernel": kernel, "peak_source": f"{peak_src} bf16 burst"}


def extra_records(dev, stream, flush, steps, warmup, peak, peak_src):
    """The other workloads, timed in the same run (CUDA events, L2 flushed
    between steps): the training step at window 96 (forward + backward
    attention rooflines), the lite layer at windows 16/32/64, the six-block
    stack and the six full SST blocks (with ConvFFN). Each entry: ms per step,
    TFLOP/s and the attention kernel's roofline."""
    import torch
    import windowed_attention_b200 as rib
    out = {}
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    sampler.start()
    for name, window in (("train", 0), ("lite", 16), ("lite", 32), ("lite", 64), ("stack", 0), ("sst", 0)):
        case = build_case(name, dev, window)
        for _ in range(warmup):
            for _, fn in case.parts:
                fn()
        torch.cuda.synchronize()
        rib.rib_device_error()
        per = time_case(case, steps, flush, stream)
        rib.rib_device_error()
        ms = statistics.mean(per["step"])
        rec = {"workload": case.wl.description, "window": (list(case.windows) if len(case.windows) > 1
                                                            else case.windows[0]),
               "ms_per_step": ms, "tflops": case.flops["layer"] / (ms / 1e3) / 1e12,
               "flops_per_step": case.flops["layer"], "steps": steps,
               "breakdown_ms": {k: statistics.mean(v) for k, v in per.items() if k != "step"},
               "gpu_launches_per_step": case.launches}
        if name == "train":
            rec["roofline_fwd"] = roofline_entry(case.flops["attention"], rec["breakdown_ms"]["attention_fwd"], peak,
                                                 peak_src, "rib_attn_fwd_kernel")
            rec["roofline_bwd"] = roofline_entry(case.flops["attention_bwd"], rec["breakdown_ms"]["attention_bwd"],
                                                 peak, peak_src, "rib_attn_bwd_dq + rib_attn_bwd_dkv + window sums")
        elif name == "lite":
            rec["roofline"] = roofline_entry(case.flops["attention"], rec["breakdown_ms"]["attention"], peak, peak_src,
                                             "rib_attn_fwd_kernel")
        key = name if name != "lite" else f"lite_w{window}"
        out[key] = rec
        del case
        torch.cuda.empty_cache()
    out["clocks"] = sampler.stop()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = env_rank()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    import windowed_attention_b200 as rib
    from windowed_attention_b200 import _lib

    rib.load()
    from dataclasses import replace
    case = build_case(args.workload, dev, args.window)
    s, wl, layer, X = case.shape, case.wl, case.layer, case.X
    T = s.B * s.H * s.W
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        for _, fn in case.parts:
            fn()
    torch.cuda.synchronize()
    rib.rib_device_error()

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id)
    K = args.steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    per = time_case(case, K, flush, stream)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    rib.rib_device_error()
    total_ms = sum(per["step"])

    # end to end through the public API: pinned host input -> layer -> host output
    Xh = X.cpu().pin_memory()
    Yout = layer.Y if case.stack is None else case.stack.x
    Yh = torch.empty(Yout.shape, dtype=Yout.dtype).pin_memory()

    def e2e_step():
        X.copy_(Xh, non_blocking=True)
        for _, fn in case.parts:
            fn()
        Yh.copy_(Yout, non_blocking=True)

    # Forward layer: the copies of step i+1's input and step i's output run on
    # their own streams (PCIe is full duplex) beside the kernels of step i, with
    # two device input and two device output buffers. Every step still copies
    # its whole input in and its whole output out inside the timed region.
    pipelined = not wl.backward and case.stack is None
    if pipelined:
        Xd = [X, torch.empty_like(X)]
        Yd = [layer.Y, torch.empty_like(layer.Y)]
        Yhb = [Yh, torch.empty(Yout.shape, dtype=torch.bfloat16).pin_memory()]
        s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n):
            s_h2d.wait_stream(stream)
            with torch.cuda.stream(s_h2d):
                Xd[0].copy_(Xh, non_blocking=True)
                ev_in[0].record(s_h2d)
            for i in range(n):
                b = i & 1
                if i + 1 < n:   # next input into the buffer step i-1 used
                    if i >= 1:
                        s_h2d.wait_event(ev_done[b ^ 1])
                    with torch.cuda.stream(s_h2d):
                        Xd[b ^ 1].copy_(Xh, non_blocking=True)
                        ev_in[b ^ 1].record(s_h2d)
                stream.wait_event(ev_in[b])
                if i >= 2:      # output buffer b read back by step i-2
                    stream.wait_event(ev_out[b])
                case.proj_and_gate(Xd[b])
                case.attention(Yd[b])
                ev_done[b].record(stream)
                s_d2h.wait_event(ev_done[b])
                with torch.cuda.stream(s_d2h):
                    Yhb[b].copy_(Yd[b], non_blocking=True)
                    ev_out[b].record(s_d2h)
            for b in range(min(n, 2)):
                stream.wait_event(ev_out[b])
    else:
        def e2e_run(n):
            for _ in range(n):
                e2e_step()

    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    e2e_run(K)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if pipelined:
        # the host copy of the last step's output equals the device output
        # (same input every step, deterministic kernels)
        last = (K - 1) & 1
        if not torch.equal(Yhb[last], Yd[last].cpu()):
            raise RuntimeError("end-to-end output differs from the device result")
    e2e_ms = e0.elapsed_time(e1)

    if world > 1:
        total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)

    f = case.flops
    windows = case.windows
    value = whole_job_tflops(world, f["layer"], K, total_ms)
    e2e_value = whole_job_tflops(world, f["layer"], K, e2e_ms)
    peaks, peak_src = measured_peaks()
    if wl.backward:
        attn_ms = statistics.mean(per["attention_fwd"]) + statistics.mean(per["attention_bwd"])
    elif case.stack is not None:
        attn_ms = statistics.mean(per["stack"])
    else:
        attn_ms = statistics.mean(per["attention"])
    attn_flops = f["attention"] + f.get("attention_bwd", 0.0)
    peak = float(peaks["bf16_tflops"])
    traffic = kernel_traffic(os.path.join(ROOT, "windowed_attention_b200", "csrc", "window_attention.cu"),
                             args.workload)
    roof = roofline_entry(attn_flops, attn_ms, peak, peak_src,
                          "rib_attn_fwd + rib_attn_bwd_dq/dkv (timed together)" if wl.backward
                          else ("the whole stack step" if case.stack is not None else "rib_attn_fwd_kernel"),
                          traffic)
    # the forward attention's two other ceilings: the MMAs it issues with the
    # padded operand widths (content DP + rank 16 for QK, 32 V columns for
    # P.V), and one exponential per score on MUFU (16 per clock per SM)
    shapes = [replace(s, window=wv) for wv in windows]
    dp = layer.DP
    roof["forward_padded_flops"] = sum(x.n_windows * x.heads * 2.0 * (x.window ** 4) * (dp + x.R + 32) for x in shapes)
    exps = sum(x.n_windows * x.heads * float(x.window ** 4) for x in shapes)
    sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    roof["forward_exps"] = exps
    roof["forward_exp_floor_ms"] = exps / (16.0 * n_sm * sm_mhz * 1e6) * 1e3
    breakdown = {k: statistics.mean(v) for k, v in per.items() if k != "step"}
    if "attention" in per:
        breakdown["attention_min"] = min(per["attention"])
    breakdown["pos_encode_once"] = case.pos_ms
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.description, "name": args.workload, "tokens": T,
                   "window": list(windows) if len(windows) > 1 else s.window,
                   "flops_per_step": f["layer"], "attention_flops": f["attention"],
                   "l2": "256 MB buffer written between timed steps (outside the event windows)",
                   "parallelism": f"replicas x{world} (independent windows, no data-path collective)"},
        "breakdown_ms": breakdown,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": X.numel() * 2,
                "d2h_bytes_per_step": Yout.numel() * Yout.element_size(), "ms_per_step": e2e_ms / K,
                "copies": ("overlapped with the kernels: copy streams, double-buffered device input/output"
                           if pipelined else "in line on the compute stream")},
        "gpu_launches": case.launches * K,
        "clocks": clocks,
    }
    del case, layer
    torch.cuda.empty_cache()
    if args.workload == "full" and not args.no_extras and world == 1:
        out["extra"] = extra_records(dev, stream, flush, args.extra_steps, 3, peak, peak_src)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_windows)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
