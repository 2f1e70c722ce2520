#!/usr/bin/env python
"""bench.py -- quantized GEMM TOPS and HBM GB/s per precision (q8 / W8A8 / q4)
on B200, with the fraction of roofline of the dominant kernel.

Workload (one "step"): the layer-sequence replay of a synthetic diffusion
transformer -- 24 blocks x {qkv 1536->4608, out 1536->1536, up 1536->6144,
down 6144->1536} at M = 432 tokens (2 CFG halves x 216 latent frames), 8
denoising steps, at each of the three precisions, with the steering add
(alpha = 0.3, unit-norm v) on block 12's out-projection. This is the shape of
the pages' generation loop ("Results": 8 steps; "What aria is": the
denoising loop replayed as one CUDA graph; "Live steering while streaming":
the steering strength lives inside the captured graph, here a device-side
schedule read by the steered launch of each step). Weights are packed once
at load, as on the pages. Per precision one CUDA graph holds the 8-step loop
(768 GEMM launches; W8A8 adds 768 per-token activation quantisations).

Beside the step, outside `value`: the unquantised fp16 rung of the
precision ladder on the same replay, the W8A8 leg with the activation
quantisation fused into the GEMM launch, the steering on/off delta (the same
graphs with the schedule set to 0), every per-shape case of the benchmark
configurations (`per_config`: q8 d=1024 at M in {1,16,432}, W8A8 d=1536 at
M in {432,4096} with its activation quantisation, q4 d=1536 at M in
{1,8,432}, the fp16 rung, the packs), the end-to-end loop through host
memory, and the CPU oracle.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --sweep            # the per-shape cases only, one JSON line each
    python bench.py --case q4 --shape 6144x1536 --m 432   # one case (ncu captures)

N > 1 runs N independent replicas (one process per GPU, launched by torchrun),
no collective on the data path; the timed region is bracketed by barriers
and the slowest rank's device time is reported. Rank 0 prints ONE JSON line.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synthetic  # noqa: E402

METRIC = "quantized GEMM TOPS and HBM GB/s per precision (q8/W8A8/q4), % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_F16 = 4.5 / 2.25       # nominal dense int8 : fp16 ratio
WORKLOAD = ("layer-sequence replay: 24 blocks x {qkv 1536->4608, out 1536->1536, up 1536->6144, "
            "down 6144->1536}, M=432, 8 steps, at q8, W8A8 and q4; steering alpha=0.3 on block 12 out-proj")


# ----------------------------------------------------------------- helpers --

def kernel_source_sha256():
    """Hash of the CUDA sources' code: comments and whitespace are stripped,
    so the traffic record stays valid across comment-only edits and goes
    stale on any change to the code."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "int8_int4_b200", "csrc", "*"))):
        with open(f, encoding="utf-8") as fh:
            t = fh.read()
        t = re.sub(r"/\*.*?\*/", " ", t, flags=re.S)
        t = re.sub(r"//[^\n]*", " ", t)
        h.update(os.path.basename(f).encode() + b"\0" + " ".join(t.split()).encode() + b"\0")
    return h.hexdigest()


def measured_traffic(kernel, alg_bytes_per_launch):
    """DRAM bytes per launch from the committed ncu record, scaled from the
    captured case to this launch's algorithmic bytes; None if the kernel
    sources changed since the counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
            rec = json.load(f)
        if rec["source_sha256"] != kernel_source_sha256():
            return None, "stale: kernel changed since the ncu capture"
        k = rec["kernels"][kernel]
        return (k["dram_bytes"] * alg_bytes_per_launch / k["algorithmic_bytes"],
                f"ncu capture of {k['case']} ({k['dram_bytes']} B DRAM for {k['algorithmic_bytes']} B "
                f"algorithmic), scaled to this launch's algorithmic bytes")
    except Exception as e:  # no record
        return None, f"unavailable ({type(e).__name__})"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.out, stderr=subprocess.DEVNULL)
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

    def summary(self):
        if self.proc is None or self.out is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.out.seek(0)
        rows = []
        for line in self.out:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            bus = parts[0].lower()
            if self.bus_id and not (bus.endswith(self.bus_id[-12:]) or self.bus_id.endswith(bus[-12:])):
                continue
            rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        loaded = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(values, ws):
    """element-wise max of a list of floats over all ranks"""
    if ws == 1:
        return list(values)
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def sum_over_ranks(values, ws):
    if ws == 1:
        return list(values)
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.cpu().tolist()


# ------------------------------------------------------------ work account --

LINEARS = synthetic.D1536
M = synthetic.REPLAY_M
BLOCKS = synthetic.REPLAY_BLOCKS
STEPS = synthetic.REPLAY_STEPS


def gemm_ops(m, n, k):
    return 2.0 * m * n * k


def bytes_wo(fmt, m, n, k, steer):
    w = n * k if fmt == "q8" else n * k // 2
    s = 4 * n if fmt == "q8" else 2 * n * (k // 32)
    return w + s + 2 * m * k + 2 * m * n + (4 * n if steer else 0)


def bytes_w8a8(m, n, k, steer):
    return m * k + 4 * m + n * k + 4 * n + 2 * m * n + (4 * n if steer else 0)


def bytes_f16(m, n, k, steer):
    return 2 * n * k + 2 * m * k + 2 * m * n + (4 * n if steer else 0)


def bytes_act_quant(m, k):
    return 3 * m * k + 4 * m


def bytes_w8a8_fused(m, n, k, steer):
    """W8A8 from fp16 activations in one launch: the fp16 X read once, the
    packed weights and scales, the fp16 output (the int8 codes' round trip
    through the workspace is not algorithmic work)."""
    return 2 * m * k + n * k + 4 * n + 2 * m * n + (4 * n if steer else 0)


def bytes_pack(fmt, n, k):
    return 2 * n * k + (n * k + 4 * n if fmt == "q8" else n * k // 2 + 2 * n * (k // 32))


def step_account():
    """ops and algorithmic bytes of one 8-step replay, per precision / kernel"""
    acc = {"q8": [0.0, 0.0], "w8a8_gemm": [0.0, 0.0], "act_quant": [0.0, 0.0], "q4": [0.0, 0.0],
           "f16": [0.0, 0.0], "w8a8": [0.0, 0.0]}
    for b in range(BLOCKS):
        for name, k, n in LINEARS:
            st = (b == synthetic.REPLAY_STEER_BLOCK and name == "out")
            o = gemm_ops(M, n, k)
            acc["q8"][0] += o
            acc["q8"][1] += bytes_wo("q8", M, n, k, st)
            acc["q4"][0] += o
            acc["q4"][1] += bytes_wo("q4", M, n, k, st)
            acc["w8a8_gemm"][0] += o
            acc["w8a8_gemm"][1] += bytes_w8a8(M, n, k, st)
            acc["act_quant"][1] += bytes_act_quant(M, k)
            acc["w8a8"][0] += o
            acc["w8a8"][1] += bytes_w8a8_fused(M, n, k, st)
            acc["f16"][0] += o
            acc["f16"][1] += bytes_f16(M, n, k, st)
    return {k: (v[0] * STEPS, v[1] * STEPS) for k, v in acc.items()}


def roofs(peaks):
    """Roofline denominators. A kernel timed inside the replay (a ~30 ms step
    at full clocks, no power-cap throttling in the clock record) or alone in
    a per-shape graph takes the burst GEMM figure; int8 is the fp16/bf16
    figure times the nominal dense int8 : fp16 ratio (2)."""
    f16 = peaks["bf16_tflops"]
    return {"f16": f16, "i8": f16 * INT8_OVER_F16, "hbm": peaks["hbm_gbs"]}


def roof_entry(ops, byts, seconds, tensor_peak, hbm):
    """TOPS, GB/s, the binding roof (the larger ideal time) and the fraction
    of it that this time reaches."""
    d = {"us": seconds * 1e6, "gbs": byts / seconds / 1e9, "hbm_frac": byts / seconds / 1e9 / hbm}
    if ops:
        d["tops"] = ops / seconds / 1e12
        d["tensor_frac"] = d["tops"] / tensor_peak
        d["bound"] = "tensor" if ops / (tensor_peak * 1e12) >= byts / (hbm * 1e9) else "hbm"
    else:
        d["bound"] = "hbm"
    d["frac"] = d["tensor_frac"] if d["bound"] == "tensor" else d["hbm_frac"]
    return d


# ------------------------------------------------------------- our arm ------

class Replay:
    """Device-resident workload and its CUDA graphs.

    Each precision has its own output buffers (the step's results stay
    distinct), the fp16 rung keeps the unquantised weights, and the inputs
    exist in `buffers` device copies so the end-to-end loop can copy the next
    step's inputs while the current step computes. The steered launch of
    step s reads its strength from `alpha[s]` (device memory)."""

    ORDER = ("q8", "act_quant", "w8a8_gemm", "q4")        # the timed step
    EXTRA = ("w8a8_fused", "f16")                         # timed beside it
    LAUNCHES_PER_STEP = len(ORDER) * STEPS * BLOCKS * len(LINEARS)

    def __init__(self, dev, buffers=1, fp16=True):
        import int8_int4_b200 as aq
        self.aq = aq
        self.dev = dev
        self.buffers = buffers
        self.fp16 = fp16
        self.steer = synthetic.replay_steer().to(dev)
        self.alpha = torch.full((STEPS,), synthetic.REPLAY_ALPHA, dtype=torch.float32, device=dev)
        self.q8, self.q4, self.w16, self.xq, self.x_host = {}, {}, {}, {}, {}
        kmax = max(k for _, k, _ in LINEARS)
        self.ws = aq.w8a8_workspace(M, kmax, device=dev)   # one workspace: the calls are in stream order
        self.x = [dict() for _ in range(buffers)]
        self.y = {k: {} for k in ("q8", "w8a8", "q4", "f16")}
        for b in range(BLOCKS):
            for name, k, n in LINEARS:
                W = synthetic.replay_weight(b, name).to(dev)
                self.q8[b, name] = aq.qpack("q8", W)
                self.q4[b, name] = aq.qpack("q4", W)
                if fp16:
                    self.w16[b, name] = W                 # the fp16 rung keeps its weights
                del W                                     # the quantised rungs release theirs
                xh = synthetic.replay_activation(b, name).pin_memory()
                self.x_host[b, name] = xh
                for i in range(buffers):
                    self.x[i][b, name] = xh.to(dev)
                self.xq[b, name] = (torch.empty(M, k, dtype=torch.int8, device=dev),
                                    torch.empty(M, dtype=torch.float32, device=dev))
                for prec in self.y:
                    if prec != "f16" or fp16:
                        self.y[prec][b, name] = torch.empty(M, n, dtype=torch.float16, device=dev)
        torch.cuda.synchronize()

    def _steer(self, s, b, name):
        if b == synthetic.REPLAY_STEER_BLOCK and name == "out":
            return dict(steer_vec=self.steer, alpha_dev=self.alpha[s:s + 1])
        return {}

    def final_outputs(self, kinds=("q8", "w8a8", "q4")):
        """The step's results: the last linear's output of each precision."""
        return [self.y[k][BLOCKS - 1, LINEARS[-1][0]] for k in kinds]

    def launch(self, kind, stream, buf=0):
        aq = self.aq
        x = self.x[buf]
        for s in range(STEPS):
            for b in range(BLOCKS):
                for name, k, n in LINEARS:
                    key = (b, name)
                    if kind == "q8":
                        aq.qgemm("q8", x[key], *self.q8[key], out=self.y["q8"][key], stream=stream,
                                 **self._steer(s, b, name))
                    elif kind == "q4":
                        aq.qgemm("q4", x[key], *self.q4[key], out=self.y["q4"][key], stream=stream,
                                 **self._steer(s, b, name))
                    elif kind == "f16":
                        aq.qgemm("f16", x[key], self.w16[key], None, out=self.y["f16"][key],
                                 stream=stream, **self._steer(s, b, name))
                    elif kind == "w8a8_fused":
                        aq.qgemm_w8a8_fused(x[key], *self.q8[key], out=self.y["w8a8"][key],
                                            workspace=self.ws, stream=stream, **self._steer(s, b, name))
                    elif kind == "act_quant":
                        aq.act_quant(x[key], out=self.xq[key], stream=stream)
                    else:
                        xq, sx = self.xq[key]
                        aq.qgemm("w8a8", xq, *self.q8[key], sx=sx, out=self.y["w8a8"][key],
                                 stream=stream, **self._steer(s, b, name))

    def kinds(self):
        return self.ORDER + tuple(k for k in self.EXTRA if k != "f16" or self.fp16)

    def capture(self):
        self.stream = torch.cuda.Stream(self.dev)
        self.copy_stream = torch.cuda.Stream(self.dev)
        self.graphs = {}
        with torch.cuda.stream(self.stream):
            for kind in self.kinds():
                self.launch(kind, self.stream)   # eager once: first-call set-up outside capture
            self.stream.synchronize()
            for kind in self.kinds():
                for buf in range(self.buffers if kind != "w8a8_gemm" else 1):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=self.stream):
                        self.launch(kind, self.stream, buf)
                    self.graphs[kind, buf] = g
        torch.cuda.synchronize()
        self.aq.device_status(self.stream)

    def run_step(self, events=None, buf=0, kinds=None):
        s = self.stream
        kinds = self.ORDER if kinds is None else kinds
        with torch.cuda.stream(s):
            for i, kind in enumerate(kinds):
                if events is not None:
                    events[i].record(s)
                self.graphs[kind, buf if kind != "w8a8_gemm" else 0].replay()
            if events is not None:
                events[-1].record(s)


def _ev():
    return torch.cuda.Event(enable_timing=True)


def time_steps(rep, steps, ws, kinds=None):
    """Device time of `steps` replays of `kinds`, bracketed by a barrier and a
    synchronize on both sides; returns (total ms, per-kind ms lists)."""
    kinds = Replay.ORDER if kinds is None else kinds
    ev = [[_ev() for _ in range(len(kinds) + 1)] for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize()
    t0, t1 = _ev(), _ev()
    t0.record(rep.stream)
    for s in range(steps):
        rep.run_step(ev[s], kinds=kinds)
    t1.record(rep.stream)
    torch.cuda.synchronize()
    barrier(ws)
    seg = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)) for i in range(len(kinds))]
    return t0.elapsed_time(t1), seg


def e2e_loop(rep, steps, out_host):
    """End to end through host memory: every step copies all of its inputs
    from pinned host memory (on a copy stream, into the input buffer the
    previous step is not using) and reads its results back. Returns ms."""
    cs, xs = rep.stream, rep.copy_stream
    nb = rep.buffers
    copied = [_ev() for _ in range(nb)]
    done = [_ev() for _ in range(nb)]
    start, end = _ev(), _ev()
    start.record(xs)
    for i in range(steps):
        b = i % nb
        with torch.cuda.stream(xs):
            if i >= nb:
                xs.wait_event(done[b])               # step i - nb has finished reading buffer b
            for key, xh in rep.x_host.items():
                rep.x[b][key].copy_(xh, non_blocking=True)
            copied[b].record(xs)
        cs.wait_event(copied[b])
        rep.run_step(buf=b)
        with torch.cuda.stream(cs):
            for o, h in zip(rep.final_outputs(), out_host):
                h.copy_(o, non_blocking=True)
            done[b].record(cs)
    end.record(cs)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def _gpu_bus_id(dev):
    try:
        return torch.cuda.get_device_properties(dev).pci_bus_id
    except Exception:
        try:
            p = torch.cuda.get_device_properties(dev)
            return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        except Exception:
            return None


def run_ours(args, ws, rank):
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    R = roofs(peaks)
    acct = step_account()

    rep = Replay(dev, buffers=2, fp16=not args.no_fp16)
    rep.capture()
    for _ in range(args.warmup):
        rep.run_step()
    torch.cuda.synchronize()

    bus = _gpu_bus_id(dev)
    with ClockSampler(bus if isinstance(bus, str) else None) as clk:
        total_ms, seg_ms = time_steps(rep, args.steps, ws)
    clocks = clk.summary()
    rep.aq.device_status(rep.stream)

    # the steering on/off delta: the same graphs, the device schedule set to 0
    rep.alpha.zero_()
    off_ms, _ = time_steps(rep, args.steps, ws)
    rep.alpha.fill_(synthetic.REPLAY_ALPHA)
    # the W8A8 leg with the activation quantisation fused into the GEMM launch (outside `value`)
    for _ in range(max(1, args.warmup // 2)):
        rep.run_step(kinds=("w8a8_fused",))
    fus_ms, _ = time_steps(rep, args.steps, ws, kinds=("w8a8_fused",))
    # the fp16 rung of the precision ladder, same replay (outside `value`)
    f16_ms = None
    if rep.fp16:
        for _ in range(max(1, args.warmup // 2)):
            rep.run_step(kinds=("f16",))
        f16_ms, _ = time_steps(rep, args.steps, ws, kinds=("f16",))
    rep.aq.device_status(rep.stream)

    # ---- end to end: pinned host inputs -> device, the same graphs, results -> host
    e2e_in = sum(t.numel() * t.element_size() for t in rep.x_host.values())
    out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in rep.final_outputs()]
    e2e_out = sum(o.numel() * o.element_size() for o in out_host)
    e2e_loop(rep, max(2, args.warmup), out_host)
    barrier(ws)
    e2e_ms = e2e_loop(rep, args.steps, out_host)
    barrier(ws)
    rep.aq.device_status(rep.stream)

    vals = max_over_ranks([total_ms, e2e_ms, off_ms, f16_ms or 0.0, fus_ms, *seg_ms], ws)
    total_ms, e2e_ms, off_ms, f16_ms_max, fus_ms, *seg_ms = vals
    if f16_ms is not None:
        f16_ms = f16_ms_max

    ops_step = acct["q8"][0] + acct["q4"][0] + acct["w8a8_gemm"][0]
    ms_per_step = total_ms / args.steps
    value = ops_step * ws / (ms_per_step * 1e-3) / 1e12
    hbm = R["hbm"]
    kinds = {"q8": (0, R["f16"]), "act_quant": (1, None), "w8a8_gemm": (2, R["i8"]), "q4": (3, R["f16"])}
    launches = STEPS * BLOCKS * len(LINEARS)
    per = {}
    for kind, (i, peak) in kinds.items():
        t = seg_ms[i] / args.steps * 1e-3
        ops, byts = acct[kind]
        d = roof_entry(ops, byts, t, peak or 1.0, hbm)
        d.update(ms_per_step=seg_ms[i] / args.steps, launches_per_step=launches,
                 avg_launch_us=t / launches * 1e6)
        per[kind] = d
    fused = roof_entry(acct["w8a8"][0], acct["w8a8"][1], fus_ms / args.steps * 1e-3, R["i8"], hbm)
    fused.update(ms_per_step=fus_ms / args.steps, launches_per_step=launches,
                 avg_launch_us=fus_ms / args.steps * 1e-3 / launches * 1e6,
                 note="the same W8A8 leg with the activation quantisation inside the GEMM launch "
                      "(aria_qgemm_w8a8_fused, 768 launches per step instead of 1536); algorithmic "
                      "bytes: fp16 X, packed weights and scales, fp16 Y; timed after the step, not in value")
    t_w = (seg_ms[1] + seg_ms[2]) / args.steps
    per_precision = {
        "q8": per["q8"], "q4": per["q4"],
        "w8a8": {"ms_per_step": t_w, "tops": acct["w8a8_gemm"][0] / (t_w * 1e-3) / 1e12,
                 "gemm": per["w8a8_gemm"], "act_quant": per["act_quant"], "fused": fused},
    }
    if f16_ms is not None:
        t = f16_ms / args.steps * 1e-3
        d = roof_entry(acct["f16"][0], acct["f16"][1], t, R["f16"], hbm)
        d.update(ms_per_step=f16_ms / args.steps, launches_per_step=launches,
                 avg_launch_us=t / launches * 1e6,
                 note="the unquantised fp16 rung (\"Results\" table), timed after the step, not in value")
        per_precision["f16"] = d
    dom = max(kinds, key=lambda k: seg_ms[kinds[k][0]])
    dd = per[dom]
    ops_l = acct[dom][0] / launches            # algorithmic work per launch (mean of 4 shapes)
    byt_l = acct[dom][1] / launches
    t_l = dd["avg_launch_us"] * 1e-6
    if dd["bound"] == "tensor":
        roof = {"bound": "tensor", "achieved": ops_l / t_l / 1e12, "peak": kinds[dom][1],
                "unit": "TFLOP/s" if dom != "w8a8_gemm" else "TOPS"}
    else:
        roof = {"bound": "hbm", "achieved": byt_l / t_l / 1e9, "peak": hbm, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = {"q8": "qgemm_kernel<Q8>", "q4": "qgemm_kernel<Q4>", "w8a8_gemm": "qgemm_kernel<W8A8>",
                      "act_quant": "row_quant_i8_kernel"}[dom]
    roof["traffic"], roof["traffic_source"] = measured_traffic(roof["kernel"], acct[dom][1] / launches)
    roof["peak_source"] = (f"{peak_src} MEASURED_PEAKS.json "
                           + ("bf16_tflops (burst: the kernel runs inside a ~30 ms step at full clocks)"
                              if roof["bound"] == "tensor" else "hbm_gbs")
                           + (" x 2 (nominal int8:fp16)" if dom == "w8a8_gemm" else ""))
    if roof["bound"] == "tensor":
        roof["frac_of_sustained"] = roof["achieved"] / (
            peaks["bf16_tflops_sustained"] * (INT8_OVER_F16 if dom == "w8a8_gemm" else 1.0))
    roof["per_launch"] = {"ops": ops_l, "bytes": byt_l, "avg_us": t_l * 1e6}

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16+i8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": M, "blocks": BLOCKS, "denoise_steps": STEPS,
                   "graphs": "one CUDA graph per precision holding the 8-step loop; the steered "
                             "launch of step s reads alpha from a device schedule",
                   "l2": "inputs larger than L2: 680 MB q8 / 382 MB q4 weights and 221 MB of "
                         "activations cycle through each step",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "per_precision": per_precision,
        "steer_delta": {"steered_ms_per_step": ms_per_step, "unsteered_ms_per_step": off_ms / args.steps,
                        "delta_ms_per_step": ms_per_step - off_ms / args.steps,
                        "note": "the same captured graphs; the device alpha schedule set to 0 "
                                "(the add is skipped) vs 0.3 on block 12's out-projection"},
        "roofline": roof,
        "gpu_launches": Replay.LAUNCHES_PER_STEP * args.steps,
        "clocks": clocks,
        "e2e": {"value": ops_step * ws / (e2e_ms / args.steps * 1e-3) / 1e12, "unit": "TOPS",
                "h2d_bytes_per_step": e2e_in, "d2h_bytes_per_step": e2e_out,
                "ms_per_step": e2e_ms / args.steps,
                "note": "every step copies all 96 input activations from pinned host memory "
                        "(double-buffered: the next step's copy overlaps this step's compute) and "
                        "reads back each precision's final output; the other outputs are "
                        "intermediates that a transformer consumes on the device"},
    }
    if rank == 0 and not args.no_per_config:
        line["per_config"] = run_cases(CONFIG_CASES, args.reps, R)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(rows=args.cpu_rows)
    return line


# ------------------------------------------------------------- oracle arm --

def _cpu_pipeline(name, k, n, fmt, rows, block):
    """One linear at one precision through the oracle: pack, act quant where
    used, GEMM and epilogue on `rows` token rows. Returns (ops, seconds)."""
    import oracle
    W = synthetic.replay_weight(block, name).numpy()
    X = synthetic.replay_activation(block, name).numpy()
    st = name == "out" and block == synthetic.REPLAY_STEER_BLOCK
    v = synthetic.replay_steer().numpy() if st else None
    a = synthetic.REPLAY_ALPHA if st else 0.0
    r = np.arange(rows)
    t0 = time.perf_counter()
    if fmt == "q4":
        P, S = oracle.pack_q4(W)
        oracle.wo_ref("q4", X[r], P, S, None, v, a)
    else:
        Wq, sw = oracle.pack_q8(W)
        if fmt == "q8":
            oracle.wo_ref("q8", X[r], Wq, sw, None, v, a)
        else:
            oracle.w8a8(X[r], Wq, sw, None, v, a)
    return gemm_ops(rows, n, k), time.perf_counter() - t0


def cpu_threads():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except Exception:
        return max(1, os.cpu_count() or 1)


def cpu_sample(rows_per_gemm=8, linears=LINEARS, block=0, fmts=("q8", "w8a8", "q4"), threads=1):
    """One bounded sample of the workload through the oracle: each precision
    x each linear of one block, the whole pipeline on `rows_per_gemm` token
    rows. The 12 pipelines run on `threads` host threads (the oracle's C
    calls release the interpreter lock). Returns (gemm ops counted like the
    GPU arm, wall seconds, threads used)."""
    jobs = [(name, k, n, fmt) for name, k, n in linears for fmt in fmts]
    threads = max(1, min(threads, len(jobs)))
    t0 = time.perf_counter()
    if threads == 1:
        res = [_cpu_pipeline(*j, rows_per_gemm, block) for j in jobs]
    else:
        with concurrent.futures.ThreadPoolExecutor(threads) as ex:
            res = list(ex.map(lambda j: _cpu_pipeline(*j, rows_per_gemm, block), jobs))
    wall = time.perf_counter() - t0
    return sum(r[0] for r in res), wall, threads


def cpu_baseline(rows=16):
    ops1, t1, _ = cpu_sample(rows_per_gemm=rows, threads=1)
    opsn, tn, nth = cpu_sample(rows_per_gemm=rows, threads=cpu_threads())
    sample = (f"block 0, all 4 linears x (q8, W8A8, q4): pack + quant + GEMM + epilogue on {rows} "
              f"of 432 token rows; plain C oracle, fp64 GEMM; ops counted as 2*rows*N*K per GEMM")
    return {"value": opsn / tn / 1e12, "unit": "TOPS", "cores": nth, "kind": "oracle",
            "seconds": tn, "sample": sample + f"; the 12 pipelines on {nth} host threads",
            "single_thread": {"value": ops1 / t1 / 1e12, "cores": 1, "seconds": t1},
            "host_cores_available": cpu_threads()}


def run_reference(args, ws, rank):
    """The oracle as the reference arm, on this arm's metric and workload."""
    if rank != 0:
        return None
    nth = cpu_threads() if args.ref_threads <= 0 else args.ref_threads
    for _ in range(args.warmup):
        cpu_sample(rows_per_gemm=1, linears=LINEARS[1:2], fmts=("q8",))
    ops, t, used = 0.0, 0.0, 1
    rows = max(1, int(args.ref_rows))
    for s in range(args.steps):
        o, dt, used = cpu_sample(rows_per_gemm=rows, block=s % BLOCKS, threads=nth)
        ops += o
        t += dt
    value = ops / t / 1e12
    sample = (f"each step: one block's 4 linears x (q8, W8A8, q4), pack + quant + GEMM + "
              f"epilogue on {rows} of 432 token rows, plain C oracle on {used} host threads")
    return {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "tokens": M, "blocks": BLOCKS, "denoise_steps": STEPS,
                       "parallelism": "single process (CPU)"},
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": used, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------ per-shape cases -----

def _d(lin):
    return {n: (k, nn) for n, k, nn in lin}


# (configuration, case, linear name, N, K, M); N, K from the configuration's shapes
CONFIG_CASES = (
    [("tiny q8 (256x256, M=64)", "q8", "tiny", 256, 256, 64)]
    + [("q8 d=1024", "q8", name, n, k, m) for m in (1, 16, 432) for name, k, n in synthetic.D1024]
    + [("W8A8 d=1536 act quant", "act_quant", "", 0, k, m) for m in (432, 4096) for k in (1536, 6144)]
    + [("W8A8 d=1536", "w8a8", name, n, k, m) for m in (432, 4096) for name, k, n in synthetic.D1536]
    + [("q4 d=1536", "q4", name, n, k, m) for m in (1, 8, 432) for name, k, n in synthetic.D1536]
    + [("fp16 d=1536 (precision ladder)", "f16", name, n, k, m) for m in (1, 432)
       for name, k, n in synthetic.D1536]
    + [("pack d=1536", "pack_q8", name, n, k, 0) for name, k, n in synthetic.D1536]
    + [("pack d=1536", "pack_q4", name, n, k, 0) for name, k, n in synthetic.D1536]
)

# performance bars of the workload: weight-bound shapes >= 70 % of HBM, W8A8 at
# M = 4096 >= 60 % of the int8 tensor peak
def case_target(case, m):
    if (case == "q8" and m in (1, 16)) or (case == "q4" and m in (1, 8)):
        return ("hbm_frac", 0.70)
    if case == "w8a8" and m == 4096:
        return ("tensor_frac", 0.60)
    return None


def _case_inputs(case, name, n, k, m):
    """Seeded inputs of one case (the configuration's own generators)."""
    if case == "act_quant":
        return None, synthetic.activation(f"w8a8d1536/act/M{m}/K{k}", m, k, outlier_channel_frac=0.01)
    if name == "tiny":
        d = synthetic.tiny_q8()
        return d["W"], d["X"]
    if not name:   # an arbitrary shape (--case): the same distributions, keyed by the shape
        return (synthetic.weight(f"case/{n}x{k}", n, k, outlier_frac=0.001 if case.endswith("q4") else 0.0),
                synthetic.activation(f"case/{max(m, 1)}x{k}", max(m, 1), k,
                                     outlier_channel_frac=0.01 if case == "w8a8" else 0.0))
    if case == "q8":
        return synthetic.q8_block_d1024(name, m)
    if case in ("w8a8", "pack_q8"):
        return synthetic.w8a8_d1536(name, max(m, 1))
    return synthetic.q4_d1536(name, max(m, 1))


def run_case(case, n, k, m, reps=200, name="", R=None, cycle=True):
    """One kernel on one shape, `reps` launches back to back in one CUDA graph
    (each launch in stream order after the previous one, as in a layer
    sequence), cycling through enough copies of what the launch streams --
    packed weights, or the fp16 weights of a pack, or the activations of the
    activation quantiser -- to exceed 3x L2. Returns one result dict."""
    import int8_int4_b200 as aq
    dev = torch.device("cuda", torch.cuda.current_device())
    W, X = _case_inputs(case, name, n, k, m)
    if case == "act_quant":
        per_copy = 3 * m * k
    elif case.startswith("pack"):
        per_copy = 2 * n * k
    else:
        per_copy = {"q8": n * k, "w8a8": n * k, "q4": 0.5625 * n * k, "f16": 2 * n * k}[case]
    copies = max(1, int(np.ceil(3 * 126e6 / per_copy))) if cycle else 1
    Y = torch.empty(max(m, 1), max(n, 1), dtype=torch.float16, device=dev)
    if case == "act_quant":
        Xs = [X.to(dev) for _ in range(copies)]
        outs = (torch.empty(m, k, dtype=torch.int8, device=dev), torch.empty(m, dtype=torch.float32, device=dev))
        launch = lambda i: aq.act_quant(Xs[i % copies], out=outs)
    elif case.startswith("pack"):
        fmt = case[5:]
        Ws = [W.to(dev) for _ in range(copies)]
        packed = aq.qpack(fmt, Ws[0])
        launch = lambda i: aq.qpack(fmt, Ws[i % copies], out=packed)
    else:
        Wd = W.to(dev)
        Xd = X.to(dev)
        if case == "f16":
            packs = [(Wd.clone(), None) for _ in range(copies)]
        else:
            p0 = aq.qpack("q8" if case == "w8a8" else case, Wd)
            packs = [tuple(t.clone() for t in p0) for _ in range(copies)]
        del Wd
        kw = {}
        if case == "w8a8":
            Xd, kw["sx"] = aq.act_quant(Xd)
        fmt = case
        launch = lambda i: aq.qgemm(fmt, Xd, *packs[i % copies], out=Y, **kw)
    for i in range(3):
        launch(i)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(reps):
                launch(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = _ev(), _ev()
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    aq.device_status()
    t = e0.elapsed_time(e1) * 1e-3 / reps
    del g
    if case in ("q8", "q4", "w8a8", "f16"):
        ops = gemm_ops(m, n, k)
        byt = {"q8": lambda: bytes_wo("q8", m, n, k, False), "q4": lambda: bytes_wo("q4", m, n, k, False),
               "w8a8": lambda: bytes_w8a8(m, n, k, False), "f16": lambda: bytes_f16(m, n, k, False)}[case]()
    elif case == "act_quant":
        ops, byt = 0.0, bytes_act_quant(m, k)
    else:
        ops, byt = 0.0, bytes_pack(case[5:], n, k)
    R = R or roofs(load_peaks()[0])
    d = {"case": case, "linear": name, "M": m, "N": n, "K": k, "reps": reps, "copies": copies}
    d.update(roof_entry(ops, byt, t, R["i8"] if case == "w8a8" else R["f16"], R["hbm"]))
    tgt = case_target(case, m)
    if tgt:
        d["target"] = {"of": tgt[0], "frac": tgt[1], "met": d[tgt[0]] >= tgt[1]}
    return d


def run_cases(cases, reps, R):
    out = []
    for label, case, name, n, k, m in cases:
        d = run_case(case, n, k, m, reps=reps, name=name, R=R)
        d["config"] = label
        out.append({kk: (round(v, 4) if isinstance(v, float) else v) for kk, v in d.items()})
        torch.cuda.empty_cache()
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--no-fp16", action="store_true", help="skip the fp16 rung of the replay")
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--ref-threads", type=int, default=0, help="reference arm threads (0: all host cores)")
    ap.add_argument("--case", choices=["q8", "q4", "w8a8", "f16", "act_quant", "pack_q8", "pack_q4"],
                    help="time one kernel on one shape instead of the workload (no bench line)")
    ap.add_argument("--shape", default="1536x1536", help="NxK of the weight for --case (K for act_quant)")
    ap.add_argument("--m", type=int, default=432, help="tokens for --case")
    ap.add_argument("--reps", type=int, default=200)
    ap.add_argument("--sweep", action="store_true", help="time every per-shape case (JSON lines)")
    ap.add_argument("--no-cycle", dest="cycle", action="store_false",
                    help="reuse one copy (L2-resident) for --case")
    args = ap.parse_args(argv)
    if args.case:
        dims = [int(v) for v in args.shape.split("x")]
        n, k = (0, dims[-1]) if args.case == "act_quant" else (dims[0], dims[1])
        print(json.dumps(run_case(args.case, n, k, args.m, reps=args.reps, cycle=args.cycle)), flush=True)
        return
    if args.sweep:
        R = roofs(load_peaks()[0])
        for c in CONFIG_CASES:
            print(json.dumps(run_cases([c], args.reps, R)[0]), flush=True)
        return
    ws, rank, _ = dist_init()
    try:
        line = run_reference(args, ws, rank) if args.impl == "reference" else run_ours(args, ws, rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
