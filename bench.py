#!/usr/bin/env python
"""bench.py -- quantized GEMM TOPS and HBM GB/s per precision (q8 / W8A8 / q4)
on B200, with the fraction of roofline of the dominant kernel.

Workload (one "step"): the layer-sequence replay of a synthetic diffusion
transformer -- 24 blocks x {qkv 1536->4608, out 1536->1536, up 1536->6144,
down 6144->1536} at M = 432 tokens (2 CFG halves x 216 latent frames), 8
denoising steps, at each of the three precisions, with the steering add
(alpha = 0.3, unit-norm v) on block 12's out-projection. This is the shape of
the pages' generation loop ("Results": 8 steps; "What aria is": the
denoising loop replayed as one CUDA graph); weights are packed once at load,
as on the pages, and the pack kernels are timed separately. Per precision
one CUDA graph holds the 8-step loop (768 GEMM launches; W8A8 adds 768
per-token activation quantisations in a graph of their own).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (one process per GPU, launched by torchrun),
no collective on the data path; the timed region is bracketed by barriers
and the slowest rank's device time is reported. Rank 0 prints ONE JSON line.
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


def bytes_act_quant(m, k):
    return 3 * m * k + 4 * m


def step_account():
    """ops and algorithmic bytes of one 8-step replay, per precision / kernel"""
    acc = {"q8": [0.0, 0.0], "w8a8_gemm": [0.0, 0.0], "act_quant": [0.0, 0.0], "q4": [0.0, 0.0]}
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
    return {k: (v[0] * STEPS, v[1] * STEPS) for k, v in acc.items()}


# ------------------------------------------------------------- our arm ------

class Replay:
    """Device-resident workload and its CUDA graphs."""

    def __init__(self, dev):
        import int8_int4_b200 as aq
        self.aq = aq
        self.dev = dev
        self.steer = synthetic.replay_steer().to(dev)
        self.q8, self.q4, self.x, self.xq, self.y = {}, {}, {}, {}, {}
        self.x_host = {}
        for b in range(BLOCKS):
            for name, k, n in LINEARS:
                W = synthetic.replay_weight(b, name).to(dev)
                self.q8[b, name] = aq.qpack("q8", W)
                self.q4[b, name] = aq.qpack("q4", W)
                del W                                   # the fp16 copy is released once packed
                xh = synthetic.replay_activation(b, name).pin_memory()
                self.x_host[b, name] = xh
                self.x[b, name] = xh.to(dev)
                self.xq[b, name] = (torch.empty(M, k, dtype=torch.int8, device=dev),
                                    torch.empty(M, dtype=torch.float32, device=dev))
                self.y[b, name] = torch.empty(M, n, dtype=torch.float16, device=dev)
        torch.cuda.synchronize()

    def _steer(self, b, name):
        if b == synthetic.REPLAY_STEER_BLOCK and name == "out":
            return dict(steer_vec=self.steer, alpha=synthetic.REPLAY_ALPHA)
        return {}

    def launch(self, kind, stream):
        aq = self.aq
        for _ in range(STEPS):
            for b in range(BLOCKS):
                for name, k, n in LINEARS:
                    key = (b, name)
                    if kind == "q8":
                        aq.qgemm("q8", self.x[key], *self.q8[key], out=self.y[key], stream=stream,
                                 **self._steer(b, name))
                    elif kind == "q4":
                        aq.qgemm("q4", self.x[key], *self.q4[key], out=self.y[key], stream=stream,
                                 **self._steer(b, name))
                    elif kind == "act_quant":
                        aq.act_quant(self.x[key], out=self.xq[key], stream=stream)
                    else:
                        xq, sx = self.xq[key]
                        aq.qgemm("w8a8", xq, *self.q8[key], sx=sx, out=self.y[key], stream=stream,
                                 **self._steer(b, name))

    def capture(self):
        self.stream = torch.cuda.Stream(self.dev)
        self.graphs = {}
        with torch.cuda.stream(self.stream):
            for kind in ("q8", "act_quant", "w8a8_gemm", "q4"):
                self.launch(kind, self.stream)   # eager once: first-call set-up outside capture
            self.stream.synchronize()
            for kind in ("q8", "act_quant", "w8a8_gemm", "q4"):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=self.stream):
                    self.launch(kind, self.stream)
                self.graphs[kind] = g
        torch.cuda.synchronize()
        self.aq.device_status(self.stream)

    ORDER = ("q8", "act_quant", "w8a8_gemm", "q4")
    LAUNCHES_PER_STEP = 4 * STEPS * BLOCKS * len(LINEARS)

    def run_step(self, events=None):
        s = self.stream
        with torch.cuda.stream(s):
            for i, kind in enumerate(self.ORDER):
                if events is not None:
                    events[i].record(s)
                self.graphs[kind].replay()
            if events is not None:
                events[-1].record(s)


def time_pack(dev, reps=3):
    """pack kernels on block 0's four d=1536 weights, each timed alone after an
    L2 flush; returns algorithmic GB/s per format"""
    import int8_int4_b200 as aq
    Ws = [synthetic.replay_weight(0, name).to(dev) for name, _, _ in LINEARS]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    res = {}
    for fmt in ("q8", "q4"):
        tot_t, tot_b = 0.0, 0.0
        for r in range(reps + 1):
            for W in Ws:
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                aq.qpack(fmt, W)
                e1.record()
                e1.synchronize()
                if r:                                  # first round is a warm-up
                    n, k = W.shape
                    tot_t += e0.elapsed_time(e1) * 1e-3
                    tot_b += 2 * n * k + (n * k + 4 * n if fmt == "q8" else n * k // 2 + 2 * n * (k // 32))
        res[fmt] = {"gbs": tot_b / tot_t / 1e9, "launches": 4 * reps}
    del Ws, flush
    return res


def run_ours(args, ws, rank):
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    acct = step_account()

    rep = Replay(dev)
    rep.capture()
    for _ in range(args.warmup):
        rep.run_step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    bus = None
    try:
        bus = torch.cuda.get_device_properties(dev).pci_bus_id
    except Exception:
        try:
            p = torch.cuda.get_device_properties(dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        except Exception:
            bus = None
    with ClockSampler(bus if isinstance(bus, str) else None) as clk:
        barrier(ws)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(rep.stream)
        for s in range(args.steps):
            rep.run_step(ev[s])
        t1.record(rep.stream)
        torch.cuda.synchronize()
        barrier(ws)
    clocks = clk.summary()
    total_ms = t0.elapsed_time(t1)
    seg_ms = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps)) for i in range(4)]
    rep.aq.device_status(rep.stream)

    # ---- end to end: pinned host inputs -> device, the same graphs, result -> host
    e2e_in = sum(t.numel() * t.element_size() for t in rep.x_host.values())
    outs = [rep.y[BLOCKS - 1, "down"]]
    out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    e2e_out = sum(o.numel() * o.element_size() for o in outs)
    for _ in range(max(1, args.warmup // 2)):
        _e2e_step(rep, out_host)
    torch.cuda.synchronize()
    barrier(ws)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(rep.stream)
    for _ in range(args.steps):
        _e2e_step(rep, out_host)
    a1.record(rep.stream)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = a0.elapsed_time(a1)

    total_ms, e2e_ms, *seg_ms = max_over_ranks([total_ms, e2e_ms, *seg_ms], ws)
    pack = time_pack(dev) if rank == 0 else None

    ops_step = acct["q8"][0] + acct["q4"][0] + acct["w8a8_gemm"][0]
    ms_per_step = total_ms / args.steps
    value = ops_step * ws / (ms_per_step * 1e-3) / 1e12
    f16_peak = peaks["bf16_tflops_sustained"]
    i8_peak = f16_peak * INT8_OVER_F16
    hbm = peaks["hbm_gbs"]
    kinds = {"q8": (0, f16_peak), "act_quant": (1, None), "w8a8_gemm": (2, i8_peak), "q4": (3, f16_peak)}
    per = {}
    launches = STEPS * BLOCKS * len(LINEARS)
    for kind, (i, peak) in kinds.items():
        t = seg_ms[i] / args.steps * 1e-3
        ops, byts = acct[kind]
        d = {"ms_per_step": seg_ms[i] / args.steps, "launches_per_step": launches,
             "avg_launch_us": t / launches * 1e6, "hbm_gbs": byts / t / 1e9,
             "hbm_frac": byts / t / 1e9 / hbm}
        if ops:
            d["tops"] = ops / t / 1e12
            d["tensor_frac"] = d["tops"] / peak
            # which roof binds at this shape: ideal time against each peak
            d["bound"] = "tensor" if ops / (peak * 1e12) >= byts / (hbm * 1e9) else "hbm"
        else:
            d["bound"] = "hbm"
        per[kind] = d
    per_precision = {
        "q8": per["q8"], "q4": per["q4"],
        "w8a8": {"ms_per_step": per["act_quant"]["ms_per_step"] + per["w8a8_gemm"]["ms_per_step"],
                 "tops": acct["w8a8_gemm"][0] / ((seg_ms[1] + seg_ms[2]) / args.steps * 1e-3) / 1e12,
                 "gemm": per["w8a8_gemm"], "act_quant": per["act_quant"]},
    }
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
                           + ("bf16_tflops_sustained" if roof["bound"] == "tensor" else "hbm_gbs")
                           + (" x 2 (nominal int8:fp16)" if dom == "w8a8_gemm" else ""))
    roof["per_launch"] = {"ops": ops_l, "bytes": byt_l, "avg_us": t_l * 1e6}

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16+i8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": M, "blocks": BLOCKS, "denoise_steps": STEPS,
                   "graphs": "one CUDA graph per precision holding the 8-step loop",
                   "l2": "inputs larger than L2: 680 MB q8 / 382 MB q4 weights and 221 MB of "
                         "activations cycle through each step",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "per_precision": per_precision,
        "pack_gbs": pack,
        "roofline": roof,
        "gpu_launches": Replay.LAUNCHES_PER_STEP * args.steps,
        "clocks": clocks,
        "e2e": {"value": ops_step * ws / (e2e_ms / args.steps * 1e-3) / 1e12, "unit": "TOPS",
                "h2d_bytes_per_step": e2e_in, "d2h_bytes_per_step": e2e_out,
                "ms_per_step": e2e_ms / args.steps},
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(rows=args.cpu_rows)
    return line


def _e2e_step(rep, out_host):
    s = rep.stream
    with torch.cuda.stream(s):
        for key, xh in rep.x_host.items():
            rep.x[key].copy_(xh, non_blocking=True)
    rep.run_step()
    with torch.cuda.stream(s):
        for o, h in zip([rep.y[BLOCKS - 1, "down"]], out_host):
            h.copy_(o, non_blocking=True)


# ------------------------------------------------------------- oracle arm --

def cpu_sample(rows_per_gemm=8, linears=LINEARS, block=0, fmts=("q8", "w8a8", "q4")):
    """One bounded sample of the workload through the oracle: for each
    precision and each linear of one block, the whole pipeline (pack, act
    quant where used, GEMM, epilogue) on `rows_per_gemm` token rows.
    Returns (gemm ops counted like the GPU arm, seconds)."""
    import oracle
    ops, t = 0.0, 0.0
    rows = np.arange(rows_per_gemm)
    for name, k, n in linears:
        W = synthetic.replay_weight(block, name).numpy()
        X = synthetic.replay_activation(block, name).numpy()
        st = name == "out" and block == synthetic.REPLAY_STEER_BLOCK
        v = synthetic.replay_steer().numpy() if st else None
        a = synthetic.REPLAY_ALPHA if st else 0.0
        for fmt in fmts:
            t0 = time.perf_counter()
            if fmt == "q4":
                P, S = oracle.pack_q4(W)
                oracle.wo_ref("q4", X[rows], P, S, None, v, a)
            else:
                Wq, sw = oracle.pack_q8(W)
                if fmt == "q8":
                    oracle.wo_ref("q8", X[rows], Wq, sw, None, v, a)
                else:
                    oracle.w8a8(X[rows], Wq, sw, None, v, a)
            t += time.perf_counter() - t0
            ops += gemm_ops(rows_per_gemm, n, k)
    return ops, t


def cpu_baseline(rows=16):
    ops, t = cpu_sample(rows_per_gemm=rows)
    return {"value": ops / t / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle",
            "seconds": t,
            "sample": f"block 0, all 4 linears x (q8, W8A8, q4): pack + quant + GEMM + epilogue "
                      f"on {rows} of 432 token rows; single-threaded plain C, fp64 GEMM; "
                      f"ops counted as 2*rows*N*K per GEMM"}


def run_reference(args, ws, rank):
    """The oracle as the reference arm, on this arm's metric and workload."""
    if rank != 0:
        return None
    for _ in range(args.warmup):
        cpu_sample(rows_per_gemm=1, linears=LINEARS[1:2])
    ops, t = 0.0, 0.0
    rows = max(1, int(args.ref_rows))
    for s in range(args.steps):
        o, dt = cpu_sample(rows_per_gemm=rows, block=s % BLOCKS)
        ops += o
        t += dt
    value = ops / t / 1e12
    sample = (f"each step: one block's 4 linears x (q8, W8A8, q4), pack + quant + GEMM + "
              f"epilogue on {rows} of 432 token rows, single-threaded plain C oracle")
    return {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "tokens": M, "blocks": BLOCKS, "denoise_steps": STEPS,
                       "parallelism": "single process (CPU)"},
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------- single-kernel case --

SWEEP = ([("q8", n, k, m) for m in (1, 16, 432) for _, k, n in synthetic.D1024]
         + [("w8a8", n, k, m) for m in (432, 4096) for _, k, n in synthetic.D1536]
         + [("act_quant", 1536, k, m) for m in (432, 4096) for k in (1536, 6144)]
         + [("q4", n, k, m) for m in (1, 8, 432) for _, k, n in synthetic.D1536]
         + [("pack_q8", n, k, 1) for _, k, n in synthetic.D1536]
         + [("pack_q4", n, k, 1) for _, k, n in synthetic.D1536])


def run_sweep(args):
    """Every per-shape case of the q8 (d=1024), W8A8 (d=1536) and q4 (d=1536)
    workloads, one JSON line each, in one process."""
    for case, n, k, m in SWEEP:
        a = argparse.Namespace(**vars(args))
        a.case, a.shape, a.m = case, f"{n}x{k}", m
        run_case(a)
        torch.cuda.empty_cache()


def run_case(args):
    """One kernel on one shape, launched `reps` times back to back, cycling
    through enough weight copies to exceed L2 (for ncu captures and per-shape
    sweeps). Prints one JSON line with the mean launch time."""
    import int8_int4_b200 as aq
    dev = torch.device("cuda", torch.cuda.current_device())
    n, k = (int(v) for v in args.shape.split("x"))
    m = args.m
    W = synthetic.weight(f"case/{n}x{k}", n, k).to(dev)
    X = synthetic.activation(f"case/{m}x{k}", m, k).to(dev)
    fmt = {"w8a8": "q8", "pack_q8": "q8", "pack_q4": "q4"}.get(args.case, args.case)
    per_copy = n * k * (2 if args.case.startswith("pack") else (0.5625 if fmt == "q4" else 1))
    copies = max(1, int(np.ceil(3 * 126e6 / per_copy))) if args.cycle else 1
    packs = [aq.qpack(fmt, W) for _ in range(1 if args.case.startswith("pack") else copies)]
    Ws = [W] + [W.clone() for _ in range(copies - 1)] if args.case.startswith("pack") else None
    Xq = aq.act_quant(X) if args.case == "w8a8" else None
    Y = torch.empty(m, n, dtype=torch.float16, device=dev)

    def launch(i):
        if args.case == "act_quant":
            aq.act_quant(X)
        elif args.case.startswith("pack"):
            aq.qpack(fmt, Ws[i % len(Ws)])
        elif args.case == "w8a8":
            aq.qgemm("w8a8", Xq[0], *packs[i % copies], sx=Xq[1], out=Y)
        else:
            aq.qgemm(fmt, X, *packs[i % copies], out=Y)

    for i in range(3):
        launch(i)
    torch.cuda.synchronize()
    # the reps launches are captured in one CUDA graph, so host launch cost
    # does not enter the per-kernel time
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(args.reps):
                launch(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    aq.device_status()
    us = e0.elapsed_time(e1) * 1e3 / args.reps
    ops = gemm_ops(m, n, k) if args.case in ("q8", "q4", "w8a8") else 0.0
    if args.case in ("q8", "q4"):
        byt = bytes_wo(fmt, m, n, k, False)
    elif args.case == "w8a8":
        byt = bytes_w8a8(m, n, k, False)
    elif args.case == "act_quant":
        byt = bytes_act_quant(m, k)
    else:
        byt = 2 * n * k + (n * k + 4 * n if fmt == "q8" else n * k // 2 + 2 * n * (k // 32))
    print(json.dumps({"case": args.case, "M": m, "N": n, "K": k, "reps": args.reps,
                      "weight_copies": copies, "avg_us": us, "tops": ops / us / 1e6,
                      "gbs": byt / us / 1e3}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--case", choices=["q8", "q4", "w8a8", "act_quant", "pack_q8", "pack_q4"],
                    help="time one kernel on one shape instead of the workload (no JSON bench line)")
    ap.add_argument("--shape", default="1536x1536", help="NxK of the weight for --case")
    ap.add_argument("--m", type=int, default=432, help="tokens for --case")
    ap.add_argument("--reps", type=int, default=200)
    ap.add_argument("--sweep", action="store_true", help="time every per-shape case (JSON lines)")
    ap.add_argument("--no-cycle", dest="cycle", action="store_false",
                    help="reuse one weight copy (L2-resident) for --case")
    args = ap.parse_args(argv)
    if args.case:
        run_case(args)
        return
    if args.sweep:
        run_sweep(args)
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
