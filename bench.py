#!/usr/bin/env python
"""Benchmark: mLSTM forward throughput on B200, one JSON line on stdout.

Workload: the 7B-like layer (B=8, H=8, T=4096, d_qk=256, d_v=512, bf16 q/k/v,
fp32 gates, zero initial state, fp32 h~ and final state), synthetic seeded
inputs.  One step = one xlstm_mlstm_fwd_chunkwise call over the whole batch.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

value      tokens/s (B*T positions per step) with inputs resident in HBM,
           timed with CUDA events on the launch stream, max over ranks;
e2e        the same call fed from pinned host buffers, H2D of the inputs and
           D2H of h~ and the final state inside the timed region;
roofline   algorithmic bytes per launch / launch time against the measured
           HBM copy bandwidth (the kernel is HBM-bound: 136 flop/B < ridge);
cpu_baseline  the float64 oracle on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank runs its own replica (heads are independent,
so the work shards with no collective on the data path): weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "layer_7b"
METRIC = "mLSTM fwd tokens/s & TFLOP/s on 1 B200; % of tensor/HBM roofline"
UNIT = "tokens/s"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def algorithmic(w, L=64):
    """Bytes and flops one forward moves/does (counting convention of the design notes)."""
    N = w.B * w.H * w.T
    e = 2 if w.dtype == "bf16" else 4
    bytes_ = N * ((2 * w.d_qk + w.d_v) * e + 8 + 4 * w.d_v) + w.B * w.H * (w.d_qk * w.d_v + w.d_qk + 1) * 4
    if w.state != "zero":
        bytes_ += w.B * w.H * (w.d_qk * w.d_v + w.d_qk + 1) * 4
    flops = N * (4 * w.d_qk * w.d_v + L * (w.d_qk + w.d_v))
    return bytes_, flops


class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def traffic_for(kernel_src_sha: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    if d.get("source_sha") != kernel_src_sha or d.get("workload") != WORKLOAD:
        return None
    return d.get("traffic_bytes_per_launch")


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "xlstm_mlstm_matrix_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def cpu_baseline(inp, budget_s=12.0):
    """Time the float64 oracle on a bounded sample: whole sequences of a few
    heads, all host threads.  Returns tokens/s in the workload's units."""
    import oracle
    w = inp["workload"]
    threads = oracle.default_threads()
    sel = lambda x, hs: None if x is None else x.reshape((w.B * w.H,) + x.shape[2:])[hs][None]
    # probe with a short prefix of one head to size the sample
    Tp = min(w.T, 256)
    t0 = time.perf_counter()
    oracle.forward(*(sel(inp[n], [0])[:, :, :Tp] for n in ("q", "k", "v", "i_pre", "f_pre")),
                   qk_scale=inp["qk_scale"], threads=1)
    per_head_token = (time.perf_counter() - t0) / Tp
    nheads = int(max(1, min(w.B * w.H, threads * budget_s / max(per_head_token * w.T, 1e-9))))
    nheads = max(1, min(nheads, threads * 2, w.B * w.H))
    hs = list(range(nheads))
    t0 = time.perf_counter()
    oracle.forward(*(sel(inp[n], hs) for n in ("q", "k", "v", "i_pre", "f_pre")),
                   qk_scale=inp["qk_scale"], threads=threads)
    dt = time.perf_counter() - t0
    tokens = nheads * w.T / w.H          # head-tokens / heads per token
    return {"value": tokens / dt, "unit": UNIT, "cores": min(threads, nheads), "kind": "oracle",
            "sample": f"{nheads} of {w.B * w.H} (batch, head) pairs, full T={w.T}, float64, "
                      f"{min(threads, nheads)} threads; tokens = head-tokens / H",
            "seconds": dt}


def run_reference(args, rank, world):
    """--impl reference: the float64 oracle on host cores, same metric/workload."""
    from xlstm_mlstm_matrix_b200 import inputs
    if rank != 0:
        return
    w = inputs.WORKLOADS[WORKLOAD]
    inp = inputs.make_sequence(w)
    # each step is a bounded sample so that the whole run stays within minutes
    budget = max(2.0, min(args.ref_budget, 150.0 / max(1, args.steps)))
    vals = []
    cb = None
    for _ in range(max(1, args.steps)):
        cb = cpu_baseline(inp, budget_s=budget)
        vals.append(cb["value"])
    value = statistics.median(vals)
    cb["value"] = value
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * w.tokens / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "T": w.T, "d_qk": w.d_qk, "d_v": w.d_v},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    from xlstm_mlstm_matrix_b200 import capi, inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    capi.load()
    w = inputs.WORKLOADS[WORKLOAD].replace(seed=inputs.WORKLOADS[WORKLOAD].seed + 1000 * rank)
    if args.B or args.H:   # smaller batch/head count of the same layer (profiling captures)
        w = w.replace(B=args.B or w.B, H=args.H or w.H)
    inp = inputs.make_sequence(w)
    scale = inp["qk_scale"]
    desc = capi.make_desc(w.B, w.H, w.T, w.d_qk, w.d_v, capi.XLSTM_BF16, scale, 64)

    def dev_t(x, bf16):
        t = torch.from_numpy(x).to(dev)
        return t.to(torch.bfloat16) if bf16 else t

    q, k, v = (dev_t(inp[n], True) for n in ("q", "k", "v"))
    ig, fg = dev_t(inp["i_pre"], False), dev_t(inp["f_pre"], False)
    h = torch.empty(w.B, w.H, w.T, w.d_v, device=dev)
    C1 = torch.empty(w.B, w.H, w.d_v, w.d_qk, device=dev)
    n1 = torch.empty(w.B, w.H, w.d_qk, device=dev)
    m1 = torch.empty(w.B, w.H, device=dev)
    wsb = capi.xlstm_mlstm_workspace_size(desc)
    ws = torch.zeros(wsb, device=dev, dtype=torch.uint8)
    stream = torch.cuda.Stream(dev)
    fn = capi.load().xlstm_mlstm_fwd_chunkwise
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    argv = (ctypes.byref(desc), P(q), P(k), P(v), P(ig), P(fg), None, None, None, P(h), P(C1),
            P(n1), P(m1), P(ws), wsb, ctypes.c_void_p(stream.cuda_stream))

    def step():
        st = fn(*argv)
        if st != 0:
            raise capi.XlstmError(st, "xlstm_mlstm_fwd_chunkwise")

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        if dist is None:
            return x
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    # device status after warm-up: no bounded wait gave up
    st, where = capi.xlstm_mlstm_workspace_status(ws, stream)
    if st != 0:
        raise capi.XlstmError(st, f"device status (where={where})")

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank if os.environ.get("CUDA_VISIBLE_DEVICES") is None else 0) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize(dev)
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms)
    st, where = capi.xlstm_mlstm_workspace_status(ws, stream)
    if st != 0:
        raise capi.XlstmError(st, f"device status (where={where})")

    tokens = w.B * w.T
    value = world * tokens / (ms * 1e-3)
    bytes_, flops = algorithmic(w)
    hbm, bf16_peak, _, peak_src = peaks()
    achieved_gbs = bytes_ / (ms * 1e-3) / 1e9
    src_sha = kernel_source_sha()

    # ---- end to end: pinned host buffers through the same call ---------------------
    hq, hk, hv = (torch.from_numpy(inp[n]).to(torch.bfloat16).pin_memory() for n in ("q", "k", "v"))
    hig, hfg = torch.from_numpy(inp["i_pre"]).pin_memory(), torch.from_numpy(inp["f_pre"]).pin_memory()
    oh = torch.empty(h.shape, dtype=torch.float32).pin_memory()
    oC = torch.empty(C1.shape, dtype=torch.float32).pin_memory()
    on = torch.empty(n1.shape, dtype=torch.float32).pin_memory()
    om = torch.empty(m1.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hig, hfg))
    d2h = sum(t.numel() * t.element_size() for t in (oh, oC, on, om))

    def e2e_step():
        for dst, src in ((q, hq), (k, hk), (v, hv), (ig, hig), (fg, hfg)):
            dst.copy_(src, non_blocking=True)
        step()
        for dst, src in ((oh, h), (oC, C1), (on, n1), (om, m1)):
            dst.copy_(src, non_blocking=True)

    e2e_steps = 0 if args.no_e2e else max(1, min(args.steps, 5))
    if e2e_steps:
        with torch.cuda.stream(stream):
            e2e_step()
            stream.synchronize()
            barrier()
            e0.record(stream)
            for _ in range(e2e_steps):
                e2e_step()
            e1.record(stream)
            e1.synchronize()
        barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps) if e2e_steps else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "T": w.T, "d_qk": w.d_qk,
                       "d_v": w.d_v, "chunk": 64, "inputs": "bf16 q/k/v, fp32 gates; fp32 h and state",
                       "l2": "inputs larger than L2 (1.1 GB per step vs 126 MB L2)",
                       "parallelism": f"replicas x{world} (independent heads)"},
            "tflops": world * flops / (ms * 1e-3) / 1e12,
            "hbm_gbs": achieved_gbs,
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": achieved_gbs / hbm, "traffic": traffic_for(src_sha),
                         "peak_source": peak_src,
                         "algorithmic_bytes_per_launch": bytes_, "flops_per_launch": flops,
                         "tensor_frac": flops / (ms * 1e-3) / 1e12 / bf16_peak},
            "gpu_launches": args.steps,
            "e2e": None if e2e_ms is None else {
                "value": world * tokens / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "clocks": clk.summary(),
            "kernel_source_sha": src_sha,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(inp, budget_s=args.ref_budget)
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ref-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--B", type=int, default=0, help="override the batch size (profiling)")
    ap.add_argument("--H", type=int, default=0, help="override the head count (profiling)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    pg = False
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        pg = True
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
