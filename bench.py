#!/usr/bin/env python
"""Benchmark: mLSTM forward throughput on B200, one JSON line on stdout.

Workload: the 7B-like layer (B=8, H=8, T=4096, d_qk=256, d_v=512, bf16 q/k/v,
fp32 gates, zero initial state, fp32 h~ and final state), synthetic seeded
inputs.  One step = one xlstm_mlstm_fwd_chunkwise call over the whole batch.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload layer_7b|long_context|many_short|decode]

The default workload is the 7B-like layer.  --workload picks another of the
synthetic workloads: a sequence workload runs one chunkwise call per step; the
decode workload (B=128, H=8, d_qk=256, d_v=512, state resident in HBM) runs one
xlstm_mlstm_step call per step and counts B tokens per step.

value      tokens/s (B*T positions per step) with inputs resident in HBM,
           timed with CUDA events on the launch stream, max over ranks;
e2e        the same call fed from pinned host buffers, H2D of the inputs and
           D2H of h~ and the final state inside the timed region, every step;
           two steps in flight (copy-in, call and copy-out on three streams,
           two sets of device buffers), as a serving loop runs it;
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

DEFAULT_WORKLOAD = "layer_7b"
METRIC = "mLSTM fwd tokens/s & TFLOP/s on 1 B200; % of tensor/HBM roofline"
UNIT = "tokens/s"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def algorithmic(w, L=64, gated=False):
    """Bytes and flops of one step (counting convention of the design notes).

    Sequence workloads: one forward over B*H*T head-tokens; inputs, h~ and the
    final state (plus the initial state when one is read).  Decode: one step
    over B*H heads; the state is read and written once, plus the step's vectors.
    gated: the fused output stage, bf16 o~ read and bf16 h written instead of
    fp32 h~.
    """
    e = 2 if w.dtype == "bf16" else 4
    state = w.d_qk * w.d_v + w.d_qk + 1
    if w.steps:
        BH = w.B * w.H
        bytes_ = BH * ((2 * w.d_qk + w.d_v) * e + 8 + 4 * w.d_v + 2 * 4 * state)
        flops = BH * (5 * w.d_qk * w.d_v + 4 * w.d_qk)
        return bytes_, flops
    N = w.B * w.H * w.T
    out_bytes = (2 + 2) * w.d_v if gated else 4 * w.d_v
    bytes_ = N * ((2 * w.d_qk + w.d_v) * e + 8 + out_bytes) + w.B * w.H * state * 4
    if w.state != "zero":
        bytes_ += w.B * w.H * state * 4
    flops = N * (4 * w.d_qk * w.d_v + L * (w.d_qk + w.d_v))
    return bytes_, flops


class ClockSampler:
    """nvidia-smi clock/throttle samples; summary() keeps those that arrived while
    the timed region ran (mark() brackets it)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []        # (arrival time, line)
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def mark(self, start: bool):
        t = time.perf_counter()
        self.window = (t, None) if start else (self.window[0], t)

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
        lines = self.lines
        if self.window and self.window[1] is not None:
            inside = [l for t, l in lines if self.window[0] <= t <= self.window[1] + 0.05]
            lines = inside if inside else [l for _, l in lines]
        else:
            lines = [l for _, l in lines]
        for line in lines:
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


def traffic_for(kernel_src_sha: str, workload, gated=False, chunk=64):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source for this workload at its full size (no --B/--H/--T
    override), on the plain output path and at the chunk length it names (64
    when it names none); else None.  workload: a Workload or a workload name
    (taken at full size)."""
    from xlstm_mlstm_matrix_b200 import inputs
    name = workload if isinstance(workload, str) else workload.name
    if not isinstance(workload, str) and workload != inputs.WORKLOADS.get(name, None).replace(seed=workload.seed):
        return None
    if gated:
        return None
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(name if chunk in (0, 64) else f"{name} L={chunk}")
    if not d or d.get("source_sha") != kernel_src_sha:
        return None
    return d.get("traffic_bytes_per_launch")


# the sources the forward chunkwise kernels are built from (the segment path included):
# a profile taken on them stays valid while none of these files changes
FORWARD_SOURCES = ("chunkwise_tc.cu", "segments.cu", "common.cuh", "sm100.cuh", "tc_common.cuh", "tma_host.cuh")


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "xlstm_mlstm_matrix_b200", "csrc")
    for f in FORWARD_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def tokens_per_step(w):
    return w.B if w.steps else w.B * w.T


def config_of(w, extra=None):
    c = {"workload": w.name, "B": w.B, "H": w.H, "T": w.T if not w.steps else 1,
         "d_qk": w.d_qk, "d_v": w.d_v}
    if w.steps:
        c["decode_steps"] = w.steps
    c.update(extra or {})
    return c


def cpu_baseline(w, inp, budget_s=12.0, gated=False):
    """Time the float64 oracle on a bounded sample of the workload, all host
    threads.  Returns the rate in the workload's tokens/s.  gated: the oracle's
    output gate follows the recurrence on the sample."""
    import oracle
    threads = oracle.default_threads()
    flat = lambda x: None if x is None else x.reshape((w.B * w.H,) + x.shape[2:])
    if w.steps:
        # decode: every (b, h) of a sample, a few steps each, state carried
        rng, C0, n0, m0 = inp["state"]
        nheads = min(w.B * w.H, max(threads * 4, 1))
        sel = lambda x: flat(x)[:nheads][None]
        C, n, m = sel(C0), sel(n0), sel(m0)
        t0 = time.perf_counter()
        nsteps = 0
        while True:
            st = inp["steps"][nsteps % len(inp["steps"])]
            _, C, n, m = oracle.step(*(sel(st[k]) for k in ("q", "k", "v", "i_pre", "f_pre")),
                                     C, n, m, qk_scale=inp["qk_scale"], threads=threads)
            nsteps += 1
            dt = time.perf_counter() - t0
            if dt >= budget_s or nsteps >= w.steps:
                break
        tokens = nsteps * nheads / w.H
        return {"value": tokens / dt, "unit": UNIT, "cores": min(threads, nheads), "kind": "oracle",
                "sample": f"{nsteps} decode steps of {nheads} of {w.B * w.H} (batch, head) pairs, "
                          f"float64, {min(threads, nheads)} threads; tokens = head-steps / H",
                "seconds": dt}
    sel = lambda x, hs: None if x is None else flat(x)[hs][None]
    # probe with a short prefix of one head to size the sample
    Tp = min(w.T, 256)
    t0 = time.perf_counter()
    oracle.forward(*(sel(inp[n], [0])[:, :, :Tp] for n in ("q", "k", "v", "i_pre", "f_pre")),
                   qk_scale=inp["qk_scale"], threads=1)
    per_head_token = (time.perf_counter() - t0) / Tp
    nheads = int(max(1, min(w.B * w.H, threads * budget_s / max(per_head_token * w.T, 1e-9))))
    hs = list(range(nheads))
    o_s = None
    if gated:
        from xlstm_mlstm_matrix_b200 import inputs as _inputs
        o_s = sel(_inputs.output_gate_pre(w, "bf16"), hs)
    t0 = time.perf_counter()
    h = oracle.forward(*(sel(inp[n], hs) for n in ("q", "k", "v", "i_pre", "f_pre", "C0", "n0", "m0")),
                       qk_scale=inp["qk_scale"], threads=threads)[0]
    if gated:
        oracle.output_gate(h, o_s)
    dt = time.perf_counter() - t0
    tokens = nheads * w.T / w.H          # head-tokens / heads per token
    return {"value": tokens / dt, "unit": UNIT, "cores": min(threads, nheads), "kind": "oracle",
            "sample": f"{nheads} of {w.B * w.H} (batch, head) pairs, full T={w.T}, float64, "
                      f"{min(threads, nheads)} threads; tokens = head-tokens / H",
            "seconds": dt}


def workload_for_rank(name, rank, B=0, H=0, T=0):
    """The workload one rank runs: every rank runs a full replica with its own
    seed (heads are independent, so ranks share nothing on the data path)."""
    from xlstm_mlstm_matrix_b200 import inputs
    base = inputs.WORKLOADS[name]
    w = base.replace(seed=base.seed + 1000 * rank)
    if B or H or T:   # a smaller case of the same layer (profiling captures)
        w = w.replace(B=B or w.B, H=H or w.H, T=T or w.T)
    return w


def max_over_ranks(x, dist=None, device=None):
    """The slowest rank's value (a float), identical on every rank."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(tokens_per_rank, world, ms_max):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def make_inputs(w, n_decode_steps=None):
    from xlstm_mlstm_matrix_b200 import inputs
    if not w.steps:
        return inputs.make_sequence(w)
    rng, C0, n0, m0 = inputs.decode_state(w)
    steps = list(inputs.decode_steps(w, rng, n_decode_steps))
    return {"state": (rng, C0, n0, m0), "steps": steps, "qk_scale": float(1.0 / np.sqrt(w.d_qk)),
            "workload": w}


def run_reference(args, rank, world):
    """--impl reference: the float64 oracle on host cores, same metric/workload."""
    from xlstm_mlstm_matrix_b200 import inputs
    if rank != 0:
        return
    w = inputs.WORKLOADS[args.workload]
    inp = make_inputs(w, n_decode_steps=32)
    # each step is a bounded sample so that the whole run stays within minutes
    budget = max(0.5, min(args.ref_budget, 120.0 / max(1, args.steps)))
    vals = []
    cb = None
    gated = args.output == "gated-bf16" and not w.steps
    for _ in range(max(1, args.steps)):
        cb = cpu_baseline(w, inp, budget_s=budget, gated=gated)
        vals.append(cb["value"])
    value = statistics.median(vals)
    cb["value"] = value
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tokens_per_step(w) / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_of(w, {"output": "gated-bf16"} if gated else None),
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _gate_overlap_split(w, dev):
    """Whether the gated tensor-core call splits its grid (one block per (sequence, 128
    value rows), one block per SM): more blocks than SMs, a partial last wave, at least
    one whole sequence before it, and at most four blocks before it for each SM that
    wave leaves idle."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    per_seq = (w.d_v + 127) // 128
    nblk = w.B * w.H * per_seq
    if nblk <= sms or nblk % sms == 0:
        return False
    first = (nblk - nblk % sms) // per_seq * per_seq
    idle = sms - (nblk - first)
    return first >= per_seq and idle >= 1 and first <= 4 * idle


def capi_output_stage(o):
    """The bf16-o~, bf16-h output stage descriptor for device tensor o."""
    from xlstm_mlstm_matrix_b200 import capi
    return capi.xlstm_mlstm_output_t(o.data_ptr(), capi.XLSTM_BF16, capi.XLSTM_BF16)


class _Sequence:
    """One chunkwise forward over the whole batch per step (gated: through the
    output stage, bf16 o~ in and bf16 h out)."""

    def __init__(self, w, inp, dev, stream, gated=False, chunk=64, kind="chunkwise"):
        import torch
        from xlstm_mlstm_matrix_b200 import capi
        self.w, self.inp, self.chunk = w, inp, chunk
        bf = w.dtype == "bf16"
        dev_t = lambda x, b: None if x is None else (
            torch.from_numpy(x).to(dev).to(torch.bfloat16) if b else torch.from_numpy(x).to(dev))
        self.ins = [dev_t(inp[n], bf) for n in ("q", "k", "v")] + \
                   [dev_t(inp[n], False) for n in ("i_pre", "f_pre", "C0", "n0", "m0")]
        self.gated = gated
        if gated:
            from xlstm_mlstm_matrix_b200 import inputs as _inputs
            self.ins.append(dev_t(_inputs.output_gate_pre(w, "bf16"), True))
        self.outs = [torch.empty(w.B, w.H, w.T, w.d_v, device=dev,
                                 dtype=torch.bfloat16 if gated else torch.float32),
                     torch.empty(w.B, w.H, w.d_v, w.d_qk, device=dev),
                     torch.empty(w.B, w.H, w.d_qk, device=dev), torch.empty(w.B, w.H, device=dev)]
        self.desc = capi.make_desc(w.B, w.H, w.T, w.d_qk, w.d_v,
                                   capi.XLSTM_BF16 if bf else capi.XLSTM_F32, inp["qk_scale"], chunk)
        # a workspace large enough for the segment-parallel path: a long sequence with few
        # heads then runs as segment summaries, their combination and the chunkwise kernel
        wsb = capi.xlstm_mlstm_workspace_size_parallel(self.desc)
        segmented = wsb > capi.xlstm_mlstm_workspace_size(self.desc)
        self.ws = torch.zeros(wsb, device=dev, dtype=torch.uint8)
        import ctypes
        P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
        if gated:
            self.fn = capi.load().xlstm_mlstm_fwd_chunkwise_out
            self.ostage = capi.xlstm_mlstm_output_t(self.ins[-1].data_ptr(), capi.XLSTM_BF16, capi.XLSTM_BF16)
            self.argv = (ctypes.byref(self.desc), ctypes.byref(self.ostage), *(P(t) for t in self.ins[:-1]),
                         *(P(t) for t in self.outs), P(self.ws), wsb, ctypes.c_void_p(stream.cuda_stream))
        else:
            self.fn = getattr(capi.load(), "xlstm_mlstm_fwd_" + kind)
            self.argv = (ctypes.byref(self.desc), *(P(t) for t in self.ins), *(P(t) for t in self.outs),
                         P(self.ws), wsb, ctypes.c_void_p(stream.cuda_stream))
        self.stream = stream
        if kind == "recurrent":   # one kernel, token by token; no segments
            segmented = False
        self.kernel = "chunkwise (segment summaries + combine + chunkwise)" if segmented else kind
        # kernels per call: the tensor-core path applies the output gate as a second, streaming
        # pass; when the grid ends in a partial wave the call splits in two launches, the gate of
        # the first overlapping the second (a segmented grid fits one wave and never splits)
        self.launches = (3 if segmented else 1) + (1 if gated else 0)
        if gated and not segmented and kind == "chunkwise" and _gate_overlap_split(w, dev):
            self.launches += 2
        if gated:
            self.kernel += " + output gate"
        self.name = "xlstm_mlstm_fwd_chunkwise_out" if gated else "xlstm_mlstm_fwd_" + kind

    def step(self, i):
        st = self.fn(*self.argv)
        if st != 0:
            from xlstm_mlstm_matrix_b200 import capi
            raise capi.XlstmError(st, self.name)

    def check_status(self):
        from xlstm_mlstm_matrix_b200 import capi
        for ws in [self.ws] + getattr(self, "e2e_ws", []):
            st, where = capi.xlstm_mlstm_workspace_status(ws, self.stream)
            if st != 0:
                raise capi.XlstmError(st, f"device status (where={where})")

    def e2e_slots(self, n=2):
        """n sets of device buffers for the end-to-end leg, each with pinned host
        copies of the step's inputs and result buffers and a call on its own device
        buffers: [(pairs_in [(dev, host)], pairs_out [(host, dev)], run)]."""
        import ctypes
        import torch
        hin = [None if t is None else t.cpu().pin_memory() for t in self.ins]
        P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
        slots = []
        for k in range(n):
            ins = self.ins if k == 0 else [None if t is None else torch.empty_like(t) for t in self.ins]
            outs = self.outs if k == 0 else [torch.empty_like(t) for t in self.outs]
            ws = self.ws if k == 0 else torch.zeros_like(self.ws)
            if k > 0:
                self.e2e_ws = getattr(self, "e2e_ws", []) + [ws]
            if self.gated:
                ost = capi_output_stage(ins[-1])
                argv = (self.argv[0], ctypes.byref(ost), *(P(t) for t in ins[:-1]), *(P(t) for t in outs), P(ws),
                        ws.numel(), ctypes.c_void_p(self.stream.cuda_stream))
            else:
                ost = None
                argv = (self.argv[0], *(P(t) for t in ins), *(P(t) for t in outs), P(ws), ws.numel(),
                        ctypes.c_void_p(self.stream.cuda_stream))

            def run(argv=argv, ost=ost):
                st = self.fn(*argv)
                if st != 0:
                    from xlstm_mlstm_matrix_b200 import capi
                    raise capi.XlstmError(st, self.name)
            hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
            slots.append(([(d, h) for d, h in zip(ins, hin) if d is not None], list(zip(hout, outs)), run))
        return slots


class _Decode:
    """One xlstm_mlstm_step per step over B*H heads, state in place in HBM."""

    def __init__(self, w, inp, dev, stream):
        import torch
        from xlstm_mlstm_matrix_b200 import capi
        self.w, self.inp = w, inp
        _, C0, n0, m0 = inp["state"]
        S = len(inp["steps"])
        stack = lambda k: np.stack([st[k] for st in inp["steps"]])
        bfd = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16)
        self.q, self.k, self.v = bfd(stack("q")), bfd(stack("k")), bfd(stack("v"))
        self.ig = torch.from_numpy(stack("i_pre")).to(dev)
        self.fg = torch.from_numpy(stack("f_pre")).to(dev)
        self.C = torch.from_numpy(C0).to(dev)
        self.n = torch.from_numpy(n0).to(dev)
        self.m = torch.from_numpy(m0).to(dev)
        self.h = torch.empty(w.B, w.H, w.d_v, device=dev)
        self.S = S
        self.desc = capi.make_desc(w.B, w.H, 1, w.d_qk, w.d_v, capi.XLSTM_BF16, inp["qk_scale"], 64)
        self.fn = capi.load().xlstm_mlstm_step
        import ctypes
        self.P = lambda t: ctypes.c_void_p(t.data_ptr())
        self.cs = ctypes.c_void_p(stream.cuda_stream)
        self.stream = stream
        self.kernel = "step"
        self.launches = 1
        self.name = "xlstm_mlstm_step"

    def step(self, i, src=None):
        import ctypes
        P = self.P
        j = i % self.S
        q, k, v, ig, fg = src if src is not None else (self.q[j], self.k[j], self.v[j], self.ig[j],
                                                       self.fg[j])
        st = self.fn(ctypes.byref(self.desc), P(q), P(k), P(v), P(ig), P(fg), P(self.C), P(self.n),
                     P(self.m), P(self.h), P(self.C), P(self.n), P(self.m), self.cs)
        if st != 0:
            from xlstm_mlstm_matrix_b200 import capi
            raise capi.XlstmError(st, self.name)

    def check_status(self):
        pass

    def e2e_slots(self, n=2):
        """n sets of device buffers for one step's inputs (q, k, v, gates) and h~,
        with pinned host copies; the state stays resident on the device and every
        step updates it in place, in order on the launch stream, as in a decode loop."""
        import ctypes
        import torch
        j = 0
        hin = [self.q[j].cpu().pin_memory(), self.k[j].cpu().pin_memory(),
               self.v[j].cpu().pin_memory(), self.ig[j].cpu().pin_memory(),
               self.fg[j].cpu().pin_memory()]
        slots = []
        for k in range(n):
            dev_in = [torch.empty_like(t, device=self.h.device) for t in hin]
            h = self.h if k == 0 else torch.empty_like(self.h)

            def run(dev_in=dev_in, h=h):
                P = self.P
                st = self.fn(ctypes.byref(self.desc), *(P(t) for t in dev_in), P(self.C), P(self.n), P(self.m),
                             P(h), P(self.C), P(self.n), P(self.m), self.cs)
                if st != 0:
                    from xlstm_mlstm_matrix_b200 import capi
                    raise capi.XlstmError(st, self.name)
            slots.append((list(zip(dev_in, hin)), [(torch.empty(h.shape, dtype=h.dtype).pin_memory(), h)], run))
        return slots


class _Backward:
    """One xlstm_mlstm_bwd_chunkwise over the whole batch per step: gradients of
    q, k, v and both gates for a synthetic upstream dh (normal, fp32)."""

    def __init__(self, w, inp, dev, stream):
        import ctypes
        import torch
        from xlstm_mlstm_matrix_b200 import capi
        seq = _Sequence(w, inp, dev, stream)
        self.ins = seq.ins
        g = torch.Generator(device=dev).manual_seed(w.seed + 31)
        self.dh = torch.randn(w.B, w.H, w.T, w.d_v, device=dev, generator=g)
        f32 = dict(device=dev, dtype=torch.float32)
        self.outs = [torch.empty(w.B, w.H, w.T, w.d_qk, **f32), torch.empty(w.B, w.H, w.T, w.d_qk, **f32),
                     torch.empty(w.B, w.H, w.T, w.d_v, **f32), torch.empty(w.B, w.H, w.T, **f32),
                     torch.empty(w.B, w.H, w.T, **f32)]
        self.desc = seq.desc
        wsb = capi.xlstm_mlstm_bwd_workspace_size(self.desc)
        self.ws = torch.empty(wsb, device=dev, dtype=torch.uint8)
        P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
        self.fn = capi.load().xlstm_mlstm_bwd_chunkwise
        self.argv = (ctypes.byref(self.desc), *(P(t) for t in self.ins), P(self.dh), None, None,
                     *(P(t) for t in self.outs), None, None, None, P(self.ws), wsb,
                     ctypes.c_void_p(stream.cuda_stream))
        self.kernel = "backward (chunk entry states, chunk exit adjoints, chunk gradients; fp32 CUDA cores)"
        self.launches = 5
        self.name = "xlstm_mlstm_bwd_chunkwise"

    def step(self, i):
        st = self.fn(*self.argv)
        if st != 0:
            from xlstm_mlstm_matrix_b200 import capi
            raise capi.XlstmError(st, self.name)

    def check_status(self):
        pass


def algorithmic_backward(w):
    """Bytes of one backward over B*H*T head-tokens: q, k, v, the gates and dh
    read; dq, dk, dv, di~, df~ written (fp32); the state's gradient if any."""
    e = 2 if w.dtype == "bf16" else 4
    N = w.B * w.H * w.T
    bytes_ = N * ((2 * w.d_qk + w.d_v) * e + 8 + 4 * w.d_v + 4 * (2 * w.d_qk + w.d_v) + 8)
    return bytes_


def time_job(job, steps, warmup, stream, dev, gpu_index):
    """Warm-up, then `steps` launches bracketed by CUDA events on the launch
    stream with clock samples during the timed region: (ms per step, clocks)."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(warmup):
            job.step(i)
    stream.synchronize()
    job.check_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_index) as clk:
        clk.mark(True)
        e0.record(stream)
        for i in range(steps):
            job.step(warmup + i)
        e1.record(stream)
        e1.synchronize()
        clk.mark(False)
    torch.cuda.synchronize(dev)
    job.check_status()
    return e0.elapsed_time(e1) / steps, clk.summary()


# (workload, chunk length or the recurrent call); plus the headline layer's backward
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # fp32 FMA lanes x 2 FLOP x max SM clock
SECONDARY = (("decode", 0), ("long_context", 64), ("long_context", 128), ("many_short", 64), ("many_short", 128),
             ("many_short", "recurrent"), ("layer_7b", "recurrent"))


def run_secondary(args, dev, stream, gpu_index):
    """The other workloads of the benchmark spec, each timed like the headline one: the
    decode step kernel (B=128 H=8 d_qk=256 d_v=512, state resident in HBM), the
    long-context and many-short-sequences layers at chunk 64 and 128, and the
    recurrent call on the many-short and 7B-like layers.  One entry each with its
    own roofline fraction (HBM; fp32 ALU for the recurrent call); the headline
    value stays the 7B-like layer."""
    hbm, bf16_peak, _, peak_src = peaks()
    out = []
    inp_of = {}
    for name, chunk in SECONDARY:
        if name == args.workload and chunk in (0, args.chunk):
            continue
        kind = "recurrent" if chunk == "recurrent" else "chunkwise"
        w = workload_for_rank(name, 0)
        if name not in inp_of:
            inp_of.clear()
            inp_of[name] = make_inputs(w)
        inp = inp_of[name]
        job = _Decode(w, inp, dev, stream) if w.steps else _Sequence(w, inp, dev, stream, chunk=chunk if
                                                                      kind == "chunkwise" else 64, kind=kind)
        steps = min(args.steps, 100 if w.steps else 50)
        ms, clocks = time_job(job, steps, args.warmup, stream, dev, gpu_index)
        bytes_, flops = algorithmic(w)
        gbs = bytes_ / (ms * 1e-3) / 1e9
        label = name if not chunk else (f"{name} recurrent" if kind == "recurrent" else f"{name} L={chunk}")
        if kind == "recurrent":
            # token by token on fp32 CUDA cores: 4 d_qk d_v + 4 d_qk FLOPs per head-token (state update
            # and readout), against the fp32 FMA peak of 148 SMs x 128 lanes x 2 FLOP x 1965 MHz
            rflops = w.B * w.H * w.T * (4 * w.d_qk * w.d_v + 4 * w.d_qk)
            tf = rflops / (ms * 1e-3) / 1e12
            roof = {"bound": "alu", "achieved": tf, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                    "frac": tf / FP32_PEAK_TFLOPS, "peak_source": "unit counts x max SM clock",
                    "flops_per_launch": rflops, "hbm_frac": gbs / hbm, "traffic": None}
        else:
            roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                    "frac": gbs / hbm, "peak_source": peak_src,
                    "algorithmic_bytes_per_launch": bytes_,
                    "traffic": traffic_for(kernel_source_sha(), w, chunk=chunk)}
        out.append({"workload": label, "kernel": job.kernel, "ms_per_step": ms,
                    "value": tokens_per_step(w) / (ms * 1e-3), "unit": UNIT,
                    "hbm_gbs": gbs, "tflops": flops / (ms * 1e-3) / 1e12,
                    "roofline": roof,
                    "gpu_launches": steps * job.launches, "steps": steps, "clocks": clocks,
                    "config": config_of(w, {"l2": "working set larger than L2 (126 MB)",
                                            **({"chunk": chunk} if kind == "chunkwise" and chunk else {}),
                                            **({"call": "xlstm_mlstm_fwd_recurrent"} if kind == "recurrent" else {})})})
        del job, inp
    inp_of.clear()
    # the backward of the headline sequence workload
    w = workload_for_rank(args.workload, 0, args.B, args.H, args.T)
    if not w.steps:
        inp = make_inputs(w)
        job = _Backward(w, inp, dev, stream)
        steps = min(args.steps, 10)
        ms, clocks = time_job(job, steps, args.warmup, stream, dev, gpu_index)
        bytes_ = algorithmic_backward(w)
        gbs = bytes_ / (ms * 1e-3) / 1e9
        out.append({"workload": f"{w.name} backward", "kernel": job.kernel, "ms_per_step": ms,
                    "value": tokens_per_step(w) / (ms * 1e-3), "unit": UNIT, "hbm_gbs": gbs,
                    "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                 "frac": gbs / hbm, "peak_source": peak_src,
                                 "algorithmic_bytes_per_launch": bytes_, "traffic": None},
                    "gpu_launches": steps * job.launches, "steps": steps, "clocks": clocks,
                    "config": config_of(w, {"l2": "working set larger than L2 (126 MB)",
                                            "upstream": "dh ~ N(0, 1) fp32; no final-state gradient"})})
        del job, inp
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    from xlstm_mlstm_matrix_b200 import capi, inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    capi.load()
    w = workload_for_rank(args.workload, rank, args.B, args.H, args.T)
    inp = make_inputs(w)
    stream = torch.cuda.Stream(dev)
    gated = args.output == "gated-bf16"
    if gated and w.steps:
        raise SystemExit("--output gated-bf16 applies to the sequence workloads")
    job = _Decode(w, inp, dev, stream) if w.steps else _Sequence(w, inp, dev, stream, gated=gated, chunk=args.chunk)

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    def slowest(x):
        return max_over_ranks(x, dist, dev)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            job.step(i)
    stream.synchronize()
    job.check_status()          # no bounded device wait gave up during warm-up

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank if os.environ.get("CUDA_VISIBLE_DEVICES") is None else 0) as clk:
        clk.mark(True)
        e0.record(stream)
        for i in range(args.steps):
            job.step(args.warmup + i)
        e1.record(stream)
        e1.synchronize()
        clk.mark(False)
    torch.cuda.synchronize(dev)
    barrier()
    ms = slowest(e0.elapsed_time(e1) / args.steps)
    job.check_status()

    tokens = tokens_per_step(w)
    value = job_rate(tokens, world, ms)
    bytes_, flops = algorithmic(w, gated=gated)
    hbm, bf16_peak, _, peak_src = peaks()
    achieved_gbs = bytes_ / (ms * 1e-3) / 1e9
    src_sha = kernel_source_sha()

    # ---- end to end: pinned host buffers through the same call ---------------------
    e2e_steps = 0 if args.no_e2e else max(1, min(args.steps, 5 if not w.steps else args.steps))
    e2e = None
    if e2e_steps:
        # Two steps in flight: step i copies its inputs in on s_in, runs on the launch
        # stream and copies its results out on s_out, with device buffer set i % 2; step
        # i+2 reuses a set once step i's call has read its inputs and its results have
        # been copied out.  Every step's copies are inside the timed region.
        slots = job.e2e_slots(2)
        h2d = sum(s.numel() * s.element_size() for _, s in slots[0][0])
        d2h = sum(d.numel() * d.element_size() for d, _ in slots[0][1])
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "call", "out")}

        def e2e_step(i):
            k = i % 2
            pairs_in, pairs_out, run = slots[k]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev["call"][k])
                for dst, src in pairs_in:
                    dst.copy_(src, non_blocking=True)
                ev["in"][k].record(s_in)
            stream.wait_event(ev["in"][k])
            if i >= 2:
                stream.wait_event(ev["out"][k])
            with torch.cuda.stream(stream):
                run()
                ev["call"][k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["call"][k])
                for dst, src in pairs_out:
                    dst.copy_(src, non_blocking=True)
                ev["out"][k].record(s_out)

        for i in range(2):   # warm-up of both buffer sets
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier()
        e0.record(s_in)
        for i in range(e2e_steps):
            e2e_step(i)
        stream.wait_stream(s_out)
        e1.record(stream)
        e1.synchronize()
        barrier()
        e2e_ms = slowest(e0.elapsed_time(e1) / e2e_steps)
        e2e = {"value": job_rate(tokens, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "pipeline": "two steps in flight: H2D, call and D2H on three streams"}
        if w.steps:
            e2e["note"] = "per step: H2D of q, k, v and gates, D2H of h~; state resident on the device"
        job.check_status()

    if rank == 0:
        l2 = (f"inputs larger than L2 ({bytes_ / 1e9:.2f} GB per step vs 126 MB L2)"
              if bytes_ > 4 * 126e6 else "working set near L2 size; no flush")
        extra = {"inputs": ("bf16 q/k/v and o~, fp32 gates; bf16 h = sigmoid(o~) h~ (output stage), fp32 state"
                            if gated else "bf16 q/k/v, fp32 gates; fp32 h and state"), "l2": l2,
                 "parallelism": f"replicas x{world} (independent heads)"}
        if not w.steps:
            extra["chunk"] = args.chunk
        if gated:
            extra["output"] = "gated-bf16"
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w, extra),
            "tflops": world * flops / (ms * 1e-3) / 1e12,
            "hbm_gbs": achieved_gbs,
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": achieved_gbs / hbm, "traffic": traffic_for(src_sha, w, gated, args.chunk),
                         "peak_source": peak_src, "kernel": job.kernel,
                         "algorithmic_bytes_per_launch": bytes_, "flops_per_launch": flops,
                         "tensor_frac": flops / (ms * 1e-3) / 1e12 / bf16_peak},
            "gpu_launches": args.steps * job.launches,
            "e2e": e2e,
            "clocks": clk.summary(),
            "kernel_source_sha": src_sha,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, inp, budget_s=args.ref_budget, gated=gated)
        if world == 1 and not args.no_secondary:
            gi = local_rank if os.environ.get("CUDA_VISIBLE_DEVICES") is None else 0
            line["secondary"] = run_secondary(args, dev, stream, gi)
        print(json.dumps(line), flush=True)


def run_mma_probe():
    """tcgen05.mma issue cost: one thread issues back-to-back MMAs (K = 16, bf16
    operands, zero data) and clock64 brackets the sequence up to the completion
    of a final commit.  Prints one table row per shape: cycles per instruction
    on one CTA and the median over 148 CTAs (one per SM), and the fraction of
    the tensor pipe's dense rate that cost implies (M = 128: 8192 flop per SM
    cycle; M = 64 runs on half the datapath)."""
    import ctypes
    import torch  # noqa: F401  (CUDA context for the probe library)
    lib = ctypes.CDLL(os.path.join(ROOT, "xlstm_mlstm_matrix_b200", "libxlstm_mma_probe.so"))
    f = lib.mma_probe_run
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 10 + [ctypes.POINTER(ctypes.c_longlong)]
    issue_names = {0: "one thread", 1: "warp + elect.sync", 2: "two warps", 3: "one thread, unrolled",
                   4: "rolled K loop", 5: "unrolled, integer op between", 6: "unrolled, runtime base",
                   7: "unrolled by 4", 8: "no MMA", 9: "one thread, unrolled (ts)",
                   10: "chunk program, rolled", 11: "chunk program, unrolled"}
    bg_names = {0: "", 1: " + bg tmem ld", 2: " + bg tmem st", 3: " + bg smem ld", 4: " + bg smem st",
                5: " + bg alu", 6: " + bg bulk copies"}
    cases = []   # (form, M, N, a_mn, b_mn, accumulators, commit_every, issue + 16 * background)
    for M, N in ((64, 64), (128, 64), (128, 128), (128, 256)):
        cases.append(("ss", M, N, 0, 0, 1, 0, 0))
    cases += [("ts", 128, 64, 0, 0, 1, 0, 0), ("ss", 128, 64, 1, 1, 1, 0, 0), ("ss", 128, 64, 0, 0, 2, 0, 0),
              ("ss", 128, 64, 0, 0, 1, 1, 0), ("ss", 128, 64, 0, 0, 1, 0, 1), ("ss", 128, 64, 0, 0, 1, 0, 2),
              ("ss", 128, 64, 0, 0, 1, 0, 4), ("ss", 128, 64, 0, 0, 1, 0, 5), ("ss", 128, 64, 0, 0, 1, 0, 6),
              ("ss", 128, 64, 0, 0, 1, 0, 7)]
    for M, N in ((64, 64), (128, 64), (128, 128), (128, 256)):
        cases.append(("ss", M, N, 0, 0, 1, 0, 3))
    for N in (64, 128, 256):
        cases.append(("ts", 128, N, 0, 0, 1, 0, 9))
    # background traffic on warps 1-3: alone, and beside unrolled MMAs
    for bg in (1, 2, 3, 4):
        cases += [("ss", 128, 64, 0, 0, 1, 0, 8 + 16 * bg), ("ss", 128, 64, 0, 0, 1, 0, 3 + 16 * bg),
                  ("ts", 128, 64, 0, 0, 1, 0, 9 + 16 * bg), ("ss", 128, 256, 0, 0, 1, 0, 3 + 16 * bg)]
    # pseudo-random operands (+256), and background traffic on 11 warps (+128)
    R, W = 256, 128
    cases += [("ss", 64, 64, 0, 0, 1, 0, 3 + R), ("ss", 128, 64, 0, 0, 1, 0, 3 + R), ("ss", 128, 128, 0, 0, 1, 0, 3 + R),
              ("ss", 128, 256, 0, 0, 1, 0, 3 + R), ("ts", 128, 64, 0, 0, 1, 0, 9 + R), ("ts", 128, 256, 0, 0, 1, 0, 9 + R),
              ("ss", 128, 64, 0, 0, 1, 0, 4 + R)]
    for bg in (1, 2, 3, 4):
        cases += [("ss", 128, 64, 0, 0, 1, 0, 8 + 16 * bg + W + R), ("ss", 128, 64, 0, 0, 1, 0, 3 + 16 * bg + W + R),
                  ("ts", 128, 64, 0, 0, 1, 0, 9 + 16 * bg + W + R)]
    # the chunkwise kernel's per-chunk MMA program (56 MMAs + 6 commits), alone and beside busy warps
    for prog in (10, 11):
        cases += [("ss", 128, 64, 0, 0, 1, 0, prog), ("ss", 128, 64, 0, 0, 1, 0, prog + 16 * 5 + W),
                  ("ss", 128, 64, 0, 0, 1, 0, prog + 16 * 3 + W), ("ss", 128, 64, 0, 0, 1, 0, prog + 16 * 1 + W),
                  ("ss", 128, 64, 0, 0, 1, 0, prog + 16 * 6)]
    cases += [("ss", 128, 64, 0, 0, 1, 0, 8 + 16 * 6), ("ss", 128, 64, 0, 0, 1, 0, 3 + 16 * 6),
              ("ts", 128, 64, 0, 0, 1, 0, 9 + 16 * 6)]
    nmma = 512
    for form, M, N, amn, bmn, nacc, ce, issue in cases:
        if issue % 16 >= 10:
            nmma = 56 * 32
        res, bgc = {}, {}
        for ctas in (1, 148):
            buf = (ctypes.c_longlong * (3 * ctas))()
            rc = f(1 if form == "ts" else 0, M, N, amn, bmn, nmma, nacc, ce, issue, ctas, buf)
            if rc != 0:
                raise SystemExit(f"probe failed rc={rc} for {form} M{M} N{N} issue {issue}")
            vals = list(buf)
            res[ctas] = statistics.median(vals[:ctas]) / nmma
            its = vals[ctas:2 * ctas]
            bgc[ctas] = statistics.median([c / i for c, i in zip(vals[2 * ctas:], its) if i > 0]) if any(its) else None
        ideal = M * N * 16 * 2 / (8192 if M == 128 else 4096)
        row = {"form": form, "M": M, "N": N, "a_mn": amn, "b_mn": bmn, "accumulators": nacc,
               "commit_every": ce, "issue": issue_names[issue % 16] + bg_names[(issue // 16) % 8] +
               (" x11 warps" if issue & 128 else "") + (", random data" if issue & 256 else ""),
               "cycles_1cta": round(res[1], 1), "cycles_148cta": round(res[148], 1), "ideal_cycles": ideal,
               "pipe_frac_148": round(ideal / res[148], 3) if res[148] else None,
               "bg_cycles_per_iter_148": None if bgc[148] is None else round(bgc[148], 1)}
        if issue % 16 >= 10:
            row["cycles_per_chunk_148"] = round(res[148] * nmma / 32)
        print(json.dumps(row), flush=True)
        nmma = 512


def main():
    from xlstm_mlstm_matrix_b200.inputs import WORKLOADS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=[k for k in WORKLOADS if k != "tiny_fp32"],
                    default=DEFAULT_WORKLOAD)
    ap.add_argument("--ref-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--output", choices=["plain", "gated-bf16"], default="plain",
                    help="gated-bf16: the fused output stage (h = sigmoid(o~) h~, bf16 o~ and h)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--chunk", type=int, choices=[64, 128], default=64,
                    help="chunk length of the headline sequence workload (128: d_qk <= 128 only)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the decode, long-context and many-short entries of the line")
    ap.add_argument("--B", type=int, default=0, help="override the batch size (profiling)")
    ap.add_argument("--H", type=int, default=0, help="override the head count (profiling)")
    ap.add_argument("--T", type=int, default=0, help="override the sequence length (profiling)")
    ap.add_argument("--probe", choices=["mma"], default=None,
                    help="mma: tcgen05.mma issue-cost microbenchmark instead of the benchmark")
    args = ap.parse_args()
    if args.probe == "mma":
        run_mma_probe()
        return
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
