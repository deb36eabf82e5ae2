"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the float64 oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from xlstm_mlstm_matrix_b200 import capi, inputs

# Tolerances (per-row normalised relative error, see inputs.relative_errors).
TOL = {"f32": dict(max=1e-4, mean=1e-4), "bf16": dict(max=2e-2, mean=4e-3)}


def to_dev(x, dtype: str):
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def gpu_sequence(inp: dict, kind: str, chunk: int = 0, qk_scale=None, state=None):
    w = inputs_workload(inp)
    dt = w.dtype
    q, k, v = (to_dev(inp[n], dt) for n in ("q", "k", "v"))
    ig, fg = to_dev(inp["i_pre"], "f32"), to_dev(inp["f_pre"], "f32")
    if state is None and inp.get("C0") is not None:
        state = tuple(to_dev(inp[n], "f32") for n in ("C0", "n0", "m0"))
    scale = inp["qk_scale"] if qk_scale is None else qk_scale
    h, (C, n, m) = capi.fwd(q, k, v, ig, fg, state=state, qk_scale=scale, chunk=chunk, kind=kind)
    torch.cuda.synchronize()
    return h.cpu().numpy(), C.cpu().numpy(), n.cpu().numpy(), m.cpu().numpy()


def inputs_workload(inp):
    return inp["workload"]


def oracle_sequence(inp: dict, qk_scale=None, heads=None):
    """Oracle on all heads, or on the listed flat (b*H + h) head indices."""
    q, k, v, ig, fg = (inp[n] for n in ("q", "k", "v", "i_pre", "f_pre"))
    C0, n0, m0 = inp.get("C0"), inp.get("n0"), inp.get("m0")
    scale = inp["qk_scale"] if qk_scale is None else qk_scale
    if heads is not None:
        B, H = q.shape[:2]
        sel = lambda x: None if x is None else x.reshape((B * H,) + x.shape[2:])[heads][None]
        q, k, v, ig, fg, C0, n0, m0 = (sel(x) for x in (q, k, v, ig, fg, C0, n0, m0))
    return oracle.forward(q, k, v, ig, fg, C0, n0, m0, qk_scale=scale)


def select_heads(x, heads):
    B, H = x.shape[:2]
    return x.reshape((B * H,) + x.shape[2:])[heads][None]


def compare(got, ref, dtype: str, what: str = "", check_state=True):
    """got/ref: (h, C, n, m).  Raises AssertionError with the error figures."""
    tol = TOL[dtype]
    h, C, n, m = got
    hr, Cr, nr, mr = ref
    mx, mean = inputs.relative_errors(h, hr)
    msgs = [f"h max {mx:.2e} mean {mean:.2e}"]
    ok = mx <= tol["max"] and mean <= tol["mean"]
    if check_state:
        # gauge-fixed state: C_gpu e^{m_gpu - m_ref} against C_ref
        g = np.exp(m.astype(np.float64) - mr)
        cmx, cmean = inputs.relative_errors(C * g[..., None, None], Cr, row_axes=2)
        nmx, nmean = inputs.relative_errors(n * g[..., None], nr)
        merr = float(np.max(np.abs(m - mr) / np.maximum(1.0, np.abs(mr)))) if m.size else 0.0
        msgs += [f"C max {cmx:.2e} mean {cmean:.2e}", f"n max {nmx:.2e} mean {nmean:.2e}",
                 f"m {merr:.2e}"]
        ok = ok and cmx <= tol["max"] and cmean <= tol["mean"] and nmx <= tol["max"] \
            and nmean <= tol["mean"] and merr <= 1e-4
    assert ok, f"{what}: " + ", ".join(msgs)
    return msgs
