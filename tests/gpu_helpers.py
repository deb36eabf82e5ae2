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


def gpu_sequence(inp: dict, kind: str, chunk: int = 0, qk_scale=None, state=None, parallel=False):
    """The CUDA path through the C ABI.  parallel=True gives the chunkwise call a
    workspace large enough for the segment-parallel evaluation."""
    w = inputs_workload(inp)
    dt = w.dtype
    q, k, v = (to_dev(inp[n], dt) for n in ("q", "k", "v"))
    ig, fg = to_dev(inp["i_pre"], "f32"), to_dev(inp["f_pre"], "f32")
    if state is None and inp.get("C0") is not None:
        state = tuple(to_dev(inp[n], "f32") for n in ("C0", "n0", "m0"))
    scale = inp["qk_scale"] if qk_scale is None else qk_scale
    ws = None
    if kind == "chunkwise":
        B, H, T, dqk = q.shape
        desc = capi.make_desc(B, H, T, dqk, v.shape[-1], capi.XLSTM_BF16 if dt == "bf16" else capi.XLSTM_F32,
                              scale, chunk)
        size = (capi.xlstm_mlstm_workspace_size_parallel if parallel else capi.xlstm_mlstm_workspace_size)(desc)
        ws = torch.zeros(max(256, size), device=q.device, dtype=torch.uint8)
    h, (C, n, m) = capi.fwd(q, k, v, ig, fg, state=state, qk_scale=scale, chunk=chunk, kind=kind, workspace=ws)
    torch.cuda.synchronize()
    if ws is not None:   # no bounded device wait gave up
        code, where = capi.xlstm_mlstm_workspace_status(ws)
        assert code == capi.XLSTM_OK, f"device status {capi.xlstm_status_string(code)} (wait {where})"
    return h.cpu().numpy(), C.cpu().numpy(), n.cpu().numpy(), m.cpu().numpy()


def small_inputs(B, H, T, dqk, dv, dtype, state, seed=7, gate="std", mean_i=0.0, std_i=1.5):
    """Seeded inputs of the tiny workload's distributions at another shape."""
    w = inputs.WORKLOADS["tiny_fp32"].replace(
        B=B, H=H, T=T, d_qk=dqk, d_v=dv, dtype=dtype, gate=gate, mean_i=mean_i, std_i=std_i,
        state="normal_m_uniform" if state else "zero", seed=seed)
    return inputs.make_sequence(w)


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


def condition_numbers(inp, qk_scale=None, heads=None):
    """Per-token condition numbers of the readout, in float64:
      kappa_den_t = sum_j |n~_tj q_tj| / max(|sum_j n~_tj q_tj|, e^{-m_t})
      kappa_num_t = max_r sum_j |C~_t,rj q_tj| / max_r |sum_j C~_t,rj q_tj|
    A row of h~ is a dot product divided by a dot product; an fp32 evaluation
    of either in any order carries a relative error of order
    (kappa_den + kappa_num) * 2^-24 on that row, so where they cancel no fp32
    kernel meets 1e-4.  These set tolerances only; nothing is compared with them."""
    q, k, v, ig, fg = (inp[x].astype(np.float64) for x in ("q", "k", "v", "i_pre", "f_pre"))
    C0, n0, m0 = inp.get("C0"), inp.get("n0"), inp.get("m0")
    if heads is not None:
        q, k, v, ig, fg = (select_heads(x, heads) for x in (q, k, v, ig, fg))
        C0, n0, m0 = (None if x is None else select_heads(x, heads) for x in (C0, n0, m0))
    scale = inp["qk_scale"] if qk_scale is None else qk_scale
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    C = np.zeros((B, H, dv, dqk)) if C0 is None else C0.astype(np.float64).copy()
    n = np.zeros((B, H, dqk)) if n0 is None else n0.astype(np.float64).copy()
    m = np.zeros((B, H)) if m0 is None else m0.astype(np.float64).copy()
    kd = np.ones((B, H, T))
    kn = np.ones((B, H, T))
    mabs = np.zeros((B, H, T))
    for t in range(T):
        mn = np.maximum(fg[:, :, t] + m, ig[:, :, t])
        fp = np.exp(fg[:, :, t] + m - mn)
        ip = np.exp(ig[:, :, t] - mn)
        C = fp[..., None, None] * C + ip[..., None, None] * v[:, :, t, :, None] * k[:, :, t, None, :]
        n = fp[..., None] * n + ip[..., None] * k[:, :, t]
        qs = scale * q[:, :, t]
        prod = n * qs
        kd[:, :, t] = np.abs(prod).sum(-1) / np.maximum(np.abs(prod.sum(-1)), np.exp(-mn))
        mag = np.einsum("bhrc,bhc->bhr", np.abs(C), np.abs(qs)).max(-1)
        val = np.abs(np.einsum("bhrc,bhc->bhr", C, qs)).max(-1)
        kn[:, :, t] = mag / np.where(val > 0, val, 1.0)
        mabs[:, :, t] = np.abs(mn)
        m = mn
    return kd, kn, mabs


def fp32_row_tolerance(inp, qk_scale=None, heads=None, base=1e-4):
    """max(base, 32 * 2^-24 * (kappa_den + kappa_num + |m_t|)) per (b, h, t) row.

    The |m_t| term covers the log-space gate arithmetic: exponents such as
    f~ + m_{t-1} - m_t are formed from numbers of size |m|, so in fp32 they carry
    an absolute error of about |m| 2^-24, a relative error of the gates."""
    kd, kn, mabs = condition_numbers(inp, qk_scale, heads)
    return np.maximum(base, 32.0 * 2.0 ** -24 * (kd + kn + mabs))


def compare(got, ref, dtype: str, what: str = "", check_state=True, row_tol=None):
    """got/ref: (h, C, n, m).  Raises AssertionError with the error figures.
    row_tol: per-(b, h, t) tolerance for fp32 inputs (fp32_row_tolerance);
    without it every row must meet 1e-4."""
    tol = TOL[dtype]
    h, C, n, m = got
    hr, Cr, nr, mr = ref
    mx, mean = inputs.relative_errors(h, hr)
    msgs = [f"h max {mx:.2e} mean {mean:.2e}"]
    if row_tol is not None and dtype == "f32" and h.size:
        scale = np.max(np.abs(hr), axis=-1, keepdims=True)
        err = np.abs(h.astype(np.float64) - hr) / np.where(scale > 0, scale, 1.0)
        worst = float(np.max(err / row_tol[..., None]))
        msgs.append(f"h max/row-tol {worst:.2f} (row-tol max {float(np.max(row_tol)):.1e})")
        ok = worst <= 1.0 and mean <= tol["mean"]
    else:
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
