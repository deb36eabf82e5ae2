"""Seeded synthetic inputs for the mLSTM forward, shared by tests, smoke check and bench.

This module holds no mLSTM arithmetic: it only draws random tensors with the
shapes and value distributions of the workloads below and rounds them to the
storage dtype (bf16 round-to-nearest-even, or fp32).  Both the CUDA path and
the float64 oracle consume exactly the rounded values it returns.

Recipe (all draws from ``numpy.random.default_rng(seed)``, in this order):
  q, k, v   standard normal (float32 draws), then rounded to the storage dtype
  i~        normal(mean_i, std_i)              (float32)
  f~        logsigmoid of normal(mu_f, std_f)  (float32); for the "mixed" gate
            recipe a second normal(0.5, 1) draw and a Bernoulli(1/2) mask pick,
            element by element, between the log-sigmoid value and the raw one
  C0, n0    normal(0, 0.1) (float32) when the workload carries an initial state
  m0        uniform(0, 5) or zero (float32)
The decode workload draws its initial state first, then q, k, v, i~, f~ per step.
Output-gate pre-activations o~ (the fused output stage) come from a generator of
their own, seeded with the workload seed + 7919, so the draws above are unchanged:
  o~        normal(0, 3) (float32), rounded to its storage dtype
"""
from __future__ import annotations

import dataclasses
from typing import Iterator

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d_qk: int
    d_v: int
    dtype: str            # "bf16" or "f32": storage type of q, k, v
    gate: str             # "std", "mixed"
    mean_i: float
    std_i: float
    mu_f: float
    std_f: float
    state: str            # "zero", "normal_m_uniform", "normal_m_zero"
    seed: int
    chunk: int = 64
    steps: int = 0        # >0: a decode workload of this many single steps

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.B * self.T if self.steps == 0 else self.B * self.steps


# The five workloads, with the shapes and distributions of the xLSTM layer
# settings they stand for (a tiny fp32 case, a 7B-like layer, a long-context
# layer, many short sequences with small heads, and recurrent decode).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 2, 256, 64, 64, "f32", "std", 0.0, 1.0, 3.0, 1.5,
                          "zero", seed=0),
    "layer_7b": Workload("layer_7b", 8, 8, 4096, 256, 512, "bf16", "std", -2.0, 1.0, 3.0, 1.5,
                         "zero", seed=1),
    "long_context": Workload("long_context", 1, 8, 65536, 128, 128, "bf16", "std", 0.0, 2.0,
                             4.0, 1.0, "normal_m_uniform", seed=2),
    "many_short": Workload("many_short", 256, 4, 512, 64, 64, "bf16", "mixed", 0.0, 1.0, 3.0, 1.5,
                           "zero", seed=3),
    "decode": Workload("decode", 128, 8, 1, 256, 512, "bf16", "std", 0.0, 1.0, 3.0, 1.5,
                       "normal_m_zero", seed=4, steps=256),
}


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of float32 values that are already bf16-exact."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not representable in bf16"
    return (u >> 16).astype(np.uint16)


def _logsigmoid(x: np.ndarray) -> np.ndarray:
    # log(1 / (1 + e^-x)) evaluated without overflow, in float64
    x = x.astype(np.float64)
    return np.where(x >= 0, -np.log1p(np.exp(-x)), x - np.log1p(np.exp(x)))


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    return round_to_bf16(x) if dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def _gates(rng, shape, w: Workload):
    ig = (rng.standard_normal(shape, dtype=np.float32) * np.float32(w.std_i)
          + np.float32(w.mean_i)).astype(np.float32)
    base = rng.standard_normal(shape, dtype=np.float32) * np.float32(w.std_f) + np.float32(w.mu_f)
    fg = _logsigmoid(base).astype(np.float32)
    if w.gate == "mixed":
        raw = (rng.standard_normal(shape, dtype=np.float32) + np.float32(0.5)).astype(np.float32)
        mask = rng.random(shape) < 0.5
        fg = np.where(mask, fg, raw).astype(np.float32)
    return ig, fg


def _state(rng, w: Workload):
    B, H, dqk, dv = w.B, w.H, w.d_qk, w.d_v
    if w.state == "zero":
        return None, None, None
    C0 = (rng.standard_normal((B, H, dv, dqk), dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    n0 = (rng.standard_normal((B, H, dqk), dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    if w.state == "normal_m_uniform":
        m0 = rng.uniform(0.0, 5.0, (B, H)).astype(np.float32)
    else:
        m0 = np.zeros((B, H), dtype=np.float32)
    return C0, n0, m0


def make_sequence(w: Workload) -> dict:
    """Inputs of one sequence workload (T axis present).  All arrays are
    float32 holding values exact in the storage dtype."""
    assert w.steps == 0
    rng = np.random.default_rng(w.seed)
    B, H, T, dqk, dv = w.B, w.H, w.T, w.d_qk, w.d_v
    q = _store(rng.standard_normal((B, H, T, dqk), dtype=np.float32), w.dtype)
    k = _store(rng.standard_normal((B, H, T, dqk), dtype=np.float32), w.dtype)
    v = _store(rng.standard_normal((B, H, T, dv), dtype=np.float32), w.dtype)
    ig, fg = _gates(rng, (B, H, T), w)
    C0, n0, m0 = _state(rng, w)
    return dict(q=q, k=k, v=v, i_pre=ig, f_pre=fg, C0=C0, n0=n0, m0=m0,
                qk_scale=float(1.0 / np.sqrt(dqk)), workload=w)


def decode_state(w: Workload, rng=None):
    """Initial state of a decode workload and the generator positioned after it."""
    rng = rng or np.random.default_rng(w.seed)
    C0, n0, m0 = _state(rng, w)
    return rng, C0, n0, m0


def decode_steps(w: Workload, rng, n_steps: int | None = None) -> Iterator[dict]:
    """Per-step inputs of a decode workload (no T axis), drawn after the state."""
    B, H, dqk, dv = w.B, w.H, w.d_qk, w.d_v
    for _ in range(w.steps if n_steps is None else n_steps):
        q = _store(rng.standard_normal((B, H, dqk), dtype=np.float32), w.dtype)
        k = _store(rng.standard_normal((B, H, dqk), dtype=np.float32), w.dtype)
        v = _store(rng.standard_normal((B, H, dv), dtype=np.float32), w.dtype)
        ig, fg = _gates(rng, (B, H), w)
        yield dict(q=q, k=k, v=v, i_pre=ig, f_pre=fg)


def output_gate_pre(w: Workload, dtype: str = "bf16") -> np.ndarray:
    """o~ [B,H,T,d_v] for the output stage, stored as dtype ("bf16" or "f32")."""
    rng = np.random.default_rng(w.seed + 7919)
    o = rng.standard_normal((w.B, w.H, w.T, w.d_v), dtype=np.float32) * np.float32(3.0)
    return _store(o, dtype)


def relative_errors(x: np.ndarray, y: np.ndarray, row_axes: int = 1):
    """Per-row normalised errors |x - y| / max_row |y| (rows = the last
    ``row_axes`` axes), returned as (max, mean).  Rows whose reference is all
    zero fall back to absolute error."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    axes = tuple(range(y.ndim - row_axes, y.ndim))
    scale = np.max(np.abs(y), axis=axes, keepdims=True)
    scale = np.where(scale > 0, scale, 1.0)
    err = np.abs(x - y) / scale
    if err.size == 0:
        return 0.0, 0.0
    return float(np.max(err)), float(np.mean(err))
