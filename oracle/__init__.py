"""float64 CPU oracle for the mLSTM forward with exponential gating.

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the benchmark's
CPU-baseline leg are the only users.  The CUDA library never imports, links or
calls anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``mlstm_oracle.c`` (plain C, one token at a time, in
the order of the recurrence on the xLSTM page's "mLSTM (matrix LSTM)" section,
eq. 1-3, with the stabilizer of its "sLSTM" section).  This module only
compiles that file with gcc and marshals numpy float64 arrays into it.

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, a brute-force quadratic form, the unstabilized recurrence and a hand
case, and the backward by ``tests/test_oracle_backward.py`` against central
finite differences of the forward and closed forms; none of those pins calls
back into this module's arithmetic other than the function it checks.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mlstm_oracle.c")
_LIB = os.path.join(_HERE, "libmlstm_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (IEEE float64; no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
             "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-o", tmp, src, "-lm", "-lpthread"])
        os.replace(tmp, out)
    return out


def _declare(lib):
    i64, dbl, ptr, cint = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
    lib.mlstm_oracle_forward.restype = cint
    lib.mlstm_oracle_forward.argtypes = [i64, i64, i64, i64, i64, dbl] + [ptr] * 12 + [cint]
    lib.mlstm_oracle_step.restype = cint
    lib.mlstm_oracle_step.argtypes = [i64, i64, i64, i64, dbl] + [ptr] * 12 + [cint]
    lib.mlstm_oracle_output_gate.restype = cint
    lib.mlstm_oracle_output_gate.argtypes = [i64, ptr, ptr, ptr]
    lib.mlstm_oracle_backward.restype = cint
    lib.mlstm_oracle_backward.argtypes = [i64, i64, i64, i64, i64, dbl] + [ptr] * 19 + [cint]
    return lib


def load_library(path: str | None = None):
    """Load (building if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def forward(q, k, v, i_pre, f_pre, C0=None, n0=None, m0=None, qk_scale=1.0,
            threads: int | None = None, lib=None):
    """Run the recurrence over a whole sequence.

    Shapes: q, k [B,H,T,dqk]; v [B,H,T,dv]; i_pre, f_pre [B,H,T];
    optional C0 [B,H,dv,dqk], n0 [B,H,dqk], m0 [B,H].
    Returns (h [B,H,T,dv], C [B,H,dv,dqk], n [B,H,dqk], m [B,H]) in float64.
    """
    q, k, v, ig, fg = (_f64(x) for x in (q, k, v, i_pre, f_pre))
    C0, n0, m0 = _f64(C0), _f64(n0), _f64(m0)
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape == (B, H, T, dv)
    assert ig.shape == (B, H, T) and fg.shape == (B, H, T)
    if C0 is not None:
        assert C0.shape == (B, H, dv, dqk)
    if n0 is not None:
        assert n0.shape == (B, H, dqk)
    if m0 is not None:
        assert m0.shape == (B, H)
    h = np.empty((B, H, T, dv))
    C = np.empty((B, H, dv, dqk))
    n = np.empty((B, H, dqk))
    m = np.empty((B, H))
    lib = lib or load_library()
    rc = lib.mlstm_oracle_forward(B, H, T, dqk, dv, float(qk_scale),
                                  _p(q), _p(k), _p(v), _p(ig), _p(fg),
                                  _p(C0), _p(n0), _p(m0),
                                  _p(h), _p(C), _p(n), _p(m),
                                  int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"mlstm_oracle_forward failed ({rc})")
    return h, C, n, m


def step(q, k, v, i_pre, f_pre, C, n, m, qk_scale=1.0, threads: int | None = None, lib=None):
    """One decode step.  q, k [B,H,dqk]; v [B,H,dv]; i_pre, f_pre [B,H];
    state C [B,H,dv,dqk], n [B,H,dqk], m [B,H].  Returns (h, C', n', m')."""
    q, k, v, ig, fg, C, n, m = (_f64(x) for x in (q, k, v, i_pre, f_pre, C, n, m))
    B, H, dqk = q.shape
    dv = v.shape[-1]
    h = np.empty((B, H, dv))
    C1 = np.empty((B, H, dv, dqk))
    n1 = np.empty((B, H, dqk))
    m1 = np.empty((B, H))
    lib = lib or load_library()
    rc = lib.mlstm_oracle_step(B, H, dqk, dv, float(qk_scale),
                               _p(q), _p(k), _p(v), _p(ig), _p(fg),
                               _p(C), _p(n), _p(m), _p(h), _p(C1), _p(n1), _p(m1),
                               int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"mlstm_oracle_step failed ({rc})")
    return h, C1, n1, m1


def backward(q, k, v, i_pre, f_pre, dh, C0=None, n0=None, m0=None, dC=None, dn=None, qk_scale=1.0,
             threads: int | None = None, lib=None):
    """Vector-Jacobian product of ``forward`` (mlstm_oracle.c states what is
    differentiated).  dh [B,H,T,dv] is the upstream gradient of h~; dC
    [B,H,dv,dqk] and dn [B,H,dqk] (optional) that of the final stored state.
    Returns dict(dq, dk, dv, di, df, dC0, dn0, dm0) in float64."""
    q, k, v, ig, fg, dh = (_f64(x) for x in (q, k, v, i_pre, f_pre, dh))
    C0, n0, m0, dC, dn = (_f64(x) for x in (C0, n0, m0, dC, dn))
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    assert dh.shape == (B, H, T, dv)
    out = dict(dq=np.empty((B, H, T, dqk)), dk=np.empty((B, H, T, dqk)), dv=np.empty((B, H, T, dv)),
               di=np.empty((B, H, T)), df=np.empty((B, H, T)), dC0=np.empty((B, H, dv, dqk)),
               dn0=np.empty((B, H, dqk)), dm0=np.empty((B, H)))
    lib = lib or load_library()
    rc = lib.mlstm_oracle_backward(B, H, T, dqk, dv, float(qk_scale), _p(q), _p(k), _p(v), _p(ig), _p(fg),
                                   _p(C0), _p(n0), _p(m0), _p(dh), _p(dC), _p(dn),
                                   *(_p(out[n]) for n in ("dq", "dk", "dv", "di", "df", "dC0", "dn0", "dm0")),
                                   int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"mlstm_oracle_backward failed ({rc})")
    return out


def output_gate(h_tilde, o_pre, lib=None):
    """h = sigmoid(o_pre) * h~, element by element (the page's eq. 3 output gate).
    h_tilde and o_pre of one shape; returns float64 of that shape."""
    h_tilde, o_pre = _f64(h_tilde), _f64(o_pre)
    assert h_tilde.shape == o_pre.shape
    h = np.empty(h_tilde.shape)
    lib = lib or load_library()
    if lib.mlstm_oracle_output_gate(h.size, _p(h_tilde), _p(o_pre), _p(h)) != 0:
        raise RuntimeError("mlstm_oracle_output_gate failed")
    return h
