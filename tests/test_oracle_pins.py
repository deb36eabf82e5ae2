"""The float64 oracle against its pins (CPU only).

See ``oracle_pins.py`` for what each pin compares with.  The mutation test
builds deliberately broken copies of the oracle source (a dropped decay, a
wrong sign, a transposed outer product, the unstabilized clamp, a missing
query scale, a stale stabilizer) and requires that at least one pin fails for
each: the pins are strong enough to catch a plausible mistake anywhere.
"""
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
from oracle_pins import PINS


@pytest.mark.parametrize("name,fn,tol", PINS, ids=[p[0] for p in PINS])
def test_pin(name, fn, tol):
    err = fn(oracle.load_library())
    assert err <= tol, f"{name}: {err:.3e} > {tol:.1e}"


def test_eq3_clamp_at_one_while_stabilizer_stays_zero():
    """xLSTM page, "mLSTM (matrix LSTM)" eq. 1-3 with the "sLSTM" stabilizer.
    With i~ = 0, f~ <= 0 and m_0 = 0 the stabilizer m_t = max(f~_t + m_{t-1}, i~_t)
    stays 0, so the stabilized gates are the raw ones (f = e^{f~}, i = 1) and the
    readout lower bound e^{-m_t} is the 1 of eq. 3.  Unrolling eq. 1-2 then gives
    C_t = sum_{s<=t} e^{F_t - F_s} v_s k_s^T and n_t = sum_{s<=t} e^{F_t - F_s} k_s
    (F_t the inclusive sum of f~), so
      h_t = sum_s e^{F_t-F_s} (q_t.k_s) v_s / max(|sum_s e^{F_t-F_s} q_t.k_s|, 1),
    evaluated here as one masked matrix product; the clamp is active on some
    tokens (the small weights at the start) and inactive on others."""
    rng = np.random.default_rng(5)
    dqk, dv, T = 6, 4, 12
    q = rng.standard_normal((T, dqk))
    k = rng.standard_normal((T, dqk))
    v = rng.standard_normal((T, dv))
    f = -rng.uniform(0.0, 1.0, T)
    i = np.zeros(T)
    F = np.cumsum(f)
    decay = np.tril(np.exp(F[:, None] - F[None, :]))
    A = (q @ k.T) * decay
    den = np.abs(A.sum(axis=1))
    assert np.any(den < 1.0) and np.any(den > 1.0), "both sides of the clamp must be exercised"
    h_closed = (A @ v) / np.maximum(den, 1.0)[:, None]
    C_closed = (v * np.exp(F[-1] - F)[:, None]).T @ k
    n_closed = np.exp(F[-1] - F) @ k
    h, C, n, m = oracle.forward(q[None, None], k[None, None], v[None, None], i[None, None], f[None, None])
    assert np.max(np.abs(h[0, 0] - h_closed)) < 1e-13
    assert np.max(np.abs(C[0, 0] - C_closed)) < 1e-13
    assert np.max(np.abs(n[0, 0] - n_closed)) < 1e-13
    assert m[0, 0] == 0.0


def test_empty_and_degenerate_shapes():
    z = np.zeros((2, 3, 0, 4))
    h, C, n, m = oracle.forward(z, z, np.zeros((2, 3, 0, 5)), np.zeros((2, 3, 0)),
                                np.zeros((2, 3, 0)))
    assert h.shape == (2, 3, 0, 5) and np.all(C == 0) and np.all(n == 0) and np.all(m == 0)
    C0 = np.ones((2, 3, 5, 4))
    _, C, _, m = oracle.forward(z, z, np.zeros((2, 3, 0, 5)), np.zeros((2, 3, 0)),
                                np.zeros((2, 3, 0)), C0, np.ones((2, 3, 4)), np.full((2, 3), 2.0))
    assert np.all(C == 1) and np.all(m == 2)


MUTANTS = {
    "no forget decay": ("Cr[c] = fp * Cr[c] + ip", "Cr[c] = Cr[c] + ip"),
    "stabilizer sign": ("exp(ft + m - m_new)", "exp(ft - m + m_new)"),
    "transposed outer product": ("ip * vt[r] * kt[c]", "ip * vt[c] * kt[r]"),
    "clamp at one": ("const double lower = exp(-m_new);", "const double lower = 1.0;"),
    "no query scale": ("qs[c] = j->qk_scale * qt[c]", "qs[c] = qt[c]"),
    "stale stabilizer": ("m = m_new;\n    }", "}"),
    "normaliser without gate": ("j->n[c] = fp * j->n[c] + ip * kt[c]", "j->n[c] = fp * j->n[c] + kt[c]"),
    "input gate unstabilized": ("const double ip = exp(it - m_new);", "const double ip = exp(it);"),
    "output gate sign": ("h_tilde[i] / (1.0 + exp(-o_pre[i]))", "h_tilde[i] / (1.0 + exp(o_pre[i]))"),
    "output gate missing": ("h_tilde[i] / (1.0 + exp(-o_pre[i]))", "h_tilde[i]"),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mlstm_oracle.c")).read()
    old, new = MUTANTS[mutant]
    assert old in src, f"mutation anchor not found: {old!r}"
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "mutant.c")
        with open(path, "w") as fh:
            fh.write(src.replace(old, new))
        lib_path = oracle.build(force=True, src=path, out=os.path.join(d, "libmutant.so"))
        lib = oracle.load_library(lib_path)
        failed = []
        for name, fn, tol in PINS:
            try:
                err = fn(lib)
            except Exception:  # a crash in a pin also counts as caught
                err = float("inf")
            if not (err <= tol):
                failed.append(name)
        assert failed, f"no pin caught mutant '{mutant}'"
