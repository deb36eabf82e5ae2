"""The float64 oracle against its pins (CPU only).

See ``oracle_pins.py`` for what each pin compares with.  The mutation test
builds deliberately broken copies of the oracle source (a dropped decay, a
wrong sign, a transposed outer product, the unstabilized clamp, a missing
query scale, a stale stabilizer) and requires that at least one pin fails for
each: the pins are strong enough to catch a plausible mistake anywhere.
"""
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import oracle
from oracle_pins import PINS


@pytest.mark.parametrize("name,fn,tol", PINS, ids=[p[0] for p in PINS])
def test_pin(name, fn, tol):
    err = fn(oracle.load_library())
    assert err <= tol, f"{name}: {err:.3e} > {tol:.1e}"


def test_listing_step_agrees_when_stabilizer_stays_zero():
    """The page's forward_recurrent listing (identity projections, o_t = 1),
    restated in torch float64.  It carries the stabilized state but clamps
    with 1, so it matches the stabilized readout only while m_t = 0; inputs
    with i~ = 0 and f~ <= 0 keep m_t = 0 at every step."""
    g = torch.Generator().manual_seed(5)
    dqk, dv, T = 6, 4, 12
    qs = torch.randn(T, dqk, generator=g, dtype=torch.float64)
    ks = torch.randn(T, dqk, generator=g, dtype=torch.float64)
    vs = torch.randn(T, dv, generator=g, dtype=torch.float64)
    fs = -torch.rand(T, generator=g, dtype=torch.float64)
    its = torch.zeros(T, dtype=torch.float64)
    C = torch.zeros(dv, dqk, dtype=torch.float64)
    n = torch.zeros(dqk, dtype=torch.float64)
    m = torch.zeros((), dtype=torch.float64)
    hs = []
    for t in range(T):
        m_t = torch.max(fs[t] + m, its[t])
        f_t = torch.exp(fs[t] + m - m_t)
        i_t = torch.exp(its[t] - m_t)
        C = f_t * C + i_t * torch.outer(vs[t], ks[t])
        n = f_t * n + i_t * ks[t]
        hs.append((C @ qs[t]) / torch.clamp(torch.abs(n @ qs[t]), min=1.0))
        m = m_t
    h, Co, no, mo = oracle.forward(qs.numpy()[None, None], ks.numpy()[None, None],
                                   vs.numpy()[None, None], its.numpy()[None, None],
                                   fs.numpy()[None, None])
    assert np.max(np.abs(h[0, 0] - torch.stack(hs).numpy())) < 1e-13
    assert np.max(np.abs(Co[0, 0] - C.numpy())) < 1e-13
    assert abs(mo[0, 0]) == 0.0


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
