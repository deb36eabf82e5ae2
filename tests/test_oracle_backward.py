"""The float64 oracle's backward (vector-Jacobian product) against its pins (CPU).

What is differentiated (mlstm_oracle.c states it in full): the readout of the
xLSTM page's "mLSTM (matrix LSTM)" section, eq. 3 with the true states of
eq. 1-2, h_t = C_t q_t / max(|n_t^T q_t|, 1); the stabilizer m of the "sLSTM"
section only stores the states and is not differentiated.  The pins:
  - central finite differences of the forward oracle, element by element, on
    small cases (clamp active and inactive, with and without an initial state,
    with an upstream gradient on the final state);
  - a directional derivative over all inputs at once on a sequence of several
    64-token stretches (the backward's recomputation from checkpoints);
  - closed forms for one token from a zero state, on both sides of the clamp;
  - planted mistakes in copies of the oracle source, each caught by some pin.
The finite-difference loss is
  L = sum dh . h~ + sum dC . C~_T e^{m_T - m*} + sum dn . n~_T e^{m_T - m*}
with m* the unperturbed m_T: the final state enters through the true state
C_T = C~_T e^{m_T}, as it does for the next call of the recurrence.
"""
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle


def _case(seed, B=1, H=2, T=6, dqk=3, dv=2, i_mu=0.0, i_sd=1.0, f_mu=2.0, state=True, final=True):
    rng = np.random.default_rng(seed)
    c = dict(q=rng.standard_normal((B, H, T, dqk)), k=rng.standard_normal((B, H, T, dqk)),
             v=rng.standard_normal((B, H, T, dv)), i_pre=rng.normal(i_mu, i_sd, (B, H, T)),
             f_pre=-np.log1p(np.exp(-rng.normal(f_mu, 1.0, (B, H, T)))),
             dh=rng.standard_normal((B, H, T, dv)), qk_scale=0.7)
    if state:
        c.update(C0=rng.normal(0, 0.5, (B, H, dv, dqk)), n0=rng.normal(0, 0.5, (B, H, dqk)),
                 m0=rng.uniform(-1, 2, (B, H)))
    else:
        c.update(C0=None, n0=None, m0=None)
    if final:
        c.update(dC=rng.standard_normal((B, H, dv, dqk)), dn=rng.standard_normal((B, H, dqk)))
    else:
        c.update(dC=None, dn=None)
    return c


INPUTS = ("q", "k", "v", "i_pre", "f_pre", "C0", "n0", "m0")
GRAD_OF = dict(q="dq", k="dk", v="dv", i_pre="di", f_pre="df", C0="dC0", n0="dn0", m0="dm0")


def _loss(c, lib, m_ref=None):
    h, C, n, m = oracle.forward(c["q"], c["k"], c["v"], c["i_pre"], c["f_pre"], c["C0"], c["n0"], c["m0"],
                                qk_scale=c["qk_scale"], threads=1, lib=lib)
    L = np.sum(c["dh"] * h)
    if c["dC"] is not None:
        mr = m if m_ref is None else m_ref
        g = np.exp(m - mr)
        L += np.sum(c["dC"] * C * g[..., None, None]) + np.sum(c["dn"] * n * g[..., None])
    return L, m


def _grads(c, lib):
    return oracle.backward(c["q"], c["k"], c["v"], c["i_pre"], c["f_pre"], c["dh"], c["C0"], c["n0"], c["m0"],
                           c["dC"], c["dn"], qk_scale=c["qk_scale"], threads=1, lib=lib)


def fd_error(c, lib, eps=1e-6):
    """Largest |analytic - central difference| / (scale of that gradient), over
    every element of every input."""
    g = _grads(c, lib)
    _, m_ref = _loss(c, lib)
    worst = 0.0
    for name in INPUTS:
        x = c[name]
        if x is None:
            continue
        num = np.empty_like(x)
        flat, nflat = x.reshape(-1), num.reshape(-1)
        for i in range(flat.size):
            x0 = flat[i]
            flat[i] = x0 + eps
            lp, _ = _loss(c, lib, m_ref)
            flat[i] = x0 - eps
            lm, _ = _loss(c, lib, m_ref)
            flat[i] = x0
            nflat[i] = (lp - lm) / (2 * eps)
        ana = g[GRAD_OF[name]]
        scale = max(1.0, float(np.max(np.abs(num))))
        worst = max(worst, float(np.max(np.abs(ana - num))) / scale)
    return worst


FD_CASES = {
    "clamp inactive, initial state, final-state gradient": dict(seed=1),
    "clamp active early (small input gates), zero state": dict(seed=2, i_mu=-4.0, state=False),
    "large input-gate jumps": dict(seed=3, i_mu=3.0, i_sd=4.0),
    "weak forgetting, no final-state gradient": dict(seed=4, f_mu=-0.5, final=False),
}


def pin_fd(lib):
    return max(fd_error(_case(**kw), lib) for kw in FD_CASES.values())


def pin_directional(lib, eps=1e-6):
    """<grad, d> against (L(x + eps d) - L(x - eps d)) / 2 eps for one random
    direction d over all inputs, on T = 150 (three stretches of the sweep)."""
    c = _case(7, B=1, H=2, T=150, dqk=6, dv=5, i_mu=-1.0)
    g = _grads(c, lib)
    _, m_ref = _loss(c, lib)
    rng = np.random.default_rng(70)
    d = {n: rng.standard_normal(c[n].shape) for n in INPUTS}
    base = {n: c[n].copy() for n in INPUTS}
    for n in INPUTS:
        c[n] = base[n] + eps * d[n]
    lp, _ = _loss(c, lib, m_ref)
    for n in INPUTS:
        c[n] = base[n] - eps * d[n]
    lm, _ = _loss(c, lib, m_ref)
    for n in INPUTS:
        c[n] = base[n]
    fd = (lp - lm) / (2 * eps)
    ana = sum(float(np.sum(g[GRAD_OF[n]] * d[n])) for n in INPUTS)
    return abs(ana - fd) / max(1.0, abs(fd))


def pin_single_token(lib):
    """One token from a zero state, f~ + 0 < i~ so that m = i~ and i' = 1:
    h~ = v (k.q) / max(|k.q|, e^{-i~}) with q scaled.  Above the clamp h~ = v sign(k.q),
    whose only gradient is dv = dh sign(k.q); on the clamp h~ = v (k.q) e^{i~}:
    dv = dh (k.q) e^{i~}, dq = s e^{i~} (dh.v) k, dk = s e^{i~} (dh.v) q, di~ = (dh.v)(k.q) e^{i~}."""
    worst = 0.0
    branches = []
    for i_val, q_mul in ((0.5, 1.0), (0.5, 1e-3)):   # q along k: |k.q| above, then below e^{-i~}
        rng = np.random.default_rng(11)
        k = rng.standard_normal((1, 1, 1, 4))
        q = (k + 0.3 * rng.standard_normal((1, 1, 1, 4))) * q_mul
        v = rng.standard_normal((1, 1, 1, 3))
        dh = rng.standard_normal((1, 1, 1, 3))
        s = 0.9
        ig, fg = np.full((1, 1, 1), i_val), np.full((1, 1, 1), -2.0)
        g = oracle.backward(q, k, v, ig, fg, dh, qk_scale=s, threads=1, lib=lib)
        kq = s * float(np.sum(k * q))
        dhv = float(np.sum(dh * v))
        branches.append(abs(kq) > np.exp(-i_val))
        if branches[-1]:
            exp = dict(dv=dh * np.sign(kq), dq=0 * q, dk=0 * k, di=np.zeros((1, 1, 1)))
        else:
            e = np.exp(i_val)
            exp = dict(dv=dh * kq * e, dq=s * e * dhv * k, dk=s * e * dhv * q, di=np.full((1, 1, 1), dhv * kq * e))
        exp["df"] = np.zeros((1, 1, 1))   # the zero state carries nothing to forget
        for n, x in exp.items():
            worst = max(worst, float(np.max(np.abs(g[n] - x))))
    assert branches == [True, False], "both sides of the clamp must be exercised"
    return worst


PINS = [("finite differences", pin_fd, 1e-6), ("directional derivative", pin_directional, 1e-6),
        ("single token closed form", pin_single_token, 1e-12)]


@pytest.mark.parametrize("name,fn,tol", PINS, ids=[p[0] for p in PINS])
def test_backward_pin(name, fn, tol):
    err = fn(oracle.load_library())
    assert err <= tol, f"{name}: {err:.3e} > {tol:.1e}"


MUTANTS = {
    "no normaliser term": ("const double ds = (fabs(s) > lower) ? -(g / den) * (s > 0.0 ? 1.0 : -1.0) : 0.0;",
                           "const double ds = 0.0;"),
    "normaliser sign": ("-(g / den) * (s > 0.0 ? 1.0 : -1.0)", "(g / den) * (s > 0.0 ? 1.0 : -1.0)"),
    "adjoint not decayed": ("for (int64_t x = 0; x < csz; ++x) dC[x] *= fp;", ""),
    "input gate via v": ("di += kt[c] * j->dk[t * dqk + c];", "di += 0.0;"),
    "forget gate on the new state": ("for (int64_t x = 0; x < csz; ++x) df += dC[x] * Cp[x];",
                                     "for (int64_t x = 0; x < csz; ++x) df += dC[x] * Ct[x];"),
    "dq without the normaliser": ("double acc = ds * nt[c];", "double acc = 0.0;"),
    "dk without dn": ("double acc = dn[c];\n                for (int64_t r = 0; r < dv; ++r) acc += dC[r * dqk + c] * vt[r];",
                      "double acc = 0.0;\n                for (int64_t r = 0; r < dv; ++r) acc += dC[r * dqk + c] * vt[r];"),
    "initial m gradient": ("dm += dC[x] * (j->C0 ? j->C0[x] : 0.0);", "dm += 0.0;"),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_backward_pins_catch_planted_mistake(mutant):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mlstm_oracle.c")).read()
    old, new = MUTANTS[mutant]
    assert old in src, f"mutation anchor not found: {old!r}"
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "mutant.c")
        with open(path, "w") as fh:
            fh.write(src.replace(old, new))
        lib = oracle.load_library(oracle.build(force=True, src=path, out=os.path.join(d, "libmutant.so")))
        failed = []
        for name, fn, tol in PINS:
            try:
                err = fn(lib)
            except Exception:
                err = float("inf")
            if not (err <= tol):
                failed.append(name)
        assert failed, f"no pin caught mutant '{mutant}'"
