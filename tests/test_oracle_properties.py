"""Properties of the float64 oracle over random small shapes (CPU only).

Two facts the recurrence fixes whatever the inputs (xLSTM page, "mLSTM (matrix
LSTM)" eq. 1-3 with the "sLSTM" stabilizer):
  composition: running T1 + T2 tokens equals running T2 tokens from the state
               left by the first T1 (gauge-fixed: C~ e^{m}, n~ e^{m});
  gauge:       shifting the entering state to (C~ e^d, n~ e^d, m - d) leaves h~
               unchanged.
Hypothesis draws the shapes, the split point and the gate regime.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle


def draw_inputs(seed, B, H, T, dqk, dv, f_mu, i_sd):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, H, T, dqk))
    k = rng.normal(size=(B, H, T, dqk))
    v = rng.normal(size=(B, H, T, dv))
    ig = rng.normal(scale=i_sd, size=(B, H, T))
    fg = -np.log1p(np.exp(-rng.normal(loc=f_mu, size=(B, H, T))))
    C0 = rng.normal(scale=0.1, size=(B, H, dv, dqk))
    n0 = rng.normal(scale=0.1, size=(B, H, dqk))
    m0 = rng.uniform(0, 5, size=(B, H))
    return q, k, v, ig, fg, C0, n0, m0


shapes = st.tuples(st.integers(1, 2), st.integers(1, 2), st.integers(2, 24), st.integers(1, 6), st.integers(1, 5))


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), shape=shapes, cut=st.floats(0.05, 0.95), f_mu=st.floats(-2.0, 5.0),
       i_sd=st.floats(0.1, 8.0))
def test_composition(seed, shape, cut, f_mu, i_sd):
    B, H, T, dqk, dv = shape
    q, k, v, ig, fg, C0, n0, m0 = draw_inputs(seed, B, H, T, dqk, dv, f_mu, i_sd)
    T1 = max(1, min(T - 1, int(round(cut * T))))
    s = 0.7
    h, C, n, m = oracle.forward(q, k, v, ig, fg, C0, n0, m0, qk_scale=s)
    h1, C1, n1, m1 = oracle.forward(q[:, :, :T1], k[:, :, :T1], v[:, :, :T1], ig[:, :, :T1], fg[:, :, :T1],
                                    C0, n0, m0, qk_scale=s)
    h2, C2, n2, m2 = oracle.forward(q[:, :, T1:], k[:, :, T1:], v[:, :, T1:], ig[:, :, T1:], fg[:, :, T1:],
                                    C1, n1, m1, qk_scale=s)
    scale = np.abs(h).max() + 1e-300
    assert np.abs(np.concatenate([h1, h2], axis=2) - h).max() <= 1e-11 * scale
    assert np.abs(m2 - m).max() <= 1e-12 * max(1.0, np.abs(m).max())
    assert np.abs(C2 - C).max() <= 1e-11 * (np.abs(C).max() + 1e-300)
    assert np.abs(n2 - n).max() <= 1e-11 * (np.abs(n).max() + 1e-300)


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), shape=shapes, d=st.floats(-30.0, 30.0), f_mu=st.floats(-2.0, 5.0),
       i_sd=st.floats(0.1, 8.0))
def test_gauge(seed, shape, d, f_mu, i_sd):
    B, H, T, dqk, dv = shape
    q, k, v, ig, fg, C0, n0, m0 = draw_inputs(seed, B, H, T, dqk, dv, f_mu, i_sd)
    h, _, _, _ = oracle.forward(q, k, v, ig, fg, C0, n0, m0, qk_scale=1.0)
    e = np.exp(d)
    hg, _, _, _ = oracle.forward(q, k, v, ig, fg, C0 * e, n0 * e, m0 - d, qk_scale=1.0)
    assert np.abs(hg - h).max() <= 1e-9 * (np.abs(h).max() + 1e-300)
