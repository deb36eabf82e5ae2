"""Pins for the float64 oracle: checks against facts the pages and mathematics fix.

Each pin takes an oracle library handle, runs the oracle through
``oracle.forward``/``oracle.step`` and compares it with something that is not
the oracle: a closed form, a brute-force all-pairs sum, the unstabilized
recurrence, a textbook matmul, or a hand-derived case.  Each returns the
worst error it saw; ``PINS`` lists (name, function, tolerance).  The mutation
test feeds deliberately broken oracle builds through the same list and
requires that some pin fails for each.

Sources: xLSTM page (obsidian-dorae222.pages.dev), section "mLSTM (matrix
LSTM)" eq. (1)-(3), and the stabilizer of its "sLSTM" section; the page's
forward_recurrent listing for the step interface.
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_case(seed, B=2, H=2, T=12, dqk=5, dv=4, i_mu=0.0, i_sd=1.0, f_mu=2.0, f_sd=1.0,
               state=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, dqk))
    k = rng.standard_normal((B, H, T, dqk))
    v = rng.standard_normal((B, H, T, dv))
    ig = rng.normal(i_mu, i_sd, (B, H, T))
    x = rng.normal(f_mu, f_sd, (B, H, T))
    fg = -np.log1p(np.exp(-x))
    if state:
        C0 = rng.normal(0, 0.5, (B, H, dv, dqk))
        n0 = rng.normal(0, 0.5, (B, H, dqk))
        m0 = rng.uniform(-1, 3, (B, H))
    else:
        C0 = n0 = m0 = None
    return q, k, v, ig, fg, C0, n0, m0


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b) / (np.abs(b) + 1e-300))) if a.size else 0.0


def _scaled(a, b):
    """max |a-b| / max |b| over the whole array."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    s = float(np.max(np.abs(b))) if b.size else 1.0
    return float(np.max(np.abs(a - b))) / (s if s > 0 else 1.0) if a.size else 0.0


# --------------------------------------------------------------------------
# P1: brute-force quadratic (all-pairs) form.  Unrolling the recurrence gives,
# with F_t = sum_{r<=t} f~_r,  D_ts = F_t - F_s + i~_s,  g_t = F_t + m0,
# m_t = max(g_t, max_{s<=t} D_ts):
#   num_t = e^{g_t-m_t} C0 q_t + sum_{s<=t} e^{D_ts-m_t} (k_s.q_t) v_s
#   den_t = e^{g_t-m_t} n0.q_t + sum_{s<=t} e^{D_ts-m_t} (k_s.q_t)
#   h_t   = num_t / max(|den_t|, e^{-m_t})
# and the final state C_T = e^{g_T-m_T} C0 + sum_s e^{D_Ts-m_T} v_s k_s^T.
# --------------------------------------------------------------------------
def quadratic_form(q, k, v, ig, fg, C0, n0, m0, scale):
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    h = np.zeros((B, H, T, dv))
    Cf = np.zeros((B, H, dv, dqk))
    nf = np.zeros((B, H, dqk))
    mf = np.zeros((B, H))
    for b in range(B):
        for hh in range(H):
            c0 = np.zeros((dv, dqk)) if C0 is None else C0[b, hh]
            nn0 = np.zeros(dqk) if n0 is None else n0[b, hh]
            mm0 = 0.0 if m0 is None else m0[b, hh]
            F = np.cumsum(fg[b, hh])
            qs = scale * q[b, hh]
            for t in range(T):
                g = F[t] + mm0
                D = np.array([F[t] - F[s] + ig[b, hh, s] for s in range(t + 1)])
                mt = max(g, D.max())
                w = np.exp(D - mt)
                sc = k[b, hh, : t + 1] @ qs[t]
                num = math.exp(g - mt) * (c0 @ qs[t]) + (w * sc) @ v[b, hh, : t + 1]
                den = math.exp(g - mt) * (nn0 @ qs[t]) + np.sum(w * sc)
                h[b, hh, t] = num / max(abs(den), math.exp(-mt))
                if t == T - 1:
                    Cf[b, hh] = math.exp(g - mt) * c0 + (v[b, hh, : t + 1] * w[:, None]).T @ k[b, hh, : t + 1]
                    nf[b, hh] = math.exp(g - mt) * nn0 + w @ k[b, hh, : t + 1]
                    mf[b, hh] = mt
    return h, Cf, nf, mf


def pin_p1_quadratic(lib):
    worst = 0.0
    for seed, state, scale in [(1, False, 1.0), (2, True, 0.5), (3, True, 1.0)]:
        args = _rand_case(seed, T=16, state=state, i_mu=0.5, i_sd=2.0)
        ho, Co, no, mo = oracle.forward(*args, qk_scale=scale, lib=lib)
        hq, Cq, nq, mq = quadratic_form(*args, scale)
        worst = max(worst, _rel(ho, hq), _scaled(Co, Cq), _scaled(no, nq),
                    float(np.max(np.abs(mo - mq))))
    return worst


# --------------------------------------------------------------------------
# P2: the unstabilized recurrence, literally eq. (1)-(3) with raw gates
# f = e^{f~}, i = e^{i~} and the clamp max(|n^T q|, 1).  Stabilization must
# not change h, and the true state is e^{m} times the stabilized one.
# --------------------------------------------------------------------------
def unstabilized(q, k, v, ig, fg, C0, n0, m0, scale):
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    C = np.zeros((B, H, dv, dqk)) if C0 is None else C0 * np.exp(m0)[..., None, None]
    n = np.zeros((B, H, dqk)) if n0 is None else n0 * np.exp(m0)[..., None]
    h = np.zeros((B, H, T, dv))
    for t in range(T):
        f = np.exp(fg[:, :, t])[..., None, None]
        i = np.exp(ig[:, :, t])[..., None, None]
        C = f * C + i * np.einsum("bhr,bhc->bhrc", v[:, :, t], k[:, :, t])
        n = f[..., 0] * n + i[..., 0] * k[:, :, t]
        qs = scale * q[:, :, t]
        num = np.einsum("bhrc,bhc->bhr", C, qs)
        den = np.maximum(np.abs(np.einsum("bhc,bhc->bh", n, qs)), 1.0)
        h[:, :, t] = num / den[..., None]
    return h, C, n


def pin_p2_unstabilized(lib):
    worst = 0.0
    for seed, state in [(11, False), (12, True)]:
        args = _rand_case(seed, T=20, state=state)
        ho, Co, no, mo = oracle.forward(*args, qk_scale=0.7, lib=lib)
        hu, Cu, nu = unstabilized(*args, 0.7)
        worst = max(worst, _rel(ho, hu),
                    _rel(Co * np.exp(mo)[..., None, None], Cu),
                    _rel(no * np.exp(mo)[..., None], nu))
    return worst


# --------------------------------------------------------------------------
# P3: shifting every i~ by c.  From zero state C and n are linear in the input
# gates, so with the unstabilized numerator N_t and normaliser d_t at c = 0:
#   h_t(c) = e^c N_t / max(e^c |d_t|, 1).
# N_t, d_t come from the all-pairs sums (m_t-free form, small exponents).
# Where |d_t| >= 1 and c >= 0 this is plain invariance, h(c) = h(0).
# --------------------------------------------------------------------------
def _num_den_unstab(q, k, v, ig, fg, scale):
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    N = np.zeros((B, H, T, dv))
    d = np.zeros((B, H, T))
    for b in range(B):
        for hh in range(H):
            F = np.cumsum(fg[b, hh])
            for t in range(T):
                w = np.exp(F[t] - F[: t + 1] + ig[b, hh, : t + 1])
                sc = k[b, hh, : t + 1] @ (scale * q[b, hh, t])
                N[b, hh, t] = (w * sc) @ v[b, hh, : t + 1]
                d[b, hh, t] = np.sum(w * sc)
    return N, d


def pin_p3_shift(lib):
    worst = 0.0
    q, k, v, ig, fg, _, _, _ = _rand_case(21, T=14)
    N, d = _num_den_unstab(q, k, v, ig, fg, 1.0)
    for c in (-3.0, 5.0, 20.0):
        ho = oracle.forward(q, k, v, ig + c, fg, qk_scale=1.0, lib=lib)[0]
        expect = math.exp(c) * N / np.maximum(math.exp(c) * np.abs(d), 1.0)[..., None]
        worst = max(worst, _rel(ho, expect))
    # literal invariance where the clamp is inactive for both shifts
    q2 = 3.0 * q
    h0 = oracle.forward(q2, k, v, ig, fg, qk_scale=1.0, lib=lib)[0]
    hc = oracle.forward(q2, k, v, ig + 4.0, fg, qk_scale=1.0, lib=lib)[0]
    _, d2 = _num_den_unstab(q2, k, v, ig, fg, 1.0)
    sel = np.abs(d2) >= 1.0
    if np.any(sel):
        worst = max(worst, _rel(hc[sel], h0[sel]))
    return worst


# --------------------------------------------------------------------------
# P4: f~ = i~ = 0 from zero state is causal linear attention with the
# max(|.|, 1) normaliser: h = tril(Q K^T) V / max(|tril(Q K^T) 1|, 1).
# --------------------------------------------------------------------------
def pin_p4_linear_attention(lib):
    worst = 0.0
    rng = np.random.default_rng(31)
    B, H, T, dqk, dv = 2, 3, 24, 6, 5
    for scale in (1.0, 0.3):
        q = rng.standard_normal((B, H, T, dqk))
        k = rng.standard_normal((B, H, T, dqk))
        v = rng.standard_normal((B, H, T, dv))
        z = np.zeros((B, H, T))
        ho, Co, no, mo = oracle.forward(q, k, v, z, z, qk_scale=scale, lib=lib)
        S = np.tril(np.matmul(scale * q, np.swapaxes(k, -1, -2)))
        expect = np.matmul(S, v) / np.maximum(np.abs(S.sum(-1)), 1.0)[..., None]
        worst = max(worst, _rel(ho, expect))
        worst = max(worst, _scaled(Co, np.matmul(np.swapaxes(v, -1, -2), k)),
                    _scaled(no, k.sum(2)), float(np.max(np.abs(mo))))
    # where every |row sum| < 1 the normaliser is inactive: plain tril(QK^T) V
    q = 0.02 * rng.standard_normal((1, 1, 8, 4))
    k = 0.02 * rng.standard_normal((1, 1, 8, 4))
    v = rng.standard_normal((1, 1, 8, 3))
    z = np.zeros((1, 1, 8))
    ho = oracle.forward(q, k, v, z, z, lib=lib)[0]
    worst = max(worst, _rel(ho, np.tril(q @ np.swapaxes(k, -1, -2)) @ v))
    return worst


# --------------------------------------------------------------------------
# P5: a single token from zero state: h = v (k.q) / max(|k.q|, e^{-i~}),
# whatever f~ is; the state is i' v k^T with i' = e^{i~ - m}, m = max(f~, i~).
# --------------------------------------------------------------------------
def pin_p5_single_token(lib):
    rng = np.random.default_rng(41)
    B, H, dqk, dv = 3, 2, 7, 5
    q = rng.standard_normal((B, H, dqk))
    k = rng.standard_normal((B, H, dqk))
    v = rng.standard_normal((B, H, dv))
    ig = rng.normal(0, 3, (B, H))
    fg = rng.normal(0, 3, (B, H))
    Z = np.zeros((B, H, dv, dqk))
    z = np.zeros((B, H, dqk))
    h, C1, n1, m1 = oracle.step(q, k, v, ig, fg, Z, z, np.zeros((B, H)), qk_scale=1.0, lib=lib)
    kq = np.sum(k * q, -1)
    expect = v * (kq / np.maximum(np.abs(kq), np.exp(-ig)))[..., None]
    m = np.maximum(fg, ig)
    ip = np.exp(ig - m)
    return max(_rel(h, expect), float(np.max(np.abs(m1 - m))),
               _rel(C1, ip[..., None, None] * v[..., :, None] * k[..., None, :]),
               _rel(n1, ip[..., None] * k))


# --------------------------------------------------------------------------
# P6: reset (f~ = -1e4): every token forgets all history, so each follows P5
# on its own and m_t = i~_t.
# --------------------------------------------------------------------------
def pin_p6_reset(lib):
    q, k, v, ig, _, C0, n0, m0 = _rand_case(51, T=10, state=True)
    fg = np.full(ig.shape, -1.0e4)
    h, C, n, m = oracle.forward(q, k, v, ig, fg, C0, n0, m0, qk_scale=1.0, lib=lib)
    kq = np.sum(k * q, -1)
    expect = v * (kq / np.maximum(np.abs(kq), np.exp(-ig)))[..., None]
    return max(_rel(h, expect), float(np.max(np.abs(m - ig[:, :, -1]))),
               _rel(C, v[:, :, -1, :, None] * k[:, :, -1, None, :]))


# --------------------------------------------------------------------------
# P7: composition.  Running T1 + T2 tokens equals running T2 tokens from the
# state left by the first T1.
# --------------------------------------------------------------------------
def pin_p7_composition(lib):
    q, k, v, ig, fg, C0, n0, m0 = _rand_case(61, T=18, state=True)
    h, C, n, m = oracle.forward(q, k, v, ig, fg, C0, n0, m0, lib=lib)
    s = 7
    h1, C1, n1, m1 = oracle.forward(q[:, :, :s], k[:, :, :s], v[:, :, :s], ig[:, :, :s],
                                    fg[:, :, :s], C0, n0, m0, lib=lib)
    h2, C2, n2, m2 = oracle.forward(q[:, :, s:], k[:, :, s:], v[:, :, s:], ig[:, :, s:],
                                    fg[:, :, s:], C1, n1, m1, lib=lib)
    return max(_rel(np.concatenate([h1, h2], 2), h), _rel(C2, C), _rel(n2, n),
               float(np.max(np.abs(m2 - m))))


# --------------------------------------------------------------------------
# P8: gauge.  (C~ e^d, n~ e^d, m - d) is the same state: h is unchanged and
# the final states agree after the same re-gauging.
# --------------------------------------------------------------------------
def pin_p8_gauge(lib):
    q, k, v, ig, fg, C0, n0, m0 = _rand_case(71, T=9, state=True)
    h, C, n, m = oracle.forward(q, k, v, ig, fg, C0, n0, m0, lib=lib)
    worst = 0.0
    for d in (-2.5, 4.0):
        h2, C2, n2, m2 = oracle.forward(q, k, v, ig, fg, C0 * math.exp(d), n0 * math.exp(d),
                                        m0 - d, lib=lib)
        worst = max(worst, _rel(h2, h),
                    _rel(C2 * np.exp(m2 - m)[..., None, None], C),
                    _rel(n2 * np.exp(m2 - m)[..., None], n))
    return worst


# --------------------------------------------------------------------------
# P10: hand-worked case (tests/golden/hand_case_d1_T3.txt).
# --------------------------------------------------------------------------
def load_hand_case(path=None):
    path = path or os.path.join(GOLDEN, "hand_case_d1_T3.txt")
    vals = {}
    env = {"E": math.e, "__builtins__": {}}
    with open(path) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rhs = (s.strip() for s in line.split("=", 1))
            vals[key] = [float(eval(x, env)) for x in rhs.split(",")]
    return vals


def pin_p10_hand_case(lib):
    g = load_hand_case()
    T = len(g["q"])
    arr = lambda key: np.array(g[key]).reshape(1, 1, T, 1)
    h, C, n, m = oracle.forward(arr("q"), arr("k"), arr("v"), np.array(g["i"]).reshape(1, 1, T),
                                np.array(g["f"]).reshape(1, 1, T), qk_scale=1.0, lib=lib)
    return max(_rel(h.ravel(), g["h"]), _rel(C.ravel(), g["C"]), _rel(n.ravel(), g["n"]),
               float(abs(m.ravel()[0] - g["m"][0])))


def pin_p11_output_gate(lib):
    """Closed forms of h = sigmoid(o) h~ (page eq. 3): o = 0 halves h~; o = ln 3
    keeps three quarters; o and -o together give h~ back (sigmoid(o) +
    sigmoid(-o) = 1); o = +40 passes h~ through, o = -40 shuts it (below e^-40)."""
    rng = np.random.default_rng(11)
    h = rng.normal(size=(3, 50)) * np.exp(rng.uniform(-20, 20, size=(3, 50)))
    o = rng.normal(scale=3.0, size=h.shape)
    g = lambda oo: oracle.output_gate(h, np.broadcast_to(oo, h.shape), lib=lib)
    errs = [_rel(g(0.0), 0.5 * h), _rel(g(np.log(3.0)), 0.75 * h),
            _rel(oracle.output_gate(h, o, lib=lib) + oracle.output_gate(h, -o, lib=lib), h),
            _rel(g(40.0), h), float(np.max(np.abs(g(-40.0)) / np.abs(h))) * 1e-3]
    return max(errs)


PINS = [
    ("P1 quadratic form", pin_p1_quadratic, 1e-12),
    ("P2 unstabilized recurrence", pin_p2_unstabilized, 1e-10),
    ("P3 input-gate shift", pin_p3_shift, 1e-11),
    ("P4 linear attention", pin_p4_linear_attention, 1e-12),
    ("P5 single token", pin_p5_single_token, 1e-13),
    ("P6 reset", pin_p6_reset, 1e-13),
    ("P7 composition", pin_p7_composition, 1e-12),
    ("P8 gauge", pin_p8_gauge, 1e-12),
    ("P10 hand case", pin_p10_hand_case, 1e-14),
    ("P11 output gate", pin_p11_output_gate, 1e-15),
]
