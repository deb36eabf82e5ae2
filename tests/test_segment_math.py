"""The segment decomposition behind the segment-parallel chunkwise path, checked
on CPU with the float64 oracle (no GPU, no CUDA code).

Over a stretch of tokens the recurrence (xLSTM page, "mLSTM (matrix LSTM)"
eq. 1-2, stabilizer of the "sLSTM" section) maps the entering state to the
leaving one affinely.  A segment's summary is the state it leaves from a zero
state whose stabilizer starts at -inf: (C_seg, n_seg) in the gauge m_seg, with
F the segment's summed log forget gates.  Chaining
    m' = max(F + m, m_seg),  C' = e^{F+m-m'} C + e^{m_seg-m'} C_seg  (n likewise)
must give the state the recurrence reaches at every segment boundary, and
running the next segment from it must give the same h~ as one long run.
"""
import numpy as np
import pytest

import oracle
from xlstm_mlstm_matrix_b200 import inputs

NEG = -1.0e300   # a stabilizer start below any reachable m (exp underflows to exactly 0)


def seq(T, gate="std", mean_i=0.0, std_i=1.0, seed=0):
    w = inputs.WORKLOADS["tiny_fp32"].replace(B=1, H=2, T=T, d_qk=8, d_v=6, dtype="f32", gate=gate,
                                              mean_i=mean_i, std_i=std_i, state="normal_m_uniform", seed=seed)
    return inputs.make_sequence(w)


def part(inp, a, b):
    return [inp[n][:, :, a:b] for n in ("q", "k", "v", "i_pre", "f_pre")]


def gauge_fixed(C, m, m_ref):
    return C * np.exp(m - m_ref)[..., None, None]


@pytest.mark.parametrize("gate,mean_i,std_i", [("std", 0.0, 1.0), ("mixed", 0.0, 1.0), ("std", 30.0, 40.0)])
def test_chained_summaries_reproduce_the_recurrence(gate, mean_i, std_i):
    inp = seq(96, gate, mean_i, std_i, seed=4)
    cuts = [0, 20, 41, 70, 96]
    s = inp["qk_scale"]
    h_full, C_full, n_full, m_full = oracle.forward(*part(inp, 0, 96), inp["C0"], inp["n0"], inp["m0"], qk_scale=s)
    C, n, m = inp["C0"].astype(np.float64), inp["n0"].astype(np.float64), inp["m0"].astype(np.float64)
    hs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        # the segment run from the chained entry state: its h~ and end state
        h_seg, C_end, n_end, m_end = oracle.forward(*part(inp, a, b), C, n, m, qk_scale=s)
        hs.append(h_seg)
        # the segment's summary from a zero state with the stabilizer at -inf
        zC, zn = np.zeros_like(C), np.zeros_like(n)
        _, Cs, ns, ms = oracle.forward(*part(inp, a, b), zC, zn, np.full_like(m, NEG), qk_scale=s)
        F = inp["f_pre"][:, :, a:b].astype(np.float64).sum(-1)
        mp = np.maximum(F + m, ms)
        C = np.exp(F + m - mp)[..., None, None] * C + np.exp(ms - mp)[..., None, None] * Cs
        n = np.exp(F + m - mp)[..., None] * n + np.exp(ms - mp)[..., None] * ns
        m = mp
        # the chained state is the recurrence's state at the boundary, canonical m included
        np.testing.assert_allclose(m, m_end, rtol=0, atol=1e-9 * max(1.0, np.abs(m_end).max()))
        np.testing.assert_allclose(gauge_fixed(C, m, m_end), C_end, rtol=1e-9, atol=1e-12 * np.abs(C_end).max())
        np.testing.assert_allclose(n * np.exp(m - m_end)[..., None], n_end, rtol=1e-9, atol=1e-12 * np.abs(n_end).max())
    # the pieces' h~ is the long run's h~
    np.testing.assert_allclose(np.concatenate(hs, axis=2), h_full, rtol=1e-9, atol=1e-12 * np.abs(h_full).max())
    np.testing.assert_allclose(m, m_full, rtol=0, atol=1e-9 * max(1.0, np.abs(m_full).max()))


def test_summary_gauge_is_the_segment_stabilizer():
    """m_seg = F + max_t (i~_t - F_t) with F_t counted from the segment start."""
    inp = seq(40, seed=9)
    s = inp["qk_scale"]
    z = np.zeros((1, 2, 6, 8))
    _, _, _, ms = oracle.forward(*part(inp, 0, 40), z, np.zeros((1, 2, 8)), np.full((1, 2), NEG), qk_scale=s)
    f = inp["f_pre"].astype(np.float64)
    Ft = np.cumsum(f, axis=-1)
    u = inp["i_pre"].astype(np.float64) - Ft
    np.testing.assert_allclose(ms, Ft[..., -1] + u.max(-1), rtol=1e-12)
