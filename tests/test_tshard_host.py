"""Sequences cut along T across ranks: the host plumbing on CPU (gloo, world 2).

xlstm_mlstm_matrix_b200.tshard orders the per-rank steps (summary of the
local stretch, one all_gather of the summaries, the chained entry state, the
local forward) and the collective.  Here each rank's three operations are the
float64 oracle's (the summary is the oracle run from a zero state with the
stabilizer at -inf; the chaining is the affine step of the xLSTM page's
"mLSTM (matrix LSTM)" eq. 1-2 in stabilized form), so the test checks the
plumbing: two gloo ranks, each holding half of every sequence, must give the
one-rank oracle's h~ and final state.
"""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

NEG = -1.0e300   # a stabilizer start below any reachable m (exp underflows to exactly 0)


class OracleOps:
    """The three per-rank operations in float64 on CPU torch tensors."""

    def summary(self, k, v, i_pre, f_pre):
        import oracle
        B, H, T, dqk = k.shape
        dv = v.shape[-1]
        z = np.zeros((B, H, T, dqk))
        _, C, n, m = oracle.forward(z, k.numpy(), v.numpy(), i_pre.numpy(), f_pre.numpy(),
                                    np.zeros((B, H, dv, dqk)), np.zeros((B, H, dqk)), np.full((B, H), NEG))
        F = f_pre.numpy().astype(np.float64).sum(-1)
        return torch.from_numpy(C), torch.from_numpy(n), torch.from_numpy(np.stack([F, m], -1))

    def combine(self, Cs, ns, Fs, state):
        S, B, H, dv, dqk = Cs.shape
        if state is None:
            C, n, m = np.zeros((B, H, dv, dqk)), np.zeros((B, H, dqk)), np.zeros((B, H))
        else:
            C, n, m = (x.numpy().astype(np.float64) for x in state)
        for g in range(S):
            F, ms = Fs[g, ..., 0].numpy(), Fs[g, ..., 1].numpy()
            mp_ = np.maximum(F + m, ms)
            a, b = np.exp(F + m - mp_), np.exp(ms - mp_)
            C = a[..., None, None] * C + b[..., None, None] * Cs[g].numpy()
            n = a[..., None] * n + b[..., None] * ns[g].numpy()
            m = mp_
        return torch.from_numpy(C), torch.from_numpy(n), torch.from_numpy(m)

    def forward(self, q, k, v, i_pre, f_pre, state, qk_scale):
        import oracle
        st = (None, None, None) if state is None else tuple(x.numpy() for x in state)
        h, C, n, m = oracle.forward(q.numpy(), k.numpy(), v.numpy(), i_pre.numpy(), f_pre.numpy(), *st,
                                    qk_scale=qk_scale)
        return torch.from_numpy(h), (torch.from_numpy(C), torch.from_numpy(n), torch.from_numpy(m))


def _inputs(state):
    from xlstm_mlstm_matrix_b200 import inputs
    w = inputs.WORKLOADS["tiny_fp32"].replace(B=2, H=2, T=96, d_qk=8, d_v=6, dtype="f32", gate="mixed",
                                              state="normal_m_uniform" if state else "zero", seed=12)
    return inputs.make_sequence(w)


def _worker(rank, world, port, state, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from xlstm_mlstm_matrix_b200 import tshard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs(state)
        T = inp["q"].shape[2]
        a, b = rank * T // world, (rank + 1) * T // world
        loc = [torch.from_numpy(inp[n][:, :, a:b].astype(np.float64)) for n in ("q", "k", "v", "i_pre", "f_pre")]
        st = None if inp["C0"] is None else tuple(torch.from_numpy(inp[n].astype(np.float64))
                                                  for n in ("C0", "n0", "m0"))
        h, (C, n, m) = tshard.fwd_tsharded(*loc, state=st, qk_scale=inp["qk_scale"], ops=OracleOps())
        out.put((rank, h.numpy(), C.numpy(), n.numpy(), m.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(state):
    import oracle
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, state, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=120) for _ in range(2)), key=lambda r: r[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    inp = _inputs(state)
    href, Cref, nref, mref = oracle.forward(inp["q"], inp["k"], inp["v"], inp["i_pre"], inp["f_pre"], inp["C0"],
                                            inp["n0"], inp["m0"], qk_scale=inp["qk_scale"])
    h = np.concatenate([r[1] for r in res], axis=2)
    np.testing.assert_allclose(h, href, rtol=1e-9, atol=1e-12 * np.abs(href).max())
    for _, _, C, n, m in res:   # every rank returns the final state, with the canonical m
        np.testing.assert_allclose(m, mref, rtol=0, atol=1e-9 * max(1.0, np.abs(mref).max()))
        g = np.exp(m - mref)
        np.testing.assert_allclose(C * g[..., None, None], Cref, rtol=1e-9, atol=1e-12 * np.abs(Cref).max())
        np.testing.assert_allclose(n * g[..., None], nref, rtol=1e-9, atol=1e-12 * np.abs(nref).max())


def test_tsharded_forward_gloo_world2_from_zero_state():
    _run(False)


def test_tsharded_forward_gloo_world2_from_given_state():
    _run(True)
