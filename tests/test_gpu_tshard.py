"""Sequences cut along T, on one GPU: the summary and chaining calls of the C ABI
and the tshard plumbing with the CUDA operations, against the float64 oracle.

The ranks of a T-sharded run are emulated one after another in this process
(the exchange step returns the stretches' summaries computed beforehand; no
collective and no kernel waits on another), so the test needs one GPU.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import compare, to_dev
import oracle
from xlstm_mlstm_matrix_b200 import capi, inputs, tshard

pytestmark = pytest.mark.gpu

NEG = -1.0e300


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    capi.load()


def _case(dqk, dv, T, state=True, seed=5):
    w = inputs.WORKLOADS["layer_7b"].replace(B=1, H=2, T=T, d_qk=dqk, d_v=dv,
                                             state="normal_m_uniform" if state else "zero", seed=seed)
    return inputs.make_sequence(w)


def _dev(inp, a, b):
    return [to_dev(np.ascontiguousarray(inp[n][:, :, a:b]), "bf16") for n in ("q", "k", "v")] + \
           [to_dev(np.ascontiguousarray(inp[n][:, :, a:b]), "f32") for n in ("i_pre", "f_pre")]


@pytest.mark.parametrize("dqk,dv", [(128, 128), (256, 512), (64, 192)])
def test_segment_summary_matches_oracle(dqk, dv):
    inp = _case(dqk, dv, 192)
    q, k, v, ig, fg = _dev(inp, 0, 192)
    C, n, Fm = capi.summary(k, v, ig, fg)
    torch.cuda.synchronize()
    B, H = 1, 2
    _, Cr, nr, mr = oracle.forward(np.zeros((B, H, 192, dqk)), inp["k"], inp["v"], inp["i_pre"], inp["f_pre"],
                                   np.zeros((B, H, dv, dqk)), np.zeros((B, H, dqk)), np.full((B, H), NEG))
    Fm = Fm.cpu().numpy()
    Fr = inp["f_pre"].astype(np.float64).sum(-1)
    np.testing.assert_allclose(Fm[..., 0], Fr, rtol=1e-12, atol=1e-9)
    np.testing.assert_allclose(Fm[..., 1], mr, rtol=0, atol=1e-4 * max(1.0, np.abs(mr).max()))
    g = np.exp(Fm[..., 1] - mr)
    cmx, cmean = inputs.relative_errors(C.cpu().numpy() * g[..., None, None], Cr, row_axes=2)
    nmx, _ = inputs.relative_errors(n.cpu().numpy() * g[..., None], nr)
    assert cmx <= 2e-2 and cmean <= 4e-3 and nmx <= 2e-2, (cmx, cmean, nmx)


def test_summary_refuses_what_its_kernel_does_not_take():
    inp = _case(128, 128, 200)
    q, k, v, ig, fg = _dev(inp, 0, 200)   # T not a multiple of 64
    with pytest.raises(capi.XlstmError) as e:
        capi.summary(k, v, ig, fg)
    assert e.value.status == capi.XLSTM_ERR_UNSUPPORTED


@pytest.mark.parametrize("dqk,dv,R,state", [(128, 128, 3, True), (256, 512, 2, False), (64, 64, 4, True)])
def test_tsharded_forward_emulated_ranks(dqk, dv, R, state):
    T = R * 128
    inp = _case(dqk, dv, T, state=state, seed=dqk + R)
    st = None if inp["C0"] is None else tuple(to_dev(inp[n], "f32") for n in ("C0", "n0", "m0"))
    stretches = [_dev(inp, r * 128, (r + 1) * 128) for r in range(R)]
    sums = [capi.summary(*s[1:]) for s in stretches]
    hs, finals = [], []
    for r, s in enumerate(stretches):
        calls = iter(range(3))

        def gather(x, r=r, calls=calls):
            j = next(calls)   # C_seg, n_seg, F_m in that order
            parts = [sm[j] for sm in sums]
            parts[r] = x
            return parts, r

        h, fin = tshard.fwd_tsharded(*s, state=st, qk_scale=inp["qk_scale"], gather=gather)
        hs.append(h)
        finals.append(fin)
    torch.cuda.synchronize()
    ref = oracle.forward(inp["q"], inp["k"], inp["v"], inp["i_pre"], inp["f_pre"], inp["C0"], inp["n0"], inp["m0"],
                         qk_scale=inp["qk_scale"])
    got_h = torch.cat(hs, dim=2).cpu().numpy()
    for r, fin in enumerate(finals):
        got = (got_h, fin[0].cpu().numpy(), fin[1].cpu().numpy(), fin[2].cpu().numpy())
        compare(got, ref, "bf16", f"T-sharded over {R} stretches, final state on rank {r}")


def test_combine_with_no_summaries_copies_the_state():
    inp = _case(64, 64, 64)
    st = tuple(to_dev(inp[n], "f32") for n in ("C0", "n0", "m0"))
    empty_C = torch.empty(0, 1, 2, 64, 64, device="cuda")
    C, n, m = capi.combine(empty_C, torch.empty(0, 1, 2, 64, device="cuda"),
                           torch.empty(0, 1, 2, 2, device="cuda", dtype=torch.float64), st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(C.cpu().numpy(), inp["C0"])
    np.testing.assert_array_equal(n.cpu().numpy(), inp["n0"])
    np.testing.assert_array_equal(m.cpu().numpy(), inp["m0"])
