"""The allocation-free chunkwise entry point (collected last on purpose).

xlstm_mlstm_fwd_chunkwise_noalloc serves callers that cannot allocate device
memory (a plug-in whose host framework owns every allocation, or a
latency-critical path that must not call cudaMalloc): it uses a fixed scratch
array inside the library instead of a caller workspace.  These tests call it
through the C ABI several times in a row, against the float64 oracle and bit
for bit against the regular entry point (which takes a caller workspace and
runs the same launch), and check that a call whose device wait timed out
leaves nothing behind for the next one.  The file is named so that pytest
collects it after every other test; it also passes on its own in a fresh
process.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import compare, oracle_sequence
from xlstm_mlstm_matrix_b200 import capi, inputs

pytestmark = pytest.mark.gpu


def _run(entry, w, tensors, ws=None, chunk=64):
    q, k, v, ig, fg, C0, n0, m0 = tensors
    h = torch.empty(w.B, w.H, w.T, w.d_v, device="cuda")
    C1 = torch.empty(w.B, w.H, w.d_v, w.d_qk, device="cuda")
    n1 = torch.empty(w.B, w.H, w.d_qk, device="cuda")
    m1 = torch.empty(w.B, w.H, device="cuda")
    desc = capi.make_desc(w.B, w.H, w.T, w.d_qk, w.d_v, capi.XLSTM_BF16, w.d_qk ** -0.5, chunk)
    if ws is None:
        st = entry(desc, q, k, v, ig, fg, C0, n0, m0, h, C1, n1, m1)
    else:
        st = entry(desc, q, k, v, ig, fg, C0, n0, m0, h, C1, n1, m1, ws, ws.numel())
    assert st == capi.XLSTM_OK, capi.xlstm_status_string(st)
    torch.cuda.synchronize()
    return [x.cpu().numpy() for x in (h, C1, n1, m1)]


def _case(d_qk, d_v):
    w = inputs.WORKLOADS["layer_7b"].replace(B=1, H=2, T=300, d_qk=d_qk, d_v=d_v,
                                             state="normal_m_uniform", seed=77)
    inp = inputs.make_sequence(w)
    dev = lambda x, bf: torch.from_numpy(x).cuda().to(torch.bfloat16) if bf else torch.from_numpy(x).cuda()
    tensors = [dev(inp[n], True) for n in ("q", "k", "v")] + \
              [dev(inp[n], False) for n in ("i_pre", "f_pre", "C0", "n0", "m0")]
    ws = torch.zeros(capi.xlstm_mlstm_workspace_size(capi.make_desc(1, 2, 300, d_qk, d_v)),
                     device="cuda", dtype=torch.uint8)
    return w, inp, tensors, ws


@pytest.mark.parametrize("d_qk,d_v,chunk", [(256, 512, 64), (128, 128, 64), (128, 128, 128)])
def test_noalloc_matches_oracle_and_workspace_entry_twice(d_qk, d_v, chunk):
    assert torch.cuda.is_available(), "needs a CUDA device"
    capi.load()
    w, inp, tensors, ws = _case(d_qk, d_v)
    ref = _run(capi.xlstm_mlstm_fwd_chunkwise, w, tensors, ws, chunk=chunk)
    oracle_ref = oracle_sequence(inp)
    for i in range(2):   # the shared scratch keeps the previous call's contents
        got = _run(capi.xlstm_mlstm_fwd_chunkwise_noalloc, w, tensors, chunk=chunk)
        assert capi.xlstm_mlstm_noalloc_status() == (capi.XLSTM_OK, 0)
        compare(got, oracle_ref, "bf16", f"noalloc call {i} against the oracle")
        for name, a, b in zip(("h", "C", "n", "m"), got, ref):
            assert np.array_equal(a, b), f"noalloc call {i}: {name} differs from the workspace entry"


def test_noalloc_call_after_a_timed_out_call_is_clean():
    """A call whose device wait gives up (one internal hand-off withheld through
    the test hook; the bounded wait ends the kernel) reports XLSTM_ERR_TIMEOUT
    in the shared array; the next call clears it and is exact again."""
    capi.load()
    w, inp, tensors, ws = _case(128, 128)
    ref = _run(capi.xlstm_mlstm_fwd_chunkwise, w, tensors, ws)
    capi.xlstm_mlstm_test_timeout_next(1)
    _run(capi.xlstm_mlstm_fwd_chunkwise_noalloc, w, tensors)
    code, where = capi.xlstm_mlstm_noalloc_status()
    assert code == capi.XLSTM_ERR_TIMEOUT and where > 0, (code, where)
    got = _run(capi.xlstm_mlstm_fwd_chunkwise_noalloc, w, tensors)
    assert capi.xlstm_mlstm_noalloc_status() == (capi.XLSTM_OK, 0)
    for name, a, b in zip(("h", "C", "n", "m"), got, ref):
        assert np.array_equal(a, b), f"after the timed-out call: {name} differs"
