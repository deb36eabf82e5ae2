"""The allocation-free chunkwise entry point (collected last on purpose).

xlstm_mlstm_fwd_chunkwise_noalloc serves callers that cannot allocate device
memory (a plug-in whose host framework owns every allocation, or a
latency-critical path that must not call cudaMalloc): it uses a fixed scratch
array inside the library instead of a caller workspace.  This test calls it
twice in a row through the C ABI and checks both results against the regular
entry point, which takes a caller workspace.  The file is named so that pytest
collects it after every other test; it also passes on its own in a fresh
process.
"""
import numpy as np
import pytest
import torch

from xlstm_mlstm_matrix_b200 import capi, inputs

pytestmark = pytest.mark.gpu


def _run(entry, w, tensors, ws=None):
    q, k, v, ig, fg, C0, n0, m0 = tensors
    h = torch.empty(w.B, w.H, w.T, w.d_v, device="cuda")
    C1 = torch.empty(w.B, w.H, w.d_v, w.d_qk, device="cuda")
    n1 = torch.empty(w.B, w.H, w.d_qk, device="cuda")
    m1 = torch.empty(w.B, w.H, device="cuda")
    desc = capi.make_desc(w.B, w.H, w.T, w.d_qk, w.d_v, capi.XLSTM_BF16, w.d_qk ** -0.5, 64)
    if ws is None:
        st = entry(desc, q, k, v, ig, fg, C0, n0, m0, h, C1, n1, m1)
    else:
        st = entry(desc, q, k, v, ig, fg, C0, n0, m0, h, C1, n1, m1, ws, ws.numel())
    assert st == capi.XLSTM_OK, capi.xlstm_status_string(st)
    torch.cuda.synchronize()
    return [x.cpu().numpy() for x in (h, C1, n1, m1)]


@pytest.mark.parametrize("d_qk,d_v", [(256, 512), (128, 128)])
def test_noalloc_matches_workspace_entry_twice(d_qk, d_v):
    assert torch.cuda.is_available(), "needs a CUDA device"
    capi.load()
    w = inputs.WORKLOADS["layer_7b"].replace(B=1, H=2, T=300, d_qk=d_qk, d_v=d_v,
                                             state="normal_m_uniform", seed=77)
    inp = inputs.make_sequence(w)
    dev = lambda x, bf: torch.from_numpy(x).cuda().to(torch.bfloat16) if bf else torch.from_numpy(x).cuda()
    tensors = [dev(inp[n], True) for n in ("q", "k", "v")] + \
              [dev(inp[n], False) for n in ("i_pre", "f_pre", "C0", "n0", "m0")]
    ws = torch.zeros(capi.xlstm_mlstm_workspace_size(capi.make_desc(1, 2, 300, d_qk, d_v)),
                     device="cuda", dtype=torch.uint8)
    ref = _run(capi.xlstm_mlstm_fwd_chunkwise, w, tensors, ws)
    for _ in range(2):   # the shared scratch keeps the previous call's contents
        got = _run(capi.xlstm_mlstm_fwd_chunkwise_noalloc, w, tensors)
        mx, mean = inputs.relative_errors(got[0], ref[0])
        assert mx <= 2e-2 and mean <= 4e-3, (mx, mean)
        g = np.exp(got[3].astype(np.float64) - ref[3])
        cmx, _ = inputs.relative_errors(got[1] * g[..., None, None], ref[1], row_axes=2)
        assert cmx <= 2e-2 and np.max(np.abs(got[3] - ref[3])) <= 1e-4
