"""Back-to-back chunkwise calls on grids of more blocks than SMs, the device status
checked after every call.

Every hand-off inside the tensor-core kernel is an mbarrier phase, and a consumer
that waits for a phase after the producer has completed the next one too waits
until its bounded wait gives up (XLSTM_ERR_TIMEOUT).  Whether a run reaches such
an interleaving depends on timing, so these tests repeat the call many times at
shapes with several blocks per SM wave (two blocks per SM at d_qk = 64, L = 64)
and with exact chunks in the mix.  Each call must also reproduce the first call's
output bit for bit.
"""
import ctypes

import pytest
import torch

from gpu_helpers import small_inputs, to_dev
from xlstm_mlstm_matrix_b200 import capi

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,T,dqk,dv,chunk,calls", [
    (64, 8, 512, 64, 64, 64, 150),     # 512 blocks, two per SM
    (64, 8, 512, 64, 64, 128, 60),
    (16, 8, 512, 128, 128, 64, 60),
    (8, 8, 512, 256, 512, 64, 30),     # 256 blocks of the 7B-like head shape
])
def test_repeated_calls_no_timeout(B, H, T, dqk, dv, chunk, calls):
    capi.load()
    lib = capi.load()
    inp = small_inputs(B, H, T, dqk, dv, "bf16", False, seed=dqk + chunk, gate="mixed")
    q, k, v = (to_dev(inp[n], "bf16") for n in ("q", "k", "v"))
    ig, fg = to_dev(inp["i_pre"], "f32"), to_dev(inp["f_pre"], "f32")
    h = torch.empty(B, H, T, dv, device="cuda")
    C = torch.empty(B, H, dv, dqk, device="cuda")
    n = torch.empty(B, H, dqk, device="cuda")
    m = torch.empty(B, H, device="cuda")
    desc = capi.make_desc(B, H, T, dqk, dv, capi.XLSTM_BF16, inp["qk_scale"], chunk)
    ws = torch.zeros(max(256, capi.xlstm_mlstm_workspace_size(desc)), device="cuda", dtype=torch.uint8)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    first = None
    for i in range(calls):
        st = lib.xlstm_mlstm_fwd_chunkwise(ctypes.byref(desc), P(q), P(k), P(v), P(ig), P(fg), None, None, None,
                                           P(h), P(C), P(n), P(m), P(ws), ctypes.c_size_t(ws.numel()), None)
        assert st == capi.XLSTM_OK, capi.xlstm_status_string(st)
        code, where = capi.xlstm_mlstm_workspace_status(ws)
        assert code == capi.XLSTM_OK, (i, code, where)
        if first is None:
            first = [t.clone() for t in (h, C, n, m)]
        elif i % 10 == 0:
            assert all(torch.equal(a, b) for a, b in zip(first, (h, C, n, m))), i
