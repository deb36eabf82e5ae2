"""The output stage of the chunkwise call, against the oracle.

xlstm_mlstm_fwd_chunkwise_out applies h = sigmoid(o~) h~ (xLSTM page,
"mLSTM (matrix LSTM)" eq. 3, with o_t = sigmoid(o~_t) as in the page's
listing) and stores h as fp32 or bf16.  The oracle's h~ goes through the
oracle's output gate; the state outputs must equal the ungated call's.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import compare, fp32_row_tolerance, oracle_sequence, small_inputs, to_dev
from xlstm_mlstm_matrix_b200 import capi, inputs

pytestmark = pytest.mark.gpu


def run(inp, o_dtype, h_dtype, parallel=False, gate=True):
    w = inp["workload"]
    q, k, v = (to_dev(inp[n], w.dtype) for n in ("q", "k", "v"))
    ig, fg = to_dev(inp["i_pre"], "f32"), to_dev(inp["f_pre"], "f32")
    state = None if inp.get("C0") is None else tuple(to_dev(inp[n], "f32") for n in ("C0", "n0", "m0"))
    o_np = inputs.output_gate_pre(w, o_dtype)
    o = to_dev(o_np, o_dtype) if gate else None
    hdt = torch.bfloat16 if h_dtype == "bf16" else torch.float32
    B, H, T, dqk = q.shape
    desc = capi.make_desc(B, H, T, dqk, v.shape[-1], capi.XLSTM_BF16 if w.dtype == "bf16" else capi.XLSTM_F32,
                          inp["qk_scale"], 0)
    size = (capi.xlstm_mlstm_workspace_size_parallel if parallel else capi.xlstm_mlstm_workspace_size)(desc)
    ws = torch.zeros(max(256, size), device=q.device, dtype=torch.uint8)
    h, (C, n, m) = capi.fwd(q, k, v, ig, fg, state=state, qk_scale=inp["qk_scale"], workspace=ws, o_pre=o,
                            h_dtype=hdt)
    torch.cuda.synchronize()
    code, where = capi.xlstm_mlstm_workspace_status(ws)
    assert code == capi.XLSTM_OK, (code, where)
    assert h.dtype == hdt
    return (h.float().cpu().numpy(), C.cpu().numpy(), n.cpu().numpy(), m.cpu().numpy()), o_np


def reference(inp, o_np, gate=True):
    h, C, n, m = oracle_sequence(inp)
    return (oracle.output_gate(h, o_np) if gate else h), C, n, m


@pytest.mark.parametrize("h_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("o_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dtype,shape", [("bf16", (1, 2, 200, 256, 128)), ("bf16", (2, 1, 130, 128, 64)),
                                         ("bf16", (1, 2, 150, 64, 192)), ("f32", (1, 2, 100, 64, 48))])
def test_gated_output_matches_oracle(dtype, shape, o_dtype, h_dtype):
    inp = small_inputs(*shape, dtype, True, seed=sum(shape) + 1)
    got, o_np = run(inp, o_dtype, h_dtype)
    ref = reference(inp, o_np)
    # a bf16 h adds its own rounding (2^-9 of the element) to the kernel's error
    compare(got, ref, "bf16" if "bf16" in (dtype, h_dtype) else "f32", f"{dtype} {shape} o {o_dtype} h {h_dtype}")


@pytest.mark.parametrize("dqk", [64, 256])
def test_bf16_h_without_gate(dqk):
    """h_dtype bf16 alone: the h~ of the plain call, rounded to bf16."""
    inp = small_inputs(1, 2, 190, dqk, 128, "bf16", True, seed=dqk)
    got, _ = run(inp, "bf16", "bf16", gate=False)
    ref = reference(inp, None, gate=False)
    compare(got, ref, "bf16", "bf16 h, no gate")


def test_gated_output_exact_chunks():
    """Input-gate jumps that force the exact-chunk epilogue through the output stage."""
    inp = small_inputs(2, 2, 300, 128, 128, "bf16", True, seed=11, gate="std", mean_i=30.0, std_i=40.0)
    got, o_np = run(inp, "bf16", "f32")
    compare(got, reference(inp, o_np), "bf16", "gated exact chunks", row_tol=fp32_row_tolerance(inp))


def test_gated_output_segments():
    """A long sequence with few heads (parallel segments) through the output stage."""
    inp = small_inputs(1, 2, 2600, 128, 128, "bf16", True, seed=3)
    d = capi.make_desc(1, 2, 2600, 128, 128, capi.XLSTM_BF16, 1.0, 64)
    assert capi.xlstm_mlstm_workspace_size_parallel(d) > capi.xlstm_mlstm_workspace_size(d)
    got, o_np = run(inp, "bf16", "bf16", parallel=True)
    compare(got, reference(inp, o_np), "bf16", "gated segments")


def test_plain_call_unchanged_by_null_output_stage():
    """out == NULL (and an output stage with no gate and fp32 h) give the plain call's bits."""
    inp = small_inputs(1, 2, 200, 256, 128, "bf16", True, seed=5)
    w = inp["workload"]
    q, k, v = (to_dev(inp[n], "bf16") for n in ("q", "k", "v"))
    ig, fg = to_dev(inp["i_pre"], "f32"), to_dev(inp["f_pre"], "f32")
    h0, st0 = capi.fwd(q, k, v, ig, fg, qk_scale=inp["qk_scale"])
    h1, st1 = capi.fwd(q, k, v, ig, fg, qk_scale=inp["qk_scale"], h_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(h0, h1) and all(torch.equal(a, b) for a, b in zip(st0, st1))


@pytest.mark.parametrize("o_dtype,h_dtype", [("bf16", "bf16"), ("f32", "bf16"), ("bf16", "f32"), ("f32", "f32")])
def test_gated_output_split_launch(o_dtype, h_dtype):
    """More blocks than SMs with a partial last wave: the call splits its grid in two
    launches and gates the first launch's h~ while the second runs.  Against the
    oracle, and element for element against the ungated call's h~ (in h's dtype) gated
    here."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    heads = sms // 4 + 3          # 4 blocks per head (d_v = 512): a partial second wave
    inp = small_inputs(1, heads, 130, 64, 512, "bf16", True, seed=29)
    got, o_np = run(inp, o_dtype, h_dtype)
    compare(got, reference(inp, o_np), "bf16", f"gated split launch, o {o_dtype} h {h_dtype}")
    plain, _ = run(inp, o_dtype, h_dtype, gate=False)
    o = torch.from_numpy(o_np.astype(np.float32))
    h_tilde = torch.from_numpy(plain[0])
    gated = h_tilde / (1.0 + torch.exp(-o))
    if h_dtype == "bf16":
        # one bf16 unit of the larger of the two where the exponentials round differently
        want, rtol = gated.to(torch.bfloat16).float().numpy(), 2 ** -7
    else:
        want, rtol = gated.numpy(), 1e-6
    np.testing.assert_allclose(got[0], want, rtol=rtol, atol=1e-30)
    for a, b in zip(got[1:], plain[1:]):
        assert np.array_equal(a, b)
