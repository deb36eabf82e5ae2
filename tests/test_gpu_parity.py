"""GPU parity: the three C-ABI calls against the float64 oracle (needs a B200).

Small shapes run the oracle on every head; the full-size workloads run the GPU
on the whole input, in the launch configuration the benchmark times, and the
oracle on sampled heads (each head is an independent recurrence).
Tolerances (per-row normalised relative error): fp32 inputs 1e-4; bf16 inputs
2e-2 max and 4e-3 mean; m within 1e-4 max(1, |m|); states compared after
fixing the gauge (C e^{m_gpu - m_ref}).
"""
import numpy as np
import pytest
import torch

from gpu_helpers import (compare, fp32_row_tolerance, gpu_sequence, oracle_sequence, select_heads, small_inputs,
                         to_dev)
import oracle
from xlstm_mlstm_matrix_b200 import capi, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    capi.load()


SMALL = [  # B, H, T, dqk, dv
    (1, 2, 1, 16, 16),
    (2, 2, 17, 32, 48),
    (1, 3, 100, 64, 64),
    (2, 1, 130, 128, 32),
    (1, 1, 64, 16, 128),
    (1, 2, 200, 256, 64),
    # shapes the tensor-core kernel takes for bf16 (d_qk in {64,128,256}, d_v % 64 == 0;
    # a d_v that is an odd multiple of 64 ends in a half-filled 128-row value slice)
    (1, 2, 200, 64, 128),
    (2, 1, 130, 128, 256),
    (1, 1, 333, 256, 128),
    (1, 2, 64, 256, 512),
    (2, 2, 1, 128, 128),
    (1, 1, 65, 64, 384),
    (2, 1, 130, 128, 192),
    (3, 2, 71, 256, 320),
    # the largest head dims the ABI takes, and odd ones (CUDA-core kernels; more than one
    # normaliser column per thread in the recurrent kernel)
    (1, 1, 70, 512, 32),
    (1, 2, 40, 384, 48),
    (2, 1, 33, 80, 16),
]
TC_SHAPES = [sh for sh in SMALL if sh[3] in (64, 128, 256) and sh[4] % 64 == 0]


@pytest.mark.parametrize("kind", ["chunkwise", "recurrent"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("state", [False, True])
def test_small_shapes(kind, dtype, shape, state):
    inp = small_inputs(*shape, dtype, state, seed=sum(shape))
    for scale in (1.0, shape[3] ** -0.5):
        got = gpu_sequence(inp, kind, qk_scale=scale)
        ref = oracle_sequence(inp, qk_scale=scale)
        compare(got, ref, dtype, f"{kind} {dtype} {shape} state={state} scale={scale:.3f}")


def test_tensor_core_path_selected():
    """bf16 inputs of the supported head sizes run on the tcgen05 kernel."""
    for B, H, T, dqk, dv in TC_SHAPES:
        d = capi.make_desc(B, H, T, dqk, dv, capi.XLSTM_BF16, 1.0, 64)
        assert capi.xlstm_mlstm_chunkwise_kernel(d) == "tcgen05", (B, H, T, dqk, dv)
        d.qkv_dtype = capi.XLSTM_F32
        assert capi.xlstm_mlstm_chunkwise_kernel(d) == "simt"
    d = capi.make_desc(8, 8, 4096, 256, 512, capi.XLSTM_BF16, 1 / 16, 64)
    assert capi.xlstm_mlstm_chunkwise_kernel(d) == "tcgen05"


@pytest.mark.parametrize("dv", [64, 128])
def test_chunk_size_invariance(dv):
    """The chunk length is an evaluation order, not part of the method (the pages
    give no chunkwise form): every supported length must give the recurrence's
    result.  fp32 inputs run on the CUDA-core kernel at L in {16, 32, 64, 128}; bf16
    inputs run on the tensor-core kernel at L in {64, 128} (checked against the
    oracle and against each other), and are compared with the CUDA-core kernel at
    L in {16, 32} on the same (bf16-exact) values."""
    f32 = small_inputs(2, 2, 203, 64, dv, "f32", True, seed=3)
    bf = small_inputs(2, 2, 203, 64, dv, "bf16", True, seed=3)
    outs = {}
    ref_f = oracle_sequence(f32)
    for L in (16, 32, 64, 128):
        outs[L] = gpu_sequence(f32, "chunkwise", chunk=L)
        compare(outs[L], ref_f, "f32", f"fp32 L={L}")
    for L in (16, 32, 128):
        mx, _ = inputs.relative_errors(outs[L][0], outs[64][0])
        assert mx <= 1e-4, f"fp32 chunk {L} vs 64: {mx:.2e}"
    B, H, T, dqk = bf["q"].shape
    d = capi.make_desc(B, H, T, dqk, dv, capi.XLSTM_BF16, bf["qk_scale"], 64)
    assert capi.xlstm_mlstm_chunkwise_kernel(d) == "tcgen05"
    got = gpu_sequence(bf, "chunkwise", chunk=64)
    ref_b = oracle_sequence(bf)
    compare(got, ref_b, "bf16", "bf16 tcgen05 L=64")
    d.chunk = 128
    assert capi.xlstm_mlstm_chunkwise_kernel(d) == "tcgen05"
    got128 = gpu_sequence(bf, "chunkwise", chunk=128)
    compare(got128, ref_b, "bf16", "bf16 tcgen05 L=128")
    mx, mean = inputs.relative_errors(got128[0], got[0])
    assert mx <= 2e-2 and mean <= 4e-3, f"bf16 tcgen05 L=128 vs L=64: {mx:.2e} / {mean:.2e}"
    # the bf16 values as fp32 inputs through the CUDA-core kernel at the other lengths
    same = dict(bf, workload=bf["workload"].replace(dtype="f32"))
    for L in (16, 32):
        other = gpu_sequence(same, "chunkwise", chunk=L)
        mx, mean = inputs.relative_errors(got[0], other[0])
        assert mx <= 2e-2 and mean <= 4e-3, f"bf16 tcgen05 L=64 vs CUDA-core L={L}: {mx:.2e} / {mean:.2e}"


@pytest.mark.parametrize("gate,mean_i,std_i", [("mixed", 0.0, 1.0), ("std", 4.0, 6.0), ("std", 30.0, 40.0)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128])
def test_stabilizer_stress(gate, mean_i, std_i, dtype, dv):
    """Positive log-forget gates (exp(f~) > 1), large input-gate jumps, and
    jumps far beyond the tensor-core kernel's lazy-rescale threshold."""
    inp = small_inputs(2, 2, 300, 64, dv, dtype, True, seed=11, gate=gate, mean_i=mean_i, std_i=std_i)
    ref = oracle_sequence(inp)
    tol = fp32_row_tolerance(inp)
    for kind in ("chunkwise", "recurrent"):
        compare(gpu_sequence(inp, kind), ref, dtype, f"{kind} {gate}", row_tol=tol)


@pytest.mark.parametrize("dqk,dv", [(64, 128), (256, 128), (64, 64)])
def test_exact_and_fast_chunks_alternating_repeated(dqk, dv):
    """Input-gate jumps far beyond the fast path's range make exact and fast chunks
    alternate; the hand-offs between the two kinds of chunk must hold however the
    warps are timed, so the same call runs many times and every run must finish
    with a clean device status and the same result."""
    inp = small_inputs(2, 2, 300, dqk, dv, "bf16", True, seed=11, gate="std", mean_i=30.0, std_i=40.0)
    ref = oracle_sequence(inp)
    first = gpu_sequence(inp, "chunkwise")
    compare(first, ref, "bf16", "alternating exact/fast", row_tol=fp32_row_tolerance(inp))
    for _ in range(24):
        got = gpu_sequence(inp, "chunkwise")   # asserts a clean device status
        np.testing.assert_array_equal(got[0], first[0])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128])
def test_reset_gates(dtype, dv):
    """f~ = -1e4 at every token: each token forgets everything before it."""
    inp = small_inputs(1, 2, 150, 64, dv, dtype, True, seed=5)
    inp["f_pre"] = np.full_like(inp["f_pre"], -1.0e4)
    ref = oracle_sequence(inp)
    for kind in ("chunkwise", "recurrent"):
        compare(gpu_sequence(inp, kind), ref, dtype, f"{kind} reset")


def test_empty_sequence_passes_state_through():
    inp = small_inputs(2, 2, 0, 32, 32, "bf16", True)
    for kind in ("chunkwise", "recurrent"):
        h, C, n, m = gpu_sequence(inp, kind)
        assert h.shape == (2, 2, 0, 32)
        np.testing.assert_array_equal(C, inp["C0"])
        np.testing.assert_array_equal(n, inp["n0"])
        np.testing.assert_array_equal(m, inp["m0"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [32, 256])
def test_composition_across_calls(dtype, dv):
    """run(T1+T2) == run(T2, state=run(T1).state), mixing call types."""
    inp = small_inputs(2, 2, 150, 64, dv, dtype, True, seed=9)
    ref = oracle_sequence(inp)
    s = 70
    first = {k: (v[:, :, :s] if k in ("q", "k", "v", "i_pre", "f_pre") else v) for k, v in inp.items()}
    second = {k: (v[:, :, s:] if k in ("q", "k", "v", "i_pre", "f_pre") else v) for k, v in inp.items()}
    for k1, k2 in (("chunkwise", "chunkwise"), ("chunkwise", "recurrent"), ("recurrent", "chunkwise")):
        h1, C1, n1, m1 = gpu_sequence(first, k1)
        st = tuple(torch.from_numpy(x).cuda() for x in (C1, n1, m1))
        h2, C2, n2, m2 = gpu_sequence(second, k2, state=st)
        compare((np.concatenate([h1, h2], 2), C2, n2, m2), ref, dtype, f"{k1}->{k2}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dqk,dv", [(64, 96), (512, 32), (80, 48)])
def test_step_matches_oracle_and_recurrent(dtype, dqk, dv):
    B, H, T = 3, 2, 40
    inp = small_inputs(B, H, T, dqk, dv, dtype, True, seed=21)
    ref = oracle_sequence(inp)
    C = to_dev(inp["C0"], "f32"); n = to_dev(inp["n0"], "f32"); m = to_dev(inp["m0"], "f32")
    hs = []
    for t in range(T):
        q, k, v = (to_dev(np.ascontiguousarray(inp[x][:, :, t]), dtype) for x in ("q", "k", "v"))
        ig, fg = (to_dev(np.ascontiguousarray(inp[x][:, :, t]), "f32") for x in ("i_pre", "f_pre"))
        h, (C, n, m) = capi.step(q, k, v, ig, fg, (C, n, m), qk_scale=inp["qk_scale"], inplace=(t % 2 == 0))
        hs.append(h.cpu().numpy())
    got = (np.stack(hs, 2), C.cpu().numpy(), n.cpu().numpy(), m.cpu().numpy())
    compare(got, ref, dtype, "step x T")
    compare(got, gpu_sequence(inp, "recurrent"), dtype, "step x T vs recurrent")


def test_invalid_arguments_rejected():
    d = capi.make_desc(1, 1, 8, 32, 32, capi.XLSTM_BF16, 1.0, 0)
    q = torch.zeros(1, 1, 8, 32, device="cuda", dtype=torch.bfloat16)
    g = torch.zeros(1, 1, 8, device="cuda")
    h = torch.empty(1, 1, 8, 32, device="cuda")
    ws = torch.zeros(256, device="cuda", dtype=torch.uint8)
    f = capi.xlstm_mlstm_fwd_chunkwise
    assert f(d, q, q, q, g, g, None, None, None, h, None, None, None, ws, 256) == capi.XLSTM_OK
    # output aliasing an input
    assert f(d, q, q, q, g, g, None, None, None, q, None, None, None, ws, 256) == capi.XLSTM_ERR_INVALID_ARG
    # workspace missing / too small
    assert f(d, q, q, q, g, g, None, None, None, h, None, None, None, None, 0) == capi.XLSTM_ERR_WORKSPACE
    assert f(d, q, q, q, g, g, None, None, None, h, None, None, None, ws, 16) == capi.XLSTM_ERR_WORKSPACE
    # misaligned pointer
    assert f(d, q.data_ptr() + 2, q, q, g, g, None, None, None, h, None, None, None, ws, 256) == capi.XLSTM_ERR_INVALID_ARG
    # unsupported chunk
    d.chunk = 48
    assert f(d, q, q, q, g, g, None, None, None, h, None, None, None, ws, 256) == capi.XLSTM_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert capi.xlstm_mlstm_workspace_status(ws)[0] == capi.XLSTM_OK


def test_device_wait_timeout_reports_status():
    """A bounded device-side wait that runs out (a hand-off withheld through
    the test hook) ends the kernel cleanly with XLSTM_ERR_TIMEOUT in the
    workspace status block; the context stays usable and the next call is
    correct."""
    inp = small_inputs(1, 2, 300, 64, 128, "bf16", True, seed=13)
    q, k, v = (to_dev(inp[n], "bf16") for n in ("q", "k", "v"))
    ig, fg = to_dev(inp["i_pre"], "f32"), to_dev(inp["f_pre"], "f32")
    st = tuple(to_dev(inp[n], "f32") for n in ("C0", "n0", "m0"))
    ws = torch.zeros(256, device="cuda", dtype=torch.uint8)
    capi.xlstm_mlstm_test_timeout_next(1)
    capi.fwd(q, k, v, ig, fg, state=st, qk_scale=inp["qk_scale"], workspace=ws)
    status, where = capi.xlstm_mlstm_workspace_status(ws)
    assert status == capi.XLSTM_ERR_TIMEOUT and where > 0, (status, where)
    h, (C, n, m) = capi.fwd(q, k, v, ig, fg, state=st, qk_scale=inp["qk_scale"], workspace=ws)
    assert capi.xlstm_mlstm_workspace_status(ws)[0] == capi.XLSTM_OK
    compare((h.cpu().numpy(), C.cpu().numpy(), n.cpu().numpy(), m.cpu().numpy()),
            oracle_sequence(inp), "bf16", "after timeout")


# ---- full-size workloads, sampled heads ------------------------------------------
_cache = {}


def full_inputs(name):
    if name not in _cache:
        _cache.clear()
        _cache[name] = inputs.make_sequence(inputs.WORKLOADS[name])
    return _cache[name]


def test_tiny_fp32_full():
    inp = full_inputs("tiny_fp32")
    ref = oracle_sequence(inp)
    for kind in ("chunkwise", "recurrent"):
        compare(gpu_sequence(inp, kind), ref, "f32", f"tiny_fp32 {kind}")


@pytest.mark.parametrize("name,heads", [("layer_7b", [0, 37, 63]), ("long_context", [2, 7]),
                                        ("many_short", [0, 511, 1023])])
@pytest.mark.parametrize("kind", ["chunkwise", "recurrent"])
def test_full_size_sampled_heads(name, heads, kind):
    inp = full_inputs(name)
    got = gpu_sequence(inp, kind)
    ref = oracle_sequence(inp, heads=heads)
    got = tuple(select_heads(x, heads) for x in got)
    compare(got, ref, inp["workload"].dtype, f"{name} {kind} heads {heads}")
    assert np.all(np.isfinite(got[0]))


def test_decode_256_steps_sampled_heads():
    w = inputs.WORKLOADS["decode"]
    rng, C0, n0, m0 = inputs.decode_state(w)
    heads = [0, 300, 1023]
    C, n, m = to_dev(C0, "f32"), to_dev(n0, "f32"), to_dev(m0, "f32")
    scale = w.d_qk ** -0.5
    hs, steps = [], []
    for st in inputs.decode_steps(w, rng):
        q, k, v = (to_dev(st[x], w.dtype) for x in ("q", "k", "v"))
        ig, fg = to_dev(st["i_pre"], "f32"), to_dev(st["f_pre"], "f32")
        h, (C, n, m) = capi.step(q, k, v, ig, fg, (C, n, m), qk_scale=scale, inplace=True)
        hs.append(select_heads(h.cpu().numpy(), heads)[0])
        steps.append({x: select_heads(st[x], heads)[0] for x in st})
    seq = {x: np.stack([s[x] for s in steps], 1)[None] for x in steps[0]}
    ref = oracle.forward(seq["q"], seq["k"], seq["v"], seq["i_pre"], seq["f_pre"],
                         select_heads(C0, heads), select_heads(n0, heads), select_heads(m0, heads),
                         qk_scale=scale)
    got = (np.stack(hs, 1)[None], select_heads(C.cpu().numpy(), heads),
           select_heads(n.cpu().numpy(), heads), select_heads(m.cpu().numpy(), heads))
    compare(got, ref, w.dtype, "decode 256 steps")
