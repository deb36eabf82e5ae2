"""Segment-parallel chunkwise forward against the float64 oracle.

Long sequences with few heads run as parallel segments when the workspace is
large enough: segment summaries from a zero state, their chaining into entry
states, then every segment at once.  These cases take that path (checked
through the workspace sizes) and must meet the bf16 tolerances of the
sequential evaluation, with the canonical final m.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import compare, gpu_sequence, oracle_sequence, select_heads, small_inputs
from xlstm_mlstm_matrix_b200 import capi, inputs

pytestmark = pytest.mark.gpu


def segmented(B, H, T, dqk, dv):
    d = capi.make_desc(B, H, T, dqk, dv, capi.XLSTM_BF16, 1.0, 64)
    return capi.xlstm_mlstm_workspace_size_parallel(d) > capi.xlstm_mlstm_workspace_size(d)


CASES = [  # B, H, T, dqk, dv: each cut into 2 .. 7 segments
    (1, 2, 2048, 64, 64),      # 4 segments of 8 chunks
    (1, 1, 4000, 128, 128),    # 7 segments of 9 chunks, ragged tail
    (1, 2, 1100, 256, 512),    # 2 segments, four value slices
    (2, 1, 1500, 128, 192),    # a half-filled value slice
    (1, 3, 1600, 256, 256),
]


@pytest.mark.parametrize("state", [False, True])
@pytest.mark.parametrize("shape", CASES, ids=lambda s: "x".join(map(str, s)))
def test_segments_match_oracle(shape, state):
    assert segmented(*shape)
    inp = small_inputs(*shape, "bf16", state, seed=sum(shape))
    ref = oracle_sequence(inp)
    got = gpu_sequence(inp, "chunkwise", parallel=True)
    compare(got, ref, "bf16", f"segments {shape} state={state}")
    seq = gpu_sequence(inp, "chunkwise")
    compare(got, seq, "bf16", "segments vs one piece")


@pytest.mark.parametrize("gate,mean_i,std_i", [("mixed", 0.0, 1.0), ("std", 30.0, 40.0), ("std", -8.0, 3.0)])
def test_segments_stabilizer_stress(gate, mean_i, std_i):
    """Positive log-forget gates, input-gate jumps that force exact chunks, and
    input gates so low that a segment's own stabilizer sits far below the
    carried one."""
    shape = (1, 2, 2600, 128, 128)
    assert segmented(*shape)
    inp = small_inputs(*shape, "bf16", True, seed=5, gate=gate, mean_i=mean_i, std_i=std_i)
    compare(gpu_sequence(inp, "chunkwise", parallel=True), oracle_sequence(inp), "bf16", f"segments {gate}")


def test_segments_reset_gates():
    shape = (1, 2, 2048, 64, 128)
    inp = small_inputs(*shape, "bf16", True, seed=9)
    inp["f_pre"] = np.full_like(inp["f_pre"], -1.0e4)
    compare(gpu_sequence(inp, "chunkwise", parallel=True), oracle_sequence(inp), "bf16", "segments reset")


def test_segments_repeatable():
    """The three launches hand off through the workspace in stream order; the
    same call repeated gives the same bits."""
    shape = (1, 2, 2600, 256, 128)
    inp = small_inputs(*shape, "bf16", True, seed=4, gate="std", mean_i=30.0, std_i=40.0)
    first = gpu_sequence(inp, "chunkwise", parallel=True)
    for _ in range(5):
        got = gpu_sequence(inp, "chunkwise", parallel=True)
        for a, b in zip(got, first):
            np.testing.assert_array_equal(a, b)


def test_long_context_full_size_sampled_heads():
    """The long-context layer (B1 H8 T65536 d128/128) runs as 18 segments."""
    w = inputs.WORKLOADS["long_context"]
    assert segmented(w.B, w.H, w.T, w.d_qk, w.d_v)
    inp = inputs.make_sequence(w)
    heads = [0, 5]
    got = tuple(select_heads(x, heads) for x in gpu_sequence(inp, "chunkwise", parallel=True))
    compare(got, oracle_sequence(inp, heads=heads), "bf16", "long_context segments")
    torch.cuda.empty_cache()
