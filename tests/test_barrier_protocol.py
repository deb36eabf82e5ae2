"""The chunkwise kernel's barrier hand-offs (model in barrier_protocol.py): no
deadlock and no phase overrun for every chunk count, V-stage count, head size class
and pattern of exact chunks tried; and the earlier forms are rejected: one B_OPS and
one B_VT barrier with two V stages, and the token group waiting for an exact chunk's
V with one V stage (a consumer could come to wait for a phase after the next one
had completed)."""
import itertools

import pytest

from barrier_protocol import chunkwise_protocol, summary_protocol

PATTERNS = [(), (0,), (1,), (0, 1), (2, 3, 5), (1, 3, 5, 7), tuple(range(9))]


@pytest.mark.parametrize("vst,big", [(2, False), (2, True), (1, False)])
@pytest.mark.parametrize("nc", [1, 2, 3, 6, 9])
def test_protocol_has_no_deadlock_or_overrun(vst, big, nc):
    for exact in PATTERNS:
        ex = tuple(c for c in exact if c < nc)
        problems = chunkwise_protocol(nc, vst, big, ex).check()
        assert not problems, (vst, big, nc, ex, problems[:3])


@pytest.mark.parametrize("big", [False, True])
def test_single_ops_and_vt_barriers_are_rejected(big):
    """With one B_OPS the state group's wait for P(c) can be overtaken; with one B_VT
    the MMA warp's wait for w V(c) can, except at d_qk = 256, where the token group
    scales V(c+1) only after the MMA warp has freed the C_lo tile of chunk c."""
    found = set()
    for nc, exact in itertools.product([3, 6], [(), (2,), (1, 4)]):
        for p in chunkwise_protocol(nc, 2, big, tuple(c for c in exact if c < nc), paired=False).check():
            assert p.startswith("overrun"), p
            found.add(p.split(":")[1].split()[0])
    assert found == ({"OPS"} if big else {"OPS", "VT"}), found


def test_exact_chunk_v_wait_with_one_v_stage_is_rejected():
    problems = chunkwise_protocol(3, 1, False, (1,), exact_v_wait=True).check()
    assert any(p.startswith("overrun: V_FULL") for p in problems), problems


def test_checker_finds_a_missing_arrival():
    """A planted defect: the state group never releases H (B_H_EMPTY)."""
    P = chunkwise_protocol(3, 2, False)
    P.roles["state"] = [op for op in P.roles["state"] if op[1] != "H_EMPTY"]
    assert any(p.startswith("deadlock") for p in P.check())


def test_checker_finds_an_underrun():
    """A planted defect: with one V stage and chunk 1 exact, a token group that no
    longer waits for S, the update or H could start waiting for V(2) while V(1),
    which it skipped, is still in flight."""
    P = chunkwise_protocol(4, 1, False, (1,))
    P.roles["token"] = [op for op in P.roles["token"] if op[1] not in ("S_FULL", "UPD_DONE", "H_FULL")]
    assert any(p.startswith("underrun: the wait of token for V_FULL") for p in P.check())


@pytest.mark.parametrize("stages", [4, 6, 8])
@pytest.mark.parametrize("nc", [1, 3, 5, 8, 13, 40])
def test_summary_protocol_has_no_deadlock_or_overrun(stages, nc):
    problems = summary_protocol(nc, stages).check()
    assert not problems, (stages, nc, problems[:3])


def _kernel_barriers(path, prefix):
    import os
    import re
    root = os.path.join(os.path.dirname(__file__), "..", "xlstm_mlstm_matrix_b200", "csrc")
    src = open(os.path.join(root, path)).read()
    return set(re.findall(r"bar\[" + re.escape(prefix) + r"(B_[A-Z0-9_]+)", src))


def _model_barriers(P):
    import re
    # model names: kernel names without "B_", slot digits appended; CONV_SPLIT / CONV_CLO
    # stand for B_CONV0 / B_CONV1
    names = {re.sub(r"\d+$", "", bar) for ops in P.roles.values() for _, bar, _ in ops}
    names = {"CONV" if n.startswith("CONV_") else n for n in names}
    return {"B_" + n for n in names}


def test_model_covers_every_barrier_of_the_chunkwise_kernel():
    """The model names every hand-off barrier the kernel waits on or arrives at (the
    drain barrier, used by one thread alone at teardown, aside); a barrier added to
    the kernel without the model fails here."""
    used = _kernel_barriers("chunkwise_tc.cu", "") - {"B_DRAIN"}
    used = {"B_CONV" if n.startswith("B_CONV") else n for n in used}
    modelled = set()
    for vst, big in ((2, False), (2, True), (1, False)):
        modelled |= _model_barriers(chunkwise_protocol(4, vst, big, (1,)))
    assert used == modelled, (used - modelled, modelled - used)


def test_model_covers_every_barrier_of_the_summary_kernel():
    used = _kernel_barriers("segments.cu", "C::") - {"B_DRAIN"}
    assert used == _model_barriers(summary_protocol(6, 4)), used
