"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The forward pass shards over independent (batch, head) pairs, so ranks run
replicas with no collective on the data path; the only cross-rank steps are
the barrier around the timed region and the max over ranks of the step time.
These tests run that host logic as two gloo processes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ms_per_rank, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(ms_per_rank[rank], dist, "cpu")
        w = bench.workload_for_rank("layer_7b", rank)
        rate = bench.job_rate(bench.tokens_per_step(w), world, ms)
        dist.barrier()
        out.put((rank, ms, rate, w.seed))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo_world2():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    ms = [1.25, 3.5]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, ms, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(2))
    # every rank sees the slowest rank's time
    assert [r[1] for r in res] == [3.5, 3.5]
    # whole-job rate: both ranks' tokens over the slowest time
    tokens = 8 * 4096
    assert res[0][2] == pytest.approx(2 * tokens / 3.5e-3)
    assert res[0][2] == res[1][2]
    # replicas draw different inputs
    assert res[0][3] != res[1][3]


def test_single_rank_helpers():
    assert bench.max_over_ranks(2.0) == 2.0
    assert bench.job_rate(1000, 1, 1.0) == pytest.approx(1e6)
    w = bench.workload_for_rank("decode", 0, B=4)
    assert (w.B, w.H, w.steps) == (4, 8, 256)
    assert bench.tokens_per_step(w) == 4          # one token per sequence per decode step
    w = bench.workload_for_rank("long_context", 1, T=1024)
    assert (w.T, w.seed) == (1024, 1002)


def test_algorithmic_bytes_match_the_counting_convention():
    # 7B-like layer: 1,109,459,200 bytes and 150.3 GFLOP per forward
    b, f = bench.algorithmic(bench.workload_for_rank("layer_7b", 0))
    assert b == 1_109_459_200
    assert f == pytest.approx(150.3e9, rel=1e-3)
    # the output stage with bf16 o~ and h: o~ read (2 B) replaces half of the fp32 h write
    bg, fg = bench.algorithmic(bench.workload_for_rank("layer_7b", 0), gated=True)
    assert bg == 1_109_459_200 and fg == f
    # decode step: the state is read and written once (about 1.08 GB at B=128, H=8)
    b, _ = bench.algorithmic(bench.workload_for_rank("decode", 0))
    assert b == pytest.approx(1.08e9, rel=0.01)


def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    """`bench.py --impl reference` under torchrun with 2 ranks: rank 0 alone
    runs the oracle sample and prints one JSON line; rank 1 exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "many_short", "--ref-budget", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_traffic_figure_only_for_the_captured_full_size_workload():
    """roofline.traffic comes from a capture of the full-size workload on the
    current kernel source: a smaller case of the same name, or the gated output
    path, reports none."""
    sha = bench.kernel_source_sha()
    full = bench.workload_for_rank("layer_7b", 0)
    small = bench.workload_for_rank("layer_7b", 0, T=1024)
    other_rank = bench.workload_for_rank("layer_7b", 3)
    assert bench.traffic_for(sha, small) is None
    assert bench.traffic_for(sha, full, gated=True) is None
    assert bench.traffic_for("0" * 16, full) is None
    assert bench.traffic_for(sha, full) == bench.traffic_for(sha, other_rank)
