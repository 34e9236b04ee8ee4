"""The multi-GPU (N > 1) host logic of bench.py on CPU: two real ranks over
the gloo backend (127.0.0.1), no GPU.  The path is partitioned by head (masks,
forward and backward are independent per head), so no data moves between
ranks; what is tested is the plumbing: rank/world discovery, the head ranges
(they tile [0, heads) exactly once), each rank's inputs equal to its slice of
the one-process inputs, the max-over-ranks timing and the sum of kept blocks
that every rank takes part in, the strong-scaling whole-job value, and the
reference arm's rule that ranks other than 0 exit without work."""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from adaptive_block_sparse_fractal_b200 import synth  # noqa: E402

W = synth.Workload("mr", 2, 4, 2, 16, 16, 64, (1, 4, 4), 0.7, backward=True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, wsz, local = bench.dist_init(world)
    dist.init_process_group("gloo", rank=r, world_size=wsz,
                            init_method="tcp://127.0.0.1:%d" % port)
    try:
        # each rank times a different step length; all must report the slowest
        got = bench.max_over_ranks(10.0 + 5.0 * r, wsz, "cpu")
        kept = bench.sum_over_ranks(100 + r, wsz, "cpu")
        h0, h1 = bench.head_range(W.heads, wsz, r)
        x = synth.make_inputs_device(W, 0, "cpu", head_range=(h0, h1))
        out.put((r, local, got, kept, (h0, h1), {k: v.clone() for k, v in x.items()}))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_head_partition():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in res] == [0, 1]
    assert [local for _, local, *_ in res] == [0, 1]
    assert all(got == 15.0 for _, _, got, *_ in res)   # the max, on every rank
    assert all(kept == 201.0 for *_, kept, _, _ in res)  # the sum, on every rank
    # the head ranges tile [0, heads) exactly once, in rank order
    ranges = [hr for *_, hr, _ in res]
    assert ranges == [(0, 2), (2, 4)]
    # each rank's inputs are its slice of the one-process problem
    full = synth.make_inputs_device(W, 0, "cpu")
    for name in ("q", "k", "v", "dout"):
        whole = full[name].view(W.B, W.heads, W.N, W.D)
        for *_, (h0, h1), x in res:
            assert torch.equal(x[name].view(W.B, h1 - h0, W.N, W.D), whole[:, h0:h1]), name
    # and the two ranks' heads differ
    assert not torch.equal(res[0][-1]["q"], res[1][-1]["q"])


def test_head_range_rejects_uneven_splits():
    assert bench.head_range(40, 8, 7) == (35, 40)
    assert bench.head_range(40, 1, 0) == (0, 40)
    with pytest.raises(SystemExit):
        bench.head_range(40, 3, 0)


def test_dist_init_checks_the_gpu_count(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.dist_init(2) == (1, 2, 1)
    with pytest.raises(SystemExit):
        bench.dist_init(4)


def test_whole_job_value_is_strong_scaling():
    # the job's FLOPs (all ranks' heads) in the slowest rank's time
    assert bench.whole_job_tflops(2e12, 1000.0) == pytest.approx(2.0)
    assert bench.whole_job_tflops(2e12, 250.0) == pytest.approx(8.0)


def test_reference_arm_runs_on_rank_0_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = bench.parse(["--impl", "reference", "--gpus", "2"])
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args) == 0
    assert buf.getvalue() == ""  # no work and no line on ranks other than 0
