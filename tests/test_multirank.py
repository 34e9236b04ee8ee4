"""The multi-GPU (N > 1) host logic of bench.py on CPU: two real ranks over
the gloo backend (127.0.0.1), no GPU.  The path shards by (batch, head) with
no data exchange, so what is tested is the plumbing: rank/world discovery,
the max-over-ranks timing reduction every rank takes part in, the weak-
scaling whole-job value, per-rank inputs, and the reference arm's rule that
ranks other than 0 exit without work."""
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
        # per-rank inputs: same recipe, own seeds
        w = synth.Workload("mr", 1, 1, 2, 16, 16, 64, (1, 4, 4), 0.7)
        x = synth.make_inputs_device(w, 0, "cpu", with_dout=False, rank=r)["q"]
        gathered = [torch.empty_like(x) for _ in range(wsz)]
        dist.all_gather(gathered, x)
        out.put((r, local, got, bool(torch.equal(gathered[0], gathered[1]))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_over_ranks_and_per_rank_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in res] == [0, 1]
    assert [local for _, local, *_ in res] == [0, 1]
    assert all(got == 15.0 for _, _, got, _ in res)   # the max, on every rank
    assert not res[0][3]                               # ranks draw different batches


def test_dist_init_checks_the_gpu_count(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.dist_init(2) == (1, 2, 1)
    with pytest.raises(SystemExit):
        bench.dist_init(4)


def test_whole_job_value_is_weak_scaling():
    # N ranks each doing F FLOP in the slowest rank's t ms -> N * F / t
    assert bench.whole_job_tflops(2e12, 1000.0, 1) == pytest.approx(2.0)
    assert bench.whole_job_tflops(2e12, 1000.0, 8) == pytest.approx(16.0)


def test_reference_arm_runs_on_rank_0_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = bench.parse(["--impl", "reference", "--gpus", "2"])
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args) == 0
    assert buf.getvalue() == ""  # no work and no line on ranks other than 0
