"""The bench's multi-rank plumbing on CPU: two gloo ranks stand in for two
GPUs (one process per GPU under torchrun).  Checked: every rank joins the
same collectives, the reported time is the maximum over ranks, the
whole-job value counts every rank's work (weak scaling), and the reference
arm prints only on rank 0."""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    r, w, _ = bench.dist_setup(world, backend="gloo")
    # Each rank's own (device) time differs; the report takes the slowest.
    mine = 10.0 + 3.0 * r
    slowest = bench.max_over_ranks(mine, w)
    bench.barrier(w)
    value = bench.whole_job_value(1e12, w, slowest)
    # The reference arm: rank 0 alone runs and prints; the others return.
    out = io.StringIO()
    if r != 0:
        with contextlib.redirect_stdout(out):
            bench.run_reference(None)
    bench.finish(w)
    queue.put((r, slowest, value, out.getvalue()))


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    for r, slowest, value, printed in results:
        assert slowest == pytest.approx(13.0)          # max over ranks
        assert value == pytest.approx(2 * 1e12 / 13e-3 / 1e12)  # both ranks' work
        assert printed == ""                            # only rank 0 prints


def test_single_rank_value_is_per_gpu_work():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.2, 1) == 4.2
    assert bench.whole_job_value(2e12, 1, 10.0) == pytest.approx(200.0)
