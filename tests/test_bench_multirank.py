"""The bench's host-side logic on CPU.

Multi-rank plumbing: two gloo ranks stand in for two GPUs (one process per
GPU under torchrun).  Checked: every rank joins the same collectives, the
reported time is the maximum over ranks, the whole-job value counts every
rank's work (weak scaling), and the reference arm prints only on rank 0.
Also the per-workload sweep's count of visible (query, key) pairs."""
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


def test_allowed_pairs_matches_brute_force():
    # the per-workload sweep's "allowed pairs" count, against a direct loop
    sys.path.insert(0, ROOT)
    import bench
    from attention_fwd_bwd_02_b200 import inputs as I
    cases = [I.make_case("ap_mod", 2, 3, 12, 12, 64, modality=(4, 8)),
             I.make_case("ap_pad", 3, 2, 5, 9, 64, kv_len_range=(0, 9)),
             I.make_case("ap_causal", 1, 2, 7, 7, 64, causal=True),
             I.make_case("ap_diag", 1, 1, 6, 6, 64, modality=(2, 4),
                         allow=((0, 1), (1, 0)), allow_diag=True)]
    for c in cases:
        n = 0
        for b in range(c.B):
            nk = c.Sk if c.kv_len is None else int(c.kv_len[b])
            for i in range(c.Sq):
                for j in range(c.Sk):
                    ok = j < nk and (not c.causal or j <= i)
                    if c.modality_ids is not None:
                        a, e = int(c.modality_ids[b, i]) & 1, int(c.modality_ids[b, j]) & 1
                        ok = ok and (bool(c.allow[a][e]) or (c.allow_diag and i == j))
                    n += ok
        assert bench._allowed_pairs(c) == n * c.N, c.name
