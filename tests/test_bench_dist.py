"""The benchmark's multi-rank plumbing on CPU: two gloo ranks join through
dist_setup, take the element-wise maximum of their times, and agree on the
whole-job value (weak scaling: tokens of all ranks over the slowest rank's
step).  The reference arm's non-zero ranks leave without work."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, ws, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(ws), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    r, local, w = bench.dist_setup(backend="gloo")
    assert (r, local, w) == (rank, rank, ws)
    times = [1.0 + rank, 10.0 - rank, 3.0]
    got = bench.max_over_ranks(times, dist, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    w0 = bench.workload(bench.HEADLINE)
    out.put((rank, got, bench.job_value(w, got[0], w0["B"], w0["N"])))


def test_two_gloo_ranks_take_the_max_and_sum_tokens():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, val in res:
        assert got == [2.0, 10.0, 3.0]
        w0 = bench.workload(bench.HEADLINE)
        assert val == pytest.approx(2 * w0["B"] * w0["N"] / (2.0e-3))


def test_single_rank_needs_no_process_group(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.dist_setup() == (0, 0, 1)
    assert bench.max_over_ranks([1.0, 2.0], None, "cpu") == [1.0, 2.0]
    assert bench.job_value(1, 1.0, 16, 131072) == pytest.approx(16 * 131072 / 1e-3)


def test_reference_arm_nonzero_rank_exits_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, ref_steps, gpus, cpu_seconds = 4, 3, 0, 2, 1.0
        workload, batch = bench.HEADLINE, None

    bench.run_reference(Args())
    assert capsys.readouterr().out == ""
