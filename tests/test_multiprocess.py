"""The N > 1 replica path of the bench on CPU (gloo, world size 2): every
rank learns the slowest rank's time, the whole-job value counts all ranks'
units over that time, and only rank 0 runs the reference arm."""
import os
import socket

import pytest
import torch.distributed as td
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [2.5, 4.0][rank]
        mx = bench.max_over_ranks(ms, td, "cpu")
        q.put((rank, mx, bench.whole_job(1e9, world, mx)))
    finally:
        td.barrier()
        td.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [4.0, 4.0]          # both ranks see the slowest time
    assert got[0][2] == pytest.approx(2 * 1e9 / 4e-3)  # all ranks' units / slowest time


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.whole_job(10.0, 1, 1.0) == pytest.approx(1e4)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(None) is None
