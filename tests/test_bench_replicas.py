"""Host logic of the multi-GPU path ("replicas only": every rank runs the whole
workload, no data exchange): the max-over-ranks time and the whole-job value,
on two gloo ranks on the CPU, and the reference arm printing on rank 0 only."""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.max_over_ranks(values[rank], world, dist, "cpu")
        dist.barrier()
        out.put((rank, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    values = [3.25, 7.5]
    procs = [ctx.Process(target=_rank, args=(r, 2, port, values, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(out.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 7.5, 1: 7.5}


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(2.5, 1) == 2.5


def test_whole_job_value_counts_the_pairs_of_all_ranks():
    # 10 steps of 21 pairs on each of 4 ranks in 84 ms (the slowest rank): 100 us per pair
    assert bench.per_pair_us(84.0, 10, 21, 4) == pytest.approx(100.0)
    assert bench.per_pair_us(84.0, 10, 21, 1) == pytest.approx(400.0)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    args = type("A", (), dict(steps=1, warmup=0, cpu_budget=0.01))()
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""
