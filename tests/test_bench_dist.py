"""Host-side test of the bench's multi-process path (replicas, one process per GPU):
two gloo ranks on the CPU go through the same rendezvous, barrier and max-over-ranks
code the NCCL run uses, and the whole-job aggregate scales with the world size."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, local = bench.dist_setup(world, backend="gloo")
    # each rank "measured" a different time; every rank must see the slowest one
    ms = bench.max_over_ranks(10.0 + 5.0 * r, w, device="cpu")
    bench.barrier(w)
    out.put((r, w, local, ms))
    dist.destroy_process_group()


def test_replicas_rendezvous_and_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(out.get(timeout=10) for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == world and g[2] == g[0] for g in got)
    assert all(g[3] == pytest.approx(15.0) for g in got)  # max over ranks


def test_whole_job_aggregate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_gbs(4.0e8, 1, 100, 26.0)
    two = bench.whole_job_gbs(4.0e8, 2, 100, 26.0)
    assert one == pytest.approx(4.0e8 * 100 / 26.0e-3 / 1e9)
    assert two == pytest.approx(2 * one)  # same per-rank work and time: twice the bytes
    assert bench.max_over_ranks(3.5, 1) == 3.5  # one rank: no collective


def test_rotations_cover_twice_the_l2(monkeypatch):
    """The bench protocol: the input copies a timed graph rotates over together exceed
    2x L2 (126 MB on a B200), for inputs from a few KB to more than L2 itself."""
    sys.path.insert(0, ROOT)
    import bench
    L2 = 126 * 2**20
    monkeypatch.setattr(bench, "l2_bytes", lambda: L2)
    for by in (1, 4096, 8 * 2**20, 25 * 2**20 + 7, 2 * L2 - 1, 2 * L2, 5 * L2):
        n = bench.rotations_for(by)
        assert n >= 1 and (n * by >= 2 * L2 or n == 1 and by >= 2 * L2)
        assert (n - 1) * by < 2 * L2  # no more copies than needed
