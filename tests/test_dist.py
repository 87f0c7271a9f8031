"""The multi-rank plumbing of bench.py on CPU with two gloo ranks: every rank
gets the sum of all ranks' work and the slowest rank's time, ranks build
batches of the same shape from different seeds, and each rank is pinned to
its own GPU index. No GPU is involved: the decode path needs no collective,
so the ranks only exchange timing."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist = bench.init_dist(world, "gloo", timeout_s=60)
    try:
        units, ms = bench.aggregate(float(rank + 1) * 1e9, 10.0 * (rank + 1), world)
        bench.barrier(world)
        b = bench.make_batch("tiny_fp32", seed=rank)
        q.put((rank, units, ms, tuple(b.q.shape), float(b.q.double().sum())))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_and_seeding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, units, ms, shape, _ in res:
        assert units == pytest.approx(3e9)  # sum of the ranks' work
        assert ms == pytest.approx(20.0)    # the slowest rank's time
        assert shape == (4, 4, 64)
    assert res[0][4] != res[1][4]           # different seeds per rank


def test_single_rank_aggregation_is_identity():
    assert bench.aggregate(5.0, 2.0, 1) == (5.0, 2.0)


def test_rank_pinned_to_its_gpu(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5,6")
    bench.pin_device(1, 3)
    assert os.environ["CUDA_VISIBLE_DEVICES"] == "5"
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    bench.pin_device(2, 4)
    assert os.environ["CUDA_VISIBLE_DEVICES"] == "2"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "0,1")
    bench.pin_device(0, 1)  # a single process keeps what it was given
    assert os.environ["CUDA_VISIBLE_DEVICES"] == "0,1"


def test_reference_arm_other_ranks_do_nothing(capsys):
    class A:
        pass
    bench.run_reference(A(), rank=1, world=2)  # returns at once, prints nothing
    assert capsys.readouterr().out == ""
