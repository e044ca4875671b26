"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

The path shards into independent chunks (weak scaling, no data-path
collective); what needs checking is the plumbing around it: rendezvous,
per-rank seeds, the max-over-ranks timing reduction, and that the reference
arm runs on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    r, l, w = bench.dist_setup(backend="gloo")
    m = bench.max_over_ranks(10.0 * (rank + 1))
    seed = bench.rank_seed(4, rank)
    bench.barrier()
    q.put((r, w, m, seed))
    dist.destroy_process_group()


def test_two_ranks_reduce_max_and_distinct_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert all(r[2] == 20.0 for r in res)  # max over ranks seen by every rank
    assert res[0][3] != res[1][3]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""


def test_headline_flops_and_workload():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.headline_flops() == 4 * 128 * 40 * 4680 * 37440
    assert abs(bench.headline_flops() / 1e12 - 3.5885) < 1e-3
