"""The benchmark's multi-rank plumbing on CPU: two gloo ranks get distinct
input seeds (independent problems per GPU), the timing reduction returns the
slowest rank's time on every rank, and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_env()
    bench.init_dist(w, "gloo")
    slow = bench.reduce_max(10.0 * (r + 1), "cpu")
    seed = bench.rank_seed(1000, r)
    # the reference arm: only rank 0 does work (and would print)
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    did = r == 0
    q.put((r, slow, seed, did))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]           # max over ranks, seen by both
    assert res[0][2] != res[1][2]                         # independent inputs per rank
    assert [r[3] for r in res] == [True, False]


def test_reference_arm_skips_other_ranks(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(bench.parse_args(["--impl", "reference"])) == 0
    assert capsys.readouterr().out == ""
