"""bench.py's multi-rank host logic (one replica per rank) on 2 gloo ranks.

The GPU benchmark runs one independent replica per rank and reports the
whole-job throughput as (units summed over ranks) / (time maxed over ranks);
this checks those reductions and the per-rank seeds without a GPU.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        t_max = bench.reduce_max(10.0 + rank, w)          # per-rank device time
        units = bench.reduce_sum(100.0 * (rank + 1), w)   # per-rank committed tokens
        q.put((r, w, lr, t_max, units, bench.rank_seed(7, r)))
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_and_seeds():
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
    assert [x[0] for x in res] == [0, 1] and all(x[1] == 2 for x in res)
    assert all(x[3] == 11.0 for x in res)          # max over ranks
    assert all(x[4] == 300.0 for x in res)         # sum over ranks
    assert res[0][5] != res[1][5]                   # independent batches


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.reduce_sum(2.0, 1) == 2.0
    assert bench.rank_seed(7, 0) == 7


def test_gpus_n_without_a_launcher_starts_n_ranks(capfd, monkeypatch):
    """bench.py --gpus 2 with no launcher starts the two ranks itself (here the
    oracle arm, which needs no GPU: rank 0 prints the record, rank 1 exits)."""
    import json
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        monkeypatch.delenv(k, raising=False)
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
                     "--warmup", "3"])
    out, err = capfd.readouterr()
    assert rc == 0, err[-2000:]
    assert "torch.distributed.run" in err and "--nproc-per-node=2" in err
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2


def test_gpus_n_refuses_rather_than_running_one_replica(capfd, monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import torch
    if torch.cuda.device_count() < 2:
        assert bench.main(["--gpus", "2"]) == 2          # too few GPUs: an error, no record
        assert "visible GPU" in capfd.readouterr().err
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--gpus", "4"]) == 2               # launcher and request disagree
    out, err = capfd.readouterr()
    assert out == "" and "WORLD_SIZE=2" in err
