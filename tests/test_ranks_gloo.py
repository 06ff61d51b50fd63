"""The multi-process plumbing of bench.py on CPU: one process per rank, gloo instead of NCCL.

The path does not shard (replicas only), so the ranks share nothing but the timing barrier and
the max over ranks of their measured times; the reference arm runs on rank 0 alone.
"""
import argparse
import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch

    import bench as b
    r = b.Ranks("gloo", timeout_s=60)
    # each rank's own "times": the max over ranks is what every rank reports
    m = r.max([1.0 + rank, 10.0 - rank, 0.5 * rank], torch.device("cpu"))
    r.barrier()
    q.put((rank, r.world, m, b.replica_rate(r.world, 4, m[0])))
    r.close()


def test_two_gloo_ranks_agree_on_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1]
    for _, world, m, rate in out:
        assert world == 2
        assert m == [2.0, 10.0, 0.5]
        assert rate == 2 * 4 / (2.0 / 1e3)  # both replicas' units over the slower rank's time


def test_one_rank_needs_no_process_group():
    import torch
    r = bench.Ranks("gloo")
    assert r.world == int(os.environ.get("WORLD_SIZE", "1")) == 1
    assert r.max([3.0, 1.5], torch.device("cpu")) == [3.0, 1.5]
    r.barrier()
    r.close()


def test_replica_rate_counts_every_rank():
    assert bench.replica_rate(4, 8, 100.0) == 320.0
    assert bench.replica_rate(1, 4, 9.6735) == 4 / 0.0096735


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="bank100m", steps=1, warmup=0)
    bench.run_reference(args)
    assert capsys.readouterr().out == ""
