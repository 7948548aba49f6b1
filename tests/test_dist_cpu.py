"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The layer shards as data-parallel replicas over tokens: no collective on the
data path. What the ranks share is host logic: barriers, the max over ranks of
the device times, per-rank token seeds, and the reference arm running on rank 0
only. These run as two gloo processes on 127.0.0.1.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from mixture_experts_layer_34_b200 import workloads as W
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        bench.init_dist(w, "gloo")
        # max over ranks of a per-rank device time
        got = bench.max_over_ranks(10.0 + rank, w, "cpu")
        bench.barrier(w)
        # every rank routes its own tokens, with distinct seeds
        seeds = [None] * w
        dist.all_gather_object(seeds, bench.rank_tokens_seed(W.V3_PREFILL, rank))
        dist.destroy_process_group()
        q.put((rank, got, seeds))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, repr(e), None))


def _run(world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_max_over_ranks_and_seeds_gloo():
    out = _run(2)
    for rank, got, seeds in out:
        assert got == 11.0, got
        assert len(set(seeds)) == 2


def test_reference_arm_only_on_rank0(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(bench.parse_args(["--impl", "reference", "--gpus", "2"]))
    assert capsys.readouterr().out == ""


def test_bench_rejects_too_few_warmup_steps():
    import bench
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
