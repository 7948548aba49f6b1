"""Multi-rank host logic on CPU (gloo, world size 2).

bench.py shards the layer as data-parallel replicas over tokens: no collective
on the data path. What the ranks share there is host logic: barriers, the max
over ranks of the device times, per-rank token seeds, and the reference arm
running on rank 0 only.

The expert-parallel layer (mixture_experts_layer_34_b200.ep) has one exchange,
the all-reduce of the fp32 partials. Its host logic (the expert and token
splits, the local weight stacks, the reduction and the finish order) runs here
over gloo with the oracle standing in for the two kernels, and the sum must be
the oracle's full forward.

These run as two gloo processes on 127.0.0.1.
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


def _run(world=2, target=None):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    target = target or _worker
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
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


# ----------------------------------------------------------------------------
# Expert-parallel layer
# ----------------------------------------------------------------------------

def test_splits_cover_every_item_once():
    from mixture_experts_layer_34_b200 import ep
    for n in (0, 1, 7, 16, 256, 257):
        for world in range(1, 10):
            parts = [ep.split_range(n, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            for (b0, e0), (b1, e1) in zip(parts, parts[1:]):
                assert e0 == b1
            sizes = [e - b for b, e in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        ep.split_range(8, 2, 2)


def test_local_stack_slots():
    from mixture_experts_layer_34_b200 import ep
    w = torch.arange(10).view(10, 1)            # E = 8 routed + S = 2 shared
    assert ep.local_stack(w, 8, 2, 3, 6).view(-1).tolist() == [3, 4, 5, 8, 9]
    assert ep.local_stack(w, 8, 2, 4, 4).view(-1).tolist() == [8, 9]


def _ep_layer():
    from mixture_experts_layer_34_b200 import workloads as W
    layer = W.BY_NAME["small_sig_bias"]
    return layer, W.make_layer(layer, "cpu")


def _ep_worker(rank, world, port, q, placed=False, sharded=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    import oracle.oracle as O
    from mixture_experts_layer_34_b200 import ep
    from mixture_experts_layer_34_b200 import ktmoe as K
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        layer, inp = _ep_layer()
        fields = layer.kernel_fields()
        E, S = layer.n_experts, layer.n_shared
        toks = list(range(0, layer.T, 5))
        x = inp["x"][toks].contiguous()
        og = O.gate(fields, inp["x"], inp["w_gate"], inp["bias"])
        idx, w = og["idx"][toks], og["w"][toks]

        class OracleRank(ep.ExpertParallelMoE):
            """The two kernels replaced by the oracle, on this rank's local stacks."""

            def local(self, x, part, topk_idx=None, topk_w=None):
                n_local = len(self.experts)
                lists = []
                for stack in (self.w1, self.w3, self.w2):
                    full = [None] * (E + S)
                    for i, e in enumerate(self.experts):
                        full[e] = stack[i]
                    for s in range(S):
                        full[E + s] = stack[n_local + s]
                    lists.append(full)
                T = x.shape[0]
                part.zero_()
                for e in self.experts:     # the rank's experts, one range each
                    yr, _ = O.forward_part(fields, x, idx, w, *lists, range(T), True, e, e + 1,
                                           shared=False)
                    part += torch.from_numpy(yr)
                sb, se = self.shared_range(T)
                if se > sb:
                    _, ys = O.forward_part(fields, x, idx, w, *lists, range(sb, se), True, 0, 0)
                    part[sb:se] += torch.from_numpy(ys)

            def buffers(self, T, device):
                return None, self._part.setdefault(T, torch.empty(T, layer.dim,
                                                                  dtype=torch.float64))

            def finish(self, part, x, y):
                y.copy_(part + (x.to(torch.float64) if layer.add_residual else 0))

            def finish_rows(self, part, x_rows, y_rows):
                self.finish(part, x_rows, y_rows)

        cfg = K.config_for(layer)
        placement = None
        if placed:   # a seeded shuffle of the experts, the same on every rank
            perm = np.random.default_rng(5).permutation(E).tolist()
            placement = [sorted(perm[r::world]) for r in range(world)]
        m = OracleRank(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"], rank,
                       world, placement=placement)
        ref = O.forward(fields, x, idx, w, inp["w1"], inp["w3"], inp["w2"], range(x.shape[0]),
                        True)
        if sharded:
            # each rank's token share, gathered here only to compare
            sb, se = m.shared_range(x.shape[0])
            ys = torch.empty(se - sb, layer.dim, dtype=torch.float64)
            m.forward_shard(x, ys)
            parts = [torch.empty_like(ys) for _ in range(world)]
            dist.all_gather(parts, ys)
            y = torch.cat(parts)
        else:
            y = torch.empty(x.shape[0], layer.dim, dtype=torch.float64)
            m.forward(x, y)
        dist.destroy_process_group()
        err = float(np.abs(y.numpy() - ref).max() / np.abs(ref).max())
        q.put((rank, (m.experts[0], m.experts[-1] + 1) if not placed else len(m.experts), err))
    except Exception as e:  # pragma: no cover - reported to the parent
        import traceback
        q.put((rank, None, traceback.format_exc()))


def test_expert_parallel_sum_is_the_forward_gloo():
    out = _run(2, _ep_worker)
    assert [r[1] for r in out] == [(0, 16), (16, 32)], out
    for rank, rng, err in out:
        assert isinstance(err, float), err
        assert err < 1e-12, (rank, err)


def _ep_worker_placed(rank, world, port, q):
    _ep_worker(rank, world, port, q, placed=True)


def test_expert_parallel_with_a_placement_gloo():
    out = _run(2, _ep_worker_placed)
    assert [r[1] for r in out] == [16, 16], out
    for rank, n, err in out:
        assert isinstance(err, float), err
        assert err < 1e-12, (rank, err)


def _ep_worker_sharded(rank, world, port, q):
    _ep_worker(rank, world, port, q, sharded=True)


def test_expert_parallel_reduce_scatter_gloo():
    """forward_shard: one reduce-scatter, each rank finishes its token share;
    the shares put together are the oracle's forward."""
    out = _run(2, _ep_worker_sharded)
    for rank, rng, err in out:
        assert isinstance(err, float), err
        assert err < 1e-12, (rank, err)


def test_balanced_placement_evens_a_skewed_load():
    import numpy as np
    from mixture_experts_layer_34_b200 import ep
    load = np.random.default_rng(3).zipf(1.3, 256).astype(float)
    for world in (2, 4, 8):
        p = ep.balanced_placement(load, world)
        assert sorted(e for r in p for e in r) == list(range(256))
        assert [len(r) for r in p] == [len(r) for r in ep.contiguous_placement(256, world)]
        per = [load[r].sum() for r in p]
        cont = [load[r].sum() for r in ep.contiguous_placement(256, world)]
        # The greedy bound: no rank exceeds the mean by more than the heaviest expert.
        assert max(per) <= load.sum() / world + load.max() + 1e-9
        assert max(per) <= max(cont)
    assert ep.slot_table([5, 2, 7], 8) == [-1, -1, 1, -1, -1, 0, -1, 2]
    with pytest.raises(ValueError):
        ep.slot_table([1, 1], 4)
