"""Expert-parallel MoE layer over a torch.distributed process group.

The multi-card form of "MoE 前向四步" in the DeepSeek-V3 model.py notes
(73biji.xyz/llm_pp_dsv3): each card loops over its own experts only, the
partial outputs are all-reduced, and the shared experts' z is added. The number
of cards is the expert_parallel_degree setting of the tuning section of the
DeepSeek model-family article (cloud.baidu.com/article/3606489).

Per rank:
  * the routed experts of one contiguous range (``expert_range``, the pages'
    form), or of any placement (``balanced_placement`` spreads the heavy
    experts of a skewed load over the ranks), held as a local weight stack:
    those experts, then the shared ones (``local_stack``);
  * the gate on all tokens (every rank routes the same tokens identically), the
    local experts on their tokens, and the shared experts on this rank's share
    of the tokens (``token_range``), summed in fp32 by ``kt_moe_forward_local``;
  * one all-reduce of that fp32 [T, dim] partial (NCCL over NVLink/NVSwitch on
    GPUs), which sums routed outputs and z in one message; or, for a next layer
    that takes its tokens sharded over the same ranks, a reduce-scatter that
    leaves each rank the sum for its own share of the tokens (half the bytes);
  * ``kt_moe_ep_finish``: the residual and the rounding to y's type.

Every arithmetic step runs in libktmoe.so's kernels; this module holds the
partition, the local weight stacks, the buffers and the collective.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ktmoe as K


def split_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """[begin, end) of rank's share of n items in world contiguous parts; the
    first n % world parts hold one more item."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad split: n={n} world={world} rank={rank}")
    base, extra = divmod(n, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def expert_range(n_experts: int, world: int, rank: int) -> tuple[int, int]:
    """Routed experts of one rank."""
    return split_range(n_experts, world, rank)


def token_range(T: int, world: int, rank: int) -> tuple[int, int]:
    """Tokens one rank runs the shared experts on."""
    return split_range(T, world, rank)


def local_stack(w, n_experts: int, n_shared: int, begin: int, end: int):
    """A rank's weight slots from a stacked [E + S, ...] weight: routed experts
    [begin, end), then the S shared experts, as one contiguous tensor."""
    return torch.cat([w[begin:end], w[n_experts:n_experts + n_shared]]).contiguous()


def local_stack_of(w, n_experts: int, n_shared: int, experts):
    """The same for any list of routed experts (slot i holds experts[i])."""
    idx = torch.as_tensor(list(experts) + list(range(n_experts, n_experts + n_shared)),
                          dtype=torch.long, device=w.device)
    return w.index_select(0, idx).contiguous()


def contiguous_placement(n_experts: int, world: int) -> list[list[int]]:
    """Each rank's experts as contiguous ranges (``expert_range``)."""
    return [list(range(*expert_range(n_experts, world, r))) for r in range(world)]


def balanced_placement(load, world: int) -> list[list[int]]:
    """Experts over ranks by expected load (for example a previous batch's
    per-expert token counts): heaviest first, each to the least-loaded rank that
    still has room, so that every rank holds as many experts as a contiguous
    split gives it. Each rank's list is in ascending expert order."""
    load = [float(v) for v in load]
    E = len(load)
    cap = [e - b for b, e in (expert_range(E, world, r) for r in range(world))]
    total = [0.0] * world
    count = [0] * world
    out: list[list[int]] = [[] for _ in range(world)]
    for e in sorted(range(E), key=lambda i: (-load[i], i)):
        r = min((r for r in range(world) if count[r] < cap[r]), key=lambda r: (total[r], r))
        out[r].append(e)
        total[r] += load[e]
        count[r] += 1
    return [sorted(x) for x in out]


def slot_table(experts, n_experts: int) -> list[int]:
    """expert -> weight slot on the rank holding ``experts`` (-1 elsewhere)."""
    tab = [-1] * n_experts
    for i, e in enumerate(experts):
        if not 0 <= e < n_experts or tab[e] != -1:
            raise ValueError(f"bad expert list: {experts}")
        tab[e] = i
    return tab


class ExpertParallelMoE:
    """One rank of the expert-parallel layer.

    cfg: the full layer's kt_moe_config (all E routed experts). w1/w3/w2: the
    full stacked weights [E + S, ...] (sliced here), or, with
    ``weights_are_local``, this rank's stack already. placement: None for
    contiguous ranges, else every rank's list of routed experts (the same
    lists on every rank). With an MXFP8 config the local stacks (bf16) are
    packed once here.
    """

    def __init__(self, cfg, w_gate, bias, w1, w3, w2, rank: int, world: int, group=None,
                 weights_are_local: bool = False, placement=None):
        self.cfg, self.rank, self.world, self.group = cfg, rank, world, group
        E, S = cfg.n_experts, cfg.n_shared
        if placement is None:
            self.eb, self.ee = expert_range(E, world, rank)
            self.experts = list(range(self.eb, self.ee))
            self.table = None
        else:
            if len(placement) != world or sorted(e for p in placement for e in p) != list(range(E)):
                raise ValueError("placement must list every routed expert exactly once")
            self.experts = list(placement[rank])
            self.table = slot_table(self.experts, E)
        if not weights_are_local:
            if self.table is None:
                w1, w3, w2 = (local_stack(w, E, S, self.eb, self.ee) for w in (w1, w3, w2))
            else:
                w1, w3, w2 = (local_stack_of(w, E, S, self.experts) for w in (w1, w3, w2))
        n_local = len(self.experts)
        n_slots = n_local + S
        for w in (w1, w3, w2):
            if w.shape[0] != n_slots:
                raise ValueError(f"local stack has {w.shape[0]} slots, expected {n_slots}")
        self.w_gate, self.bias = w_gate, bias
        self.mxfp8 = cfg.dtype in (K.KT_DTYPE_MXFP8, K.KT_DTYPE_MXFP4)   # block-scaled weights
        if self.mxfp8:
            self.q = K.pack_mxfp8_local(cfg, 0, n_local, w1, w3, w2)
            self.w1 = self.w3 = self.w2 = None
        else:
            self.q = None
            self.w1, self.w3, self.w2 = w1, w3, w2
        self._ws: dict[int, torch.Tensor] = {}
        self._part: dict[int, torch.Tensor] = {}
        self._shard: dict[int, torch.Tensor] = {}

    def shared_range(self, T: int) -> tuple[int, int]:
        return token_range(T, self.world, self.rank)

    def buffers(self, T: int, device) -> tuple[torch.Tensor, torch.Tensor]:
        """The workspace and the fp32 partial for T tokens (allocated once per T)."""
        if T not in self._ws:
            self._ws[T] = K.alloc_workspace(self.cfg, T, device)
            self._part[T] = torch.empty((T, self.cfg.dim), dtype=torch.float32, device=device)
        return self._ws[T], self._part[T]

    def local(self, x, part, topk_idx=None, topk_w=None):
        """This rank's fp32 partial into ``part`` (every row written)."""
        T = x.shape[0]
        ws, _ = self.buffers(T, x.device)
        sb, se = self.shared_range(T)
        q = self.q
        if self.table is not None and self.mxfp8:
            K.kt_moe_forward_placed_mxfp8(self.cfg, T, x, self.w_gate, self.bias, self.table, sb, se,
                                          q["w1q"], q["w3q"], q["w2q"], q["sf_up"], q["sf_down"],
                                          part, topk_idx, topk_w, ws)
        elif self.table is not None:
            K.kt_moe_forward_placed(self.cfg, T, x, self.w_gate, self.bias, self.table, sb, se,
                                    self.w1, self.w3, self.w2, part, topk_idx, topk_w, ws)
        elif self.mxfp8:
            K.kt_moe_forward_local_mxfp8(self.cfg, T, x, self.w_gate, self.bias, self.eb, self.ee,
                                         sb, se, q["w1q"], q["w3q"], q["w2q"], q["sf_up"],
                                         q["sf_down"], part, topk_idx, topk_w, ws)
        else:
            K.kt_moe_forward_local(self.cfg, T, x, self.w_gate, self.bias, self.eb, self.ee, sb,
                                   se, self.w1, self.w3, self.w2, part, topk_idx, topk_w, ws)

    def reduce(self, part):
        """Sum of the partials over the ranks, in place."""
        if self.world > 1:
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)

    def finish(self, part, x, y):
        K.kt_moe_ep_finish(self.cfg, x.shape[0], part, x, y)

    def forward(self, x, y, topk_idx=None, topk_w=None):
        """y = the layer's output for tokens x (the same x on every rank)."""
        _, part = self.buffers(x.shape[0], x.device)
        self.local(x, part, topk_idx, topk_w)
        self.reduce(part)
        self.finish(part, x, y)
        return y

    def forward_shard(self, x, y_shard, topk_idx=None, topk_w=None):
        """The output rows of this rank's token share only (``token_range``;
        T must be a multiple of the world size): one reduce-scatter instead of
        the all-reduce. y_shard is [T / world, dim]."""
        T = x.shape[0]
        if T % self.world:
            raise ValueError(f"reduce-scatter needs T ({T}) divisible by the world size")
        _, part = self.buffers(T, x.device)
        self.local(x, part, topk_idx, topk_w)
        sb, se = self.shared_range(T)
        if self.world > 1:
            if T not in self._shard:
                self._shard[T] = torch.empty((se - sb, self.cfg.dim), dtype=part.dtype,
                                             device=x.device)
            shard = self._shard[T]
            dist.reduce_scatter_tensor(shard, part, op=dist.ReduceOp.SUM, group=self.group)
        else:
            shard = part
        self.finish_rows(shard, x[sb:se], y_shard)
        return y_shard

    def finish_rows(self, part, x_rows, y_rows):
        K.kt_moe_ep_finish(self.cfg, x_rows.shape[0], part, x_rows, y_rows)

    def graph(self, x, y, topk_idx=None, topk_w=None) -> "EpGraph":
        """The whole step (local forward, all-reduce, finish) captured once as a
        CUDA graph on these buffers; ``replay()`` reruns it (x is read in place,
        so a decode loop rewrites x between replays). NCCL's all-reduce is
        captured with the kernels when the group has more than one rank."""
        T = x.shape[0]
        self.buffers(T, x.device)
        # One eager step first: the library's one-time host setup (kernel
        # attributes) stays out of the capture, and NCCL's communicator exists.
        self.forward(x, y, topk_idx, topk_w)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            self.forward(x, y, topk_idx, topk_w)
        return EpGraph(g, (x, y, topk_idx, topk_w))


class EpGraph:
    """A captured expert-parallel step; holds the tensors bound into it."""

    def __init__(self, g, keep):
        self._g, self._keep = g, keep

    def replay(self):
        self._g.replay()
