"""Expert-parallel form on one GPU, through the C ABI.

Ranks run one after another on the same GPU (independent launches; nothing
waits on another rank), each with its expert range, its local weight stack and
its share of the shared experts' tokens. The partials are summed here in rank
order, which is what the all-reduce computes, and kt_moe_ep_finish finishes.

Checks:
  * each rank's routing equals kt_moe_forward's, bit for bit;
  * each rank's fp32 partial matches the oracle's part (routed experts of the
    range on every token, shared experts on the rank's tokens) within the
    layer's tolerance, relative to the full output's RMS;
  * the finished sum matches the oracle's forward within the same tolerance
    and kt_moe_forward within 1e-4 of its RMS (the expert rows are the same
    arithmetic; only the order of the fp32 sum differs);
  * one rank holding everything is kt_moe_forward bit for bit (same rows, same
    sum order, the residual last);
  * MXFP8: the local pack is the full pack's slots, byte for byte, and the
    finished sum matches kt_moe_forward_mxfp8 within 1e-4 of its RMS.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.oracle as O
from mixture_experts_layer_34_b200 import ep
from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import oracle_gate, oracle_outputs, routing_agreement, run_forward, tolerance

pytestmark = pytest.mark.gpu

SUM_ORDER_TOL = 1e-4


def _rank_partial(layer, inp, cfg, rank, world, ws):
    E, S, T = layer.n_experts, layer.n_shared, layer.T
    eb, ee = ep.expert_range(E, world, rank)
    sb, se = ep.token_range(T, world, rank)
    w1, w3, w2 = (ep.local_stack(inp[k], E, S, eb, ee) for k in ("w1", "w3", "w2"))
    part = torch.full((T, layer.dim), float("nan"), device="cuda")
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device="cuda")
    w = torch.empty((T, layer.topk), dtype=torch.float32, device="cuda")
    K.kt_moe_forward_local(cfg, T, inp["x"], inp["w_gate"], inp["bias"], eb, ee, sb, se, w1, w3,
                           w2, part, idx, w, ws)
    assert K.kt_moe_check(ws) == K.KT_OK
    return dict(part=part, idx=idx, w=w, eb=eb, ee=ee, sb=sb, se=se)


def _finish(layer, inp, y_sum, y_fp32):
    cfg = K.config_for(layer, y_fp32=y_fp32)
    dt = torch.float32 if y_fp32 or layer.dtype == "f32" else torch.bfloat16
    y = torch.full((layer.T, layer.dim), float("nan"), dtype=dt, device="cuda")
    K.kt_moe_ep_finish(cfg, layer.T, y_sum, inp["x"], y)
    return y


def _oracle_part(layer, inp, og, eb, ee, sb, se, toks):
    """The oracle's part for tokens toks: routed [eb, ee) plus shared if in [sb, se)."""
    E, S = layer.n_experts, layer.n_shared
    need = set(range(E, E + S))
    for t in toks:
        need.update(int(e) for e in og["idx"][t] if eb <= e < ee)
    pick = lambda k: [inp[k][e].cpu() if e in need else None for e in range(E + S)]
    w1, w3, w2 = pick("w1"), pick("w3"), pick("w2")
    has_bias = inp["bias"] is not None
    yr, ys = O.forward_part(layer.kernel_fields(), inp["x"].cpu(), og["idx"], og["w"], w1, w3,
                            w2, toks, has_bias, eb, ee)
    mine = np.array([sb <= t < se for t in toks])
    return yr + ys * mine[:, None]


def _ep_check(layer, world, toks):
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer, y_fp32=True)
    ws = K.alloc_workspace(cfg, layer.T)
    full = run_forward(layer, inp, y_fp32=True)
    og = oracle_gate(layer, inp)
    diff, near = routing_agreement(layer, og, full["idx"].cpu().numpy())
    assert near[diff].all()
    keep = [t for t in toks if t not in set(diff.tolist())]
    y_ref = oracle_outputs(layer, inp, og, keep)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    tol = tolerance(layer)
    y_sum = torch.zeros((layer.T, layer.dim), device="cuda")
    sel = torch.as_tensor(keep, device="cuda")
    for rank in range(world):
        r = _rank_partial(layer, inp, cfg, rank, world, ws)
        assert torch.equal(r["idx"], full["idx"]) and torch.equal(r["w"], full["w"]), rank
        assert not torch.isnan(r["part"]).any(), rank
        ref = _oracle_part(layer, inp, og, r["eb"], r["ee"], r["sb"], r["se"], keep)
        err = float(np.abs(r["part"][sel].cpu().numpy() - ref).max())
        assert err <= tol * rms, (rank, err / rms)
        y_sum += r["part"]
    y32 = _finish(layer, inp, y_sum, True)
    err = float(np.abs(y32[sel].cpu().numpy() - y_ref).max())
    print(f"{layer.name} world {world}: max|dy|/RMS = {err / rms:.3e} over {len(keep)} tokens")
    assert err <= tol * rms
    yf = full["y"]
    frms = float(yf.square().mean().sqrt())
    assert float((y32 - yf).abs().max()) <= SUM_ORDER_TOL * frms
    if layer.dtype == "bf16":
        y16 = _finish(layer, inp, y_sum, False)
        assert torch.equal(y16, y32.to(torch.bfloat16))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", ["small_sig_bias", "small_softmax_ragged", "small_odd_dims",
                                  "small_fp32_groups"])
def test_small_layers_every_token(name, world):
    layer = W.BY_NAME[name]
    _ep_check(layer, world, list(range(layer.T)))


def test_more_ranks_than_some_ranges():
    """world 5 over 8 experts and 77 tokens: uneven splits (2,2,2,1,1)."""
    layer = W.BY_NAME["small_odd_dims"]
    _ep_check(layer, 5, list(range(layer.T)))


def test_v3_prefill_eight_ranks_sampled_tokens():
    layer = W.V3_PREFILL
    rng = np.random.default_rng(23)
    _ep_check(layer, 8, sorted(rng.choice(layer.T, 4, replace=False).tolist()))


@pytest.mark.parametrize("name", ["small_sig_bias", "small_softmax_ragged", "small_fp32_groups"])
def test_one_rank_is_the_forward_bit_for_bit(name):
    layer = W.BY_NAME[name]
    inp = W.make_layer(layer, "cuda")
    for y_fp32 in (True, False):
        full = run_forward(layer, inp, y_fp32=y_fp32)
        cfg = K.config_for(layer, y_fp32=y_fp32)
        m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                                 rank=0, world=1)
        y = torch.empty_like(full["y"])
        idx = torch.empty_like(full["idx"])
        m.forward(inp["x"], y, idx)
        assert torch.equal(idx, full["idx"])
        assert torch.equal(y, full["y"])


def test_rank_without_work_writes_zeros():
    layer = W.BY_NAME["small_sig_bias"]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    ws = K.alloc_workspace(cfg, layer.T)
    ws.fill_(0xFF)
    E, S = layer.n_experts, layer.n_shared
    part = torch.full((layer.T, layer.dim), float("nan"), device="cuda")
    w1, w3, w2 = (ep.local_stack(inp[k], E, S, 5, 5) for k in ("w1", "w3", "w2"))
    K.kt_moe_forward_local(cfg, layer.T, inp["x"], inp["w_gate"], inp["bias"], 5, 5, 7, 7, w1, w3,
                           w2, part, None, None, ws)
    assert K.kt_moe_check(ws) == K.KT_OK
    assert not part.any()


def test_local_output_does_not_depend_on_workspace_contents():
    layer = W.BY_NAME["small_softmax_ragged"]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    E, S = layer.n_experts, layer.n_shared
    w1, w3, w2 = (ep.local_stack(inp[k], E, S, 4, 11) for k in ("w1", "w3", "w2"))
    outs = []
    for fill in (0x00, 0xFF):
        ws = K.alloc_workspace(cfg, layer.T)
        ws.fill_(fill)
        part = torch.empty((layer.T, layer.dim), device="cuda")
        K.kt_moe_forward_local(cfg, layer.T, inp["x"], inp["w_gate"], inp["bias"], 4, 11, 50, 200,
                               w1, w3, w2, part, None, None, ws)
        assert K.kt_moe_check(ws) == K.KT_OK
        outs.append(part)
    assert not torch.isnan(outs[1]).any()
    assert torch.equal(outs[0], outs[1])


# ----------------------------------------------------------------------------
# MXFP8
# ----------------------------------------------------------------------------

def _group_bytes(sf, n_slots):
    """Packed scales split per weight slot (each slot's blocks are contiguous)."""
    return sf.view(n_slots, -1)


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("name", ["small_sig_bias_mxfp8", "small_softmax_mxfp8"])
def test_mxfp8_ranks_sum_to_the_forward(name, world):
    layer = W.BY_NAME[name]
    inp = W.make_layer(layer, "cuda")
    E, S, T = layer.n_experts, layer.n_shared, layer.T
    cfg = K.config_for(layer, y_fp32=True)
    qf = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    ws = K.alloc_workspace(cfg, T)
    yf = torch.empty((T, layer.dim), device="cuda")
    K.kt_moe_forward_mxfp8(cfg, T, inp["x"], inp["w_gate"], inp["bias"], qf["w1q"], qf["w3q"],
                           qf["w2q"], qf["sf_up"], qf["sf_down"], yf, None, None, ws)
    assert K.kt_moe_check(ws) == K.KT_OK
    y_sum = torch.zeros((T, layer.dim), device="cuda")
    for rank in range(world):
        eb, ee = ep.expert_range(E, world, rank)
        sb, se = ep.token_range(T, world, rank)
        loc = [ep.local_stack(inp[k], E, S, eb, ee) for k in ("w1", "w3", "w2")]
        q = K.pack_mxfp8_local(cfg, eb, ee, *loc)
        slots = list(range(eb, ee)) + list(range(E, E + S))
        for key in ("w1q", "w3q", "w2q"):
            assert torch.equal(q[key], qf[key][slots]), (rank, key)
        for key in ("sf_up", "sf_down"):
            assert torch.equal(_group_bytes(q[key], len(slots)),
                               _group_bytes(qf[key], E + S)[slots]), (rank, key)
        part = torch.full((T, layer.dim), float("nan"), device="cuda")
        K.kt_moe_forward_local_mxfp8(cfg, T, inp["x"], inp["w_gate"], inp["bias"], eb, ee, sb, se,
                                     q["w1q"], q["w3q"], q["w2q"], q["sf_up"], q["sf_down"], part,
                                     None, None, ws)
        assert K.kt_moe_check(ws) == K.KT_OK
        assert not torch.isnan(part).any()
        y_sum += part
    y = _finish(layer, inp, y_sum, True)
    rms = float(yf.square().mean().sqrt())
    err = float((y - yf).abs().max())
    print(f"{name} world {world}: max|y_ep - y|/RMS = {err / rms:.3e}")
    assert err <= SUM_ORDER_TOL * rms


def test_mxfp8_class_one_rank_is_the_forward():
    layer = W.BY_NAME["small_sig_bias_mxfp8"]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    qf = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    ws = K.alloc_workspace(cfg, layer.T)
    yf = torch.empty((layer.T, layer.dim), dtype=torch.bfloat16, device="cuda")
    K.kt_moe_forward_mxfp8(cfg, layer.T, inp["x"], inp["w_gate"], inp["bias"], qf["w1q"],
                           qf["w3q"], qf["w2q"], qf["sf_up"], qf["sf_down"], yf, None, None, ws)
    m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                             rank=0, world=1)
    y = torch.empty_like(yf)
    m.forward(inp["x"], y)
    assert torch.equal(y, yf)


# ----------------------------------------------------------------------------
# Placements other than contiguous ranges (kt_moe_forward_placed)
# ----------------------------------------------------------------------------

def _shuffled_placement(E, world, seed=9):
    perm = np.random.default_rng(seed).permutation(E).tolist()
    return [sorted(perm[r::world]) for r in range(world)]


def _oracle_set_part(layer, inp, og, experts, sb, se, toks):
    """The oracle's part for a set of routed experts: one range per expert."""
    total = np.zeros((len(toks), layer.dim))
    for e in experts:
        total += _oracle_part(layer, inp, og, e, e + 1, 0, 0, toks)
    return total + _oracle_part(layer, inp, og, 0, 0, sb, se, toks)


@pytest.mark.parametrize("name", ["small_sig_bias", "small_softmax_ragged", "small_fp32_groups"])
def test_placed_ranks_match_the_oracle(name):
    layer = W.BY_NAME[name]
    world = 3
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer, y_fp32=True)
    full = run_forward(layer, inp, y_fp32=True)
    og = oracle_gate(layer, inp)
    diff, near = routing_agreement(layer, og, full["idx"].cpu().numpy())
    assert near[diff].all()
    toks = [t for t in range(layer.T) if t not in set(diff.tolist())]
    sel = torch.as_tensor(toks, device="cuda")
    y_ref = oracle_outputs(layer, inp, og, toks)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    placement = _shuffled_placement(layer.n_experts, world)
    y_sum = torch.zeros((layer.T, layer.dim), device="cuda")
    for rank in range(world):
        m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                                 rank, world, placement=placement)
        ws, part = m.buffers(layer.T, inp["x"].device)
        part.fill_(float("nan"))
        idx = torch.empty_like(full["idx"])
        m.local(inp["x"], part, idx)
        assert K.kt_moe_check(ws) == K.KT_OK
        assert torch.equal(idx, full["idx"])
        sb, se = m.shared_range(layer.T)
        ref = _oracle_set_part(layer, inp, og, m.experts, sb, se, toks)
        err = float(np.abs(part[sel].cpu().numpy() - ref).max())
        assert err <= tolerance(layer) * rms, (rank, err / rms)
        y_sum += part
    y = _finish(layer, inp, y_sum, True)
    assert float(np.abs(y[sel].cpu().numpy() - y_ref).max()) <= tolerance(layer) * rms
    frms = float(full["y"].square().mean().sqrt())
    assert float((y - full["y"]).abs().max()) <= SUM_ORDER_TOL * frms


def test_mxfp8_placed_ranks_sum_to_the_forward():
    layer = W.BY_NAME["small_sig_bias_mxfp8"]
    world = 4
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer, y_fp32=True)
    qf = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    ws = K.alloc_workspace(cfg, layer.T)
    yf = torch.empty((layer.T, layer.dim), device="cuda")
    K.kt_moe_forward_mxfp8(cfg, layer.T, inp["x"], inp["w_gate"], inp["bias"], qf["w1q"],
                           qf["w3q"], qf["w2q"], qf["sf_up"], qf["sf_down"], yf, None, None, ws)
    placement = _shuffled_placement(layer.n_experts, world, seed=4)
    y_sum = torch.zeros((layer.T, layer.dim), device="cuda")
    for rank in range(world):
        m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                                 rank, world, placement=placement)
        _, part = m.buffers(layer.T, inp["x"].device)
        m.local(inp["x"], part)
        y_sum += part
    y = _finish(layer, inp, y_sum, True)
    rms = float(yf.square().mean().sqrt())
    assert float((y - yf).abs().max()) <= SUM_ORDER_TOL * rms


@pytest.mark.parametrize("name", ["small_sig_bias", "small_sig_bias_mxfp8"])
def test_graph_replay_is_the_eager_step(name):
    """The captured step (local forward + finish; one rank, so no all-reduce)
    replays to the eager step's output bit for bit, and follows new x."""
    layer = W.BY_NAME[name]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    placement = _shuffled_placement(layer.n_experts, 1)
    m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                             0, 1, placement=placement)
    x = inp["x"].clone()
    y = torch.empty((layer.T, layer.dim), dtype=torch.bfloat16, device="cuda")
    g = m.graph(x, y)
    ref = torch.empty_like(y)
    for step in range(3):
        x.copy_(inp["x"] * (1.0 + 0.25 * step))
        g.replay()
        m.forward(x, ref)
        torch.cuda.synchronize()
        assert torch.equal(y, ref), step


def test_sharded_finish_is_the_full_finish_on_each_share():
    """forward_shard with one rank equals forward; with the partials of 4 ranks
    summed, finishing each rank's token share (x offset into its rows) gives
    the rows of the full finish, bit for bit."""
    layer = W.BY_NAME["small_odd_dims"]           # residual on: the finish reads x rows
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    T = 76                                          # a multiple of 4 (the layer has 77)
    x = inp["x"][:T].contiguous()
    m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                             0, 1)
    y = torch.empty((T, layer.dim), dtype=torch.bfloat16, device="cuda")
    ys = torch.empty_like(y)
    m.forward(x, y)
    m.forward_shard(x, ys)
    assert torch.equal(y, ys)
    world = 4
    y_sum = torch.zeros((T, layer.dim), device="cuda")
    for rank in range(world):
        r = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"],
                                 inp["w2"], rank, world)
        _, part = r.buffers(T, x.device)
        r.local(x, part)
        y_sum += part
    full = torch.empty_like(y)
    K.kt_moe_ep_finish(cfg, T, y_sum, x, full)
    for rank in range(world):
        sb, se = ep.token_range(T, world, rank)
        shard = torch.empty((se - sb, layer.dim), dtype=torch.bfloat16, device="cuda")
        m.finish_rows(y_sum[sb:se].contiguous(), x[sb:se], shard)
        assert torch.equal(shard, full[sb:se]), rank
