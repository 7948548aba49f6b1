"""Pins of the oracle to things other than itself (CPU only).

Each test checks the oracle against what the pages or the mathematics fix:
hand-worked examples, brute-force enumeration on tiny inputs, closed forms,
library routines for special cases, and invariants. The gate steps follow the
DeepSeek-V3 model.py notes (73biji.xyz/llm_pp_dsv3), "Gate 选专家流程（model.py，五步）";
the forward follows the same page's "MoE 前向四步" and the total-output equation
of its "DeepSeekMoE 三改进" passage.
"""
from __future__ import annotations

import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy import special

import oracle.oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _cfg(**kw):
    base = dict(n_experts=8, n_groups=1, topk_groups=1, topk=2, route_scale=1.0, score_func=0,
                dim=16, inter=8, n_shared=0, norm_topk=-1, group_score=0, add_residual=0)
    base.update(kw)
    return base


# ----------------------------------------------------------------------------
# Hand-worked examples (tests/golden/gate_worked_examples.json)
# ----------------------------------------------------------------------------

def test_worked_examples():
    doc = json.load(open(os.path.join(GOLDEN, "gate_worked_examples.json")))
    for ex in doc["examples"]:
        s = np.array([ex["scores"]], np.float32)
        b = None if ex["bias"] is None else np.array(ex["bias"], np.float32)
        r = O.select(ex["cfg"], s, b)
        assert r["idx"][0].tolist() == ex["idx"], ex["name"]
        assert r["w"][0].tolist() == ex["w"], ex["name"]
        assert r["gsc"][0].tolist() == ex["group_scores"], ex["name"]


# ----------------------------------------------------------------------------
# Brute force over group and expert subsets (tiny configs)
# ----------------------------------------------------------------------------

def _brute_select(s, bias, cfg):
    """Enumerate every subset; exact (Fraction) sums; lexicographic tie order."""
    E, G, TG, k = cfg["n_experts"], cfg["n_groups"], cfg["topk_groups"], cfg["topk"]
    rc = O.resolve(cfg, bias is not None)
    key = s if bias is None else (s + bias).astype(np.float32)
    gs = E // G
    if G > 1:
        def gscore(g):
            vals = [key[e] for e in range(g * gs, (g + 1) * gs)]
            if rc["group_score"] == O.AMAX:
                return max(vals)
            # "sum of the two largest" == the largest sum over pairs
            return max(np.float32(vals[i] + vals[j])
                       for i in range(gs) for j in range(i + 1, gs))
        gsc = [gscore(g) for g in range(G)]
        best, best_tot = None, None
        for sub in itertools.combinations(range(G), TG):   # lexicographic order
            tot = sum(Fraction(float(gsc[g])) for g in sub)
            if best is None or tot > best_tot:
                best, best_tot = sub, tot
        allowed = [e for e in range(E) if e // gs in best]
    else:
        allowed = list(range(E))
    best, best_tot = None, None
    for sub in itertools.combinations(allowed, k):
        tot = sum(Fraction(float(key[e])) for e in sub)
        if best is None or tot > best_tot:
            best, best_tot = sub, tot
    order = sorted(best, key=lambda e: (-Fraction(float(key[e])), e))
    return order


TINY_CFGS = [
    _cfg(n_experts=16, n_groups=4, topk_groups=2, topk=4),                  # the tiny layer's shape
    _cfg(n_experts=8, n_groups=4, topk_groups=2, topk=2),
    _cfg(n_experts=12, n_groups=3, topk_groups=1, topk=3),
    _cfg(n_experts=12, n_groups=3, topk_groups=2, topk=5, score_func=1),   # softmax, amax
    _cfg(n_experts=10, n_groups=1, topk_groups=1, topk=3),
    _cfg(n_experts=9, n_groups=3, topk_groups=3, topk=4, group_score=1),   # all groups kept
]


@pytest.mark.parametrize("ci", range(len(TINY_CFGS)))
@pytest.mark.parametrize("with_bias", [False, True])
def test_select_matches_bruteforce(ci, with_bias):
    cfg = TINY_CFGS[ci]
    rng = np.random.default_rng(100 + ci * 2 + with_bias)
    T, E = 40, cfg["n_experts"]
    s = rng.random((T, E)).astype(np.float32)
    bias = rng.normal(0, 0.1, E).astype(np.float32) if with_bias else None
    r = O.select(cfg, s, bias)
    for t in range(T):
        assert r["idx"][t].tolist() == _brute_select(s[t], bias, cfg), t


@pytest.mark.parametrize("ci", range(len(TINY_CFGS)))
def test_select_bruteforce_with_exact_ties(ci):
    """Scores on a coarse dyadic grid: many exact ties, all resolved by index."""
    cfg = TINY_CFGS[ci]
    rng = np.random.default_rng(7 + ci)
    T, E = 60, cfg["n_experts"]
    s = (rng.integers(1, 6, (T, E)) / 8.0).astype(np.float32)
    bias = (rng.integers(-2, 3, E) / 16.0).astype(np.float32)
    for b in (None, bias):
        r = O.select(cfg, s, b)
        for t in range(T):
            assert r["idx"][t].tolist() == _brute_select(s[t], b, cfg), t


# ----------------------------------------------------------------------------
# Library routines for the special cases
# ----------------------------------------------------------------------------

def test_logits_match_float64_matmul():
    rng = np.random.default_rng(1)
    cfg = _cfg(n_experts=24, dim=200)
    x = rng.normal(size=(50, 200)).astype(np.float32)
    wg = (rng.normal(size=(24, 200)) * 0.05).astype(np.float32)
    l = O.gate_logits(cfg, x, wg)
    ref = (x.astype(np.float64) @ wg.astype(np.float64).T).astype(np.float32)
    ulp = np.abs(l.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1


def test_logits_bf16_inputs_match_float64_matmul():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(33, 136, generator=g).to(torch.bfloat16)
    wg = (torch.randn(20, 136, generator=g) * 0.02).to(torch.bfloat16)
    cfg = _cfg(n_experts=20, dim=136)
    l = O.gate_logits(cfg, x, wg)
    ref = (x.double() @ wg.double().T).float().numpy()
    ulp = np.abs(l.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1


def test_sigmoid_and_softmax_match_scipy():
    rng = np.random.default_rng(2)
    l = (rng.normal(size=(64, 37)) * 3).astype(np.float32)
    sig = O.scores(_cfg(n_experts=37, score_func=0), l)
    ref = special.expit(l.astype(np.float64)).astype(np.float32)
    assert np.abs(sig.view(np.int32) - ref.view(np.int32)).max() <= 1
    sm = O.scores(_cfg(n_experts=37, score_func=1), l)
    ref = special.softmax(l.astype(np.float64), axis=1).astype(np.float32)
    assert np.abs(sm.view(np.int32) - ref.view(np.int32)).max() <= 1
    assert np.abs(sm.astype(np.float64).sum(1) - 1).max() < 1e-6


def test_plain_top2_sketch_is_torch_topk():
    """G=1, no bias, no shared expert: the plain top-2 routing sketch of the
    Baidu cloud article ('动态路由算法伪代码示例') — idx is torch.topk, weights
    are the gathered scores."""
    rng = np.random.default_rng(4)
    s = rng.random((100, 10)).astype(np.float32)
    cfg = _cfg(n_experts=10, topk=2, score_func=1, norm_topk=0)
    r = O.select(cfg, s, None)
    tv, ti = torch.topk(torch.from_numpy(s), 2, dim=1)
    assert np.array_equal(r["idx"], ti.numpy().astype(np.int32))
    assert np.array_equal(r["w"], tv.numpy())


def test_sigmoid_no_groups_is_topk_of_biased_scores():
    rng = np.random.default_rng(5)
    s = rng.random((100, 16)).astype(np.float32)
    b = rng.normal(0, 0.1, 16).astype(np.float32)
    cfg = _cfg(n_experts=16, topk=4, route_scale=2.5)
    r = O.select(cfg, s, b)
    ti = torch.topk(torch.from_numpy(s) + torch.from_numpy(b), 4, dim=1).indices.numpy()
    assert np.array_equal(r["idx"], ti.astype(np.int32))
    g = np.take_along_axis(s, ti, 1)
    ref = (g / g.sum(1, keepdims=True)) * 2.5
    assert np.allclose(r["w"], ref, rtol=1e-6, atol=0)


# ----------------------------------------------------------------------------
# Invariants of the gate
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("ci", range(len(TINY_CFGS)))
def test_gate_invariants(ci):
    cfg = dict(TINY_CFGS[ci], route_scale=2.5)
    rng = np.random.default_rng(50 + ci)
    T, E, G = 200, cfg["n_experts"], cfg["n_groups"]
    l = rng.normal(0, 2, (T, E)).astype(np.float32)
    s = O.scores(cfg, l)
    b = rng.normal(0, 0.1, E).astype(np.float32) if cfg["score_func"] == 0 else None
    r = O.select(cfg, s, b)
    rc = O.resolve(cfg, b is not None)
    gs = E // G
    key = s + (b if b is not None else 0)
    for t in range(T):
        idx = r["idx"][t]
        assert len(set(idx.tolist())) == len(idx)
        if G > 1:
            kept = np.argsort(-r["gsc"][t], kind="stable")[: cfg["topk_groups"]]
            assert all((e // gs) in kept for e in idx)
            allowed = [e for e in range(E) if e // gs in kept]
        else:
            allowed = list(range(E))
        rest = [e for e in allowed if e not in idx]
        if rest:
            assert key[t, idx].min() >= key[t, rest].max()
        assert (r["w"][t] > 0).all()
        if rc["norm_topk"]:
            assert abs(float(r["w"][t].astype(np.float64).sum()) - 2.5) < 1e-5
        else:
            assert np.array_equal(r["w"][t], (s[t, idx] * np.float32(2.5)).astype(np.float32))
    if cfg["score_func"] == 1:
        assert np.abs(s.astype(np.float64).sum(1) - 1).max() < 1e-6


def test_bias_shift_keeps_selection_up_to_near_ties():
    cfg = _cfg(n_experts=16, n_groups=4, topk_groups=2, topk=4, route_scale=2.5)
    rng = np.random.default_rng(9)
    s = O.scores(cfg, rng.normal(0, 2, (500, 16)).astype(np.float32))
    b = rng.normal(0, 0.1, 16).astype(np.float32)
    r0 = O.select(cfg, s, b)
    r1 = O.select(cfg, s, (b + np.float32(0.25)).astype(np.float32))
    clear = (r0["kth_margin"] > 1e-5) & (r0["grp_margin"] > 1e-5)
    assert clear.mean() > 0.95
    assert np.array_equal(r0["idx"][clear], r1["idx"][clear])


# ----------------------------------------------------------------------------
# The forward: textbook reduction, linearity, shared-expert merge, relabelling
# ----------------------------------------------------------------------------

def _rand_layer(rng, E, S, d, I, T):
    x = rng.normal(size=(T, d)).astype(np.float32)
    wg = (rng.normal(size=(E, d)) / np.sqrt(d)).astype(np.float32)
    w1 = (rng.normal(size=(E + S, I, d)) / np.sqrt(d)).astype(np.float32)
    w3 = (rng.normal(size=(E + S, I, d)) / np.sqrt(d)).astype(np.float32)
    w2 = (rng.normal(size=(E + S, d, I)) / np.sqrt(I)).astype(np.float32)
    return x, wg, w1, w3, w2


def _swiglu_torch(x, w1, w3, w2):
    x, w1, w3, w2 = (torch.from_numpy(np.asarray(a, np.float64)) for a in (x, w1, w3, w2))
    return ((F.silu(x @ w1.T) * (x @ w3.T)) @ w2.T).numpy()


def test_single_expert_weight_one_is_textbook_swiglu():
    """k=1, G=1, renormalised: the token's one weight is exactly 1, so the layer
    is that expert's SwiGLU FFN, checked against torch.nn.functional."""
    rng = np.random.default_rng(11)
    E, d, I, T = 4, 64, 48, 6
    x, wg, w1, w3, w2 = _rand_layer(rng, E, 0, d, I, T)
    cfg = _cfg(n_experts=E, topk=1, dim=d, inter=I, route_scale=1.0, norm_topk=1)
    for target in range(E):
        bias = np.full(E, -20.0, np.float32)
        bias[target] = 20.0
        gt = O.gate(cfg, x, wg, bias)
        assert (gt["idx"] == target).all() and (gt["w"] == 1.0).all()
        y = O.forward(cfg, x, gt["idx"], gt["w"], w1, w3, w2, range(T), True)
        ref = _swiglu_torch(x, w1[target], w3[target], w2[target])
        assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()


def test_expert_hidden_is_textbook():
    rng = np.random.default_rng(12)
    x, wg, w1, w3, w2 = _rand_layer(rng, 2, 0, 40, 24, 5)
    cfg = _cfg(n_experts=2, dim=40, inter=24)
    h = O.expert_hidden(cfg, x, w1[1], w3[1], range(5))
    xt = torch.from_numpy(x.astype(np.float64))
    ref = (F.silu(xt @ torch.from_numpy(w1[1].astype(np.float64)).T)
           * (xt @ torch.from_numpy(w3[1].astype(np.float64)).T)).numpy()
    assert np.abs(h - ref).max() <= 1e-12 * np.abs(ref).max()


def test_forward_is_gate_weighted_sum_of_experts():
    """Full layer = shared FFNs + sum_j w_j FFN_{idx_j}, each FFN from torch."""
    rng = np.random.default_rng(13)
    E, S, d, I, T = 8, 2, 32, 24, 7
    x, wg, w1, w3, w2 = _rand_layer(rng, E, S, d, I, T)
    cfg = _cfg(n_experts=E, n_groups=4, topk_groups=2, topk=3, dim=d, inter=I, n_shared=S,
               route_scale=2.5)
    b = rng.normal(0, 0.1, E).astype(np.float32)
    gt = O.gate(cfg, x, wg, b)
    y = O.forward(cfg, x, gt["idx"], gt["w"], w1, w3, w2, range(T), True)
    for t in range(T):
        ref = sum(_swiglu_torch(x[t:t + 1], w1[E + s], w3[E + s], w2[E + s])[0] for s in range(S))
        for j in range(3):
            e = gt["idx"][t, j]
            ref = ref + float(gt["w"][t, j]) * _swiglu_torch(x[t:t + 1], w1[e], w3[e], w2[e])[0]
        assert np.abs(y[t] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_residual_adds_input():
    rng = np.random.default_rng(14)
    x, wg, w1, w3, w2 = _rand_layer(rng, 4, 1, 16, 8, 5)
    cfg = _cfg(n_experts=4, topk=2, dim=16, inter=8, n_shared=1)
    gt = O.gate(cfg, x, wg, None)
    y0 = O.forward(cfg, x, gt["idx"], gt["w"], w1, w3, w2, range(5), False)
    y1 = O.forward(dict(cfg, add_residual=1), x, gt["idx"], gt["w"], w1, w3, w2, range(5), False)
    assert np.abs(y1 - y0 - x).max() <= 1e-12 * np.abs(y1).max()


def test_linearity_in_w2_and_route_scale():
    rng = np.random.default_rng(15)
    E, d, I, T = 8, 24, 16, 9
    x, wg, w1, w3, w2 = _rand_layer(rng, E, 0, d, I, T)
    cfg = _cfg(n_experts=E, n_groups=2, topk_groups=1, topk=3, dim=d, inter=I, route_scale=1.0)
    b = rng.normal(0, 0.1, E).astype(np.float32)
    g1 = O.gate(cfg, x, wg, b)
    y = O.forward(cfg, x, g1["idx"], g1["w"], w1, w3, w2, range(T), True)
    y_w2 = O.forward(cfg, x, g1["idx"], g1["w"], w1, w3, 2 * w2, range(T), True)
    assert np.array_equal(y_w2, 2 * y)
    g2 = O.gate(dict(cfg, route_scale=2.0), x, wg, b)
    assert np.array_equal(g2["w"], 2 * g1["w"])
    y_rs = O.forward(cfg, x, g2["idx"], g2["w"], w1, w3, w2, range(T), True)
    assert np.array_equal(y_rs, 2 * y)


def test_two_shared_experts_equal_one_of_double_width():
    rng = np.random.default_rng(16)
    E, d, I, T = 6, 20, 12, 8
    x, wg, w1, w3, w2 = _rand_layer(rng, E, 2, d, I, T)
    cfg = _cfg(n_experts=E, topk=2, dim=d, inter=I, n_shared=2, score_func=1)
    gt = O.gate(cfg, x, wg, None)
    y2 = O.forward(cfg, x, gt["idx"], gt["w"], w1, w3, w2, range(T), False)
    # one shared expert of width 2I: concatenated rows of W1/W3, columns of W2
    cfgm = dict(cfg, n_shared=1, inter=2 * I)
    pad = np.zeros((E, I, d), np.float32)
    w1m = [np.concatenate([w1[e], pad[e]]) for e in range(E)] + [np.concatenate([w1[E], w1[E + 1]])]
    w3m = [np.concatenate([w3[e], pad[e]]) for e in range(E)] + [np.concatenate([w3[E], w3[E + 1]])]
    w2m = [np.concatenate([w2[e], np.zeros((d, I), np.float32)], 1) for e in range(E)] + \
          [np.concatenate([w2[E], w2[E + 1]], 1)]
    y1 = O.forward(cfgm, x, gt["idx"], gt["w"], w1m, w3m, w2m, range(T), False)
    assert np.abs(y1 - y2).max() <= 1e-12 * np.abs(y2).max()


def test_relabelling_experts_within_and_across_groups():
    rng = np.random.default_rng(17)
    E, G, d, I, T = 12, 3, 16, 8, 30
    x, wg, w1, w3, w2 = _rand_layer(rng, E, 1, d, I, T)
    cfg = _cfg(n_experts=E, n_groups=G, topk_groups=2, topk=3, dim=d, inter=I, n_shared=1,
               route_scale=2.5)
    b = rng.normal(0, 0.1, E).astype(np.float32)
    g0 = O.gate(cfg, x, wg, b)
    y0 = O.forward(cfg, x, g0["idx"], g0["w"], w1, w3, w2, range(T), True)
    gs = E // G
    gperm = rng.permutation(G)
    perm = np.concatenate([gperm[g] * gs + rng.permutation(gs) for g in range(G)])  # new e -> old
    full = np.concatenate([perm, [E]])
    g1 = O.gate(cfg, x, wg[perm], b[perm])
    assert np.array_equal(perm[g1["idx"]], g0["idx"])
    y1 = O.forward(cfg, x, g1["idx"], g1["w"], w1[full], w3[full], w2[full], range(T), True)
    assert np.array_equal(y0, y1)
