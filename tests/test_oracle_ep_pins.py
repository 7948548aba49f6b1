"""Pins of the oracle's expert-parallel part (CPU only).

``forward_part`` is one rank's share of the multi-card form of "MoE 前向四步"
(DeepSeek-V3 model.py notes, 73biji.xyz/llm_pp_dsv3): the routed experts of a
range, and the shared experts. It is pinned to the pinned full forward through
what the split must preserve: over any partition of the experts into ranges,
the parts sum to the forward (the residual added once); a range holding no
picked expert gives exact zeros; and a range of one expert gives that expert's
weighted term alone, which is the forward of a layer whose other picks carry
weight zero.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.oracle as O


def _cfg(**kw):
    base = dict(n_experts=8, n_groups=1, topk_groups=1, topk=3, route_scale=1.0, score_func=0,
                dim=64, inter=48, n_shared=2, norm_topk=-1, group_score=0, add_residual=0)
    base.update(kw)
    return base


def _layer(cfg, T, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    E, S, d, I = cfg["n_experts"], cfg["n_shared"], cfg["dim"], cfg["inter"]
    x = torch.randn(T, d, generator=g).to(dtype)
    w1 = (torch.randn(E + S, I, d, generator=g) * 0.1).to(dtype)
    w3 = (torch.randn(E + S, I, d, generator=g) * 0.1).to(dtype)
    w2 = (torch.randn(E + S, d, I, generator=g) * 0.1).to(dtype)
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, cfg["topk"], replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.05, 1.0, (T, cfg["topk"])).astype(np.float32)
    return x, w1, w3, w2, idx, w


def _partitions(E):
    yield [(0, E)]
    yield [(0, E // 2), (E // 2, E)]
    yield [(0, 3), (3, 3), (3, 7), (7, E)]          # an empty range in the middle
    yield [(e, e + 1) for e in range(E)]


@pytest.mark.parametrize("residual", [0, 1])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_parts_over_a_partition_sum_to_the_forward(residual, dtype):
    cfg = _cfg(add_residual=residual)
    T = 24
    x, w1, w3, w2, idx, w = _layer(cfg, T, 7, dtype)
    toks = list(range(T))
    y = O.forward(cfg, x, idx, w, w1, w3, w2, toks, False)
    for parts in _partitions(cfg["n_experts"]):
        total = np.zeros_like(y)
        # shared experts on a split of the tokens, one share per range
        bounds = np.linspace(0, T, len(parts) + 1).astype(int)
        for r, (b, e) in enumerate(parts):
            yr, _ = O.forward_part(cfg, x, idx, w, w1, w3, w2, toks, False, b, e, shared=False)
            total += yr
            mine = list(range(bounds[r], bounds[r + 1]))
            if mine:
                _, ys = O.forward_part(cfg, x, idx, w, w1, w3, w2, mine, False, b, e)
                total[mine] += ys
        if residual:
            total += x.to(torch.float64).numpy()
        np.testing.assert_allclose(total, y, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_range_without_picks_is_exactly_zero():
    cfg = _cfg()
    T = 10
    x, w1, w3, w2, idx, w = _layer(cfg, T, 8)
    idx[:] = np.array([0, 1, 2], np.int32)            # every token picks experts 0..2
    yr, ys = O.forward_part(cfg, x, idx, w, w1, w3, w2, range(T), False, 3, 8)
    assert not yr.any()
    yr, _ = O.forward_part(cfg, x, idx, w, w1, w3, w2, range(T), False, 4, 4)
    assert not yr.any()
    # The shared part does not depend on the range.
    _, ys2 = O.forward_part(cfg, x, idx, w, w1, w3, w2, range(T), False, 0, 8)
    assert np.array_equal(ys, ys2)


def test_one_expert_range_is_that_experts_weighted_term():
    """forward_part over [e, e + 1) equals the forward of the same layer with
    every other pick's weight set to zero and no shared experts."""
    cfg = _cfg()
    T = 16
    x, w1, w3, w2, idx, w = _layer(cfg, T, 9)
    cfg0 = dict(cfg, n_shared=0)
    for e in range(cfg["n_experts"]):
        yr, _ = O.forward_part(cfg, x, idx, w, w1, w3, w2, range(T), False, e, e + 1,
                               shared=False)
        w_only = np.where(idx == e, w, 0.0).astype(np.float32)
        ref = O.forward(cfg0, x, idx, w_only, w1[:8], w3[:8], w2[:8], range(T), False)
        np.testing.assert_allclose(yr, ref, rtol=1e-13, atol=1e-15)


def test_shared_part_is_the_forward_without_routed_picks():
    """y_shared = the forward with every routed weight zero."""
    cfg = _cfg()
    T = 12
    x, w1, w3, w2, idx, w = _layer(cfg, T, 10)
    _, ys = O.forward_part(cfg, x, idx, w, w1, w3, w2, range(T), False, 0, 0)
    ref = O.forward(cfg, x, idx, np.zeros_like(w), w1, w3, w2, range(T), False)
    np.testing.assert_allclose(ys, ref, rtol=1e-13, atol=1e-15)


def test_bad_token_id_raises():
    cfg = _cfg()
    x, w1, w3, w2, idx, w = _layer(cfg, 4, 11)
    with pytest.raises(ValueError):
        O.forward_part(cfg, x, idx, w, w1, w3, w2, [4], False, 0, 8)
