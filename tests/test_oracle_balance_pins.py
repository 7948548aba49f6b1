"""Pins of the oracle's load statistics (CPU only): expert load, the
aux-loss-free bias update and the sequence-wise balance statistics.

Sources: the DeepSeek-V3 model.py notes (73biji.xyz/llm_pp_dsv3), "V3 改进①：
无辅助损失负载均衡" (the bias follows each expert's load, at a speed gamma; an
overloaded expert's bias goes down, an underloaded one's up, as the Baidu cloud
article also puts it) and "V3 改进②：序列级平衡损失" (L_Bal = alpha * sum f_i P_i).
The pins are hand-worked examples, numpy's bincount, exact rational arithmetic
on tiny inputs, closed forms and invariants.
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle.oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _cfg(E, k):
    return dict(n_experts=E, n_groups=1, topk_groups=1, topk=k, route_scale=1.0, score_func=0,
                dim=8, inter=8, n_shared=0)


def _golden():
    with open(os.path.join(GOLDEN, "balance_worked_examples.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("i", range(3))
def test_bias_update_worked_examples(i):
    ex = _golden()["bias_update"][i]
    got = O.bias_update(_cfg(ex["n_experts"], ex["topk"]), np.array(ex["idx"], np.int32),
                        ex["gamma"], np.array(ex["bias"], np.float32))
    assert got.tolist() == ex["expected"], ex["note"]


@pytest.mark.parametrize("i", range(2))
def test_balance_worked_examples(i):
    ex = _golden()["balance"][i]
    s = np.array(ex["scores"], np.float32)
    out = O.balance_stats(_cfg(s.shape[1], ex["topk"]), s, np.array(ex["idx"], np.int32),
                          ex["alpha"])
    assert out["f"].tolist() == ex["f"]
    assert out["P"].tolist() == ex["P"]
    assert abs(out["loss"] - ex["loss"]) <= 1e-15


def _random_routing(rng, T, E, k):
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (37, 16, 4), (256, 64, 6), (500, 256, 8)])
def test_load_is_numpy_bincount(T, E, k):
    rng = np.random.default_rng(T + E)
    idx = _random_routing(rng, T, E, k)
    got = O.expert_load(_cfg(E, k), idx)
    assert np.array_equal(got, np.bincount(idx.ravel(), minlength=E))
    assert got.sum() == T * k


def test_load_rejects_out_of_range_index():
    with pytest.raises(ValueError):
        O.expert_load(_cfg(4, 1), np.array([[0], [4]], np.int32))


@pytest.mark.parametrize("T,E,k", [(3, 4, 2), (50, 16, 4), (333, 64, 6), (1000, 256, 8)])
def test_bias_update_moves_each_bias_by_gamma_against_its_load(T, E, k):
    """Each bias moves by exactly one fp32 addition of -gamma (load above the
    mean T*k/E, decided in exact rationals here), +gamma (below) or not at all."""
    rng = np.random.default_rng(7 * T + E)
    idx = _random_routing(rng, T, E, k)
    bias = rng.normal(0, 0.1, E).astype(np.float32)
    gamma = np.float32(1e-3)
    got = O.bias_update(_cfg(E, k), idx, float(gamma), bias)
    load = np.bincount(idx.ravel(), minlength=E)
    mean = Fraction(T * k, E)
    for e in range(E):
        if Fraction(int(load[e])) > mean:
            want = np.float32(bias[e] - gamma)
        elif Fraction(int(load[e])) < mean:
            want = np.float32(bias[e] + gamma)
        else:
            want = bias[e]
        assert got[e] == want, (e, load[e], mean)


def test_bias_update_lowers_the_overloaded_and_raises_the_underloaded():
    """Every token picks experts 0 and 1 of 4: they are overloaded (T each
    against a mean of T/2), experts 2 and 3 idle."""
    T = 10
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    got = O.bias_update(_cfg(4, 2), idx, 0.25, np.zeros(4, np.float32))
    assert got.tolist() == [-0.25, -0.25, 0.25, 0.25]


def _exact_stats(s, idx, alpha):
    T, E = s.shape
    f = [Fraction(0)] * E
    P = [Fraction(0)] * E
    for t in range(T):
        z = sum(Fraction(float(v)) for v in s[t])
        for e in range(E):
            P[e] += Fraction(float(s[t, e])) / z
        for e in idx[t]:
            f[int(e)] += 1
    f = [v / T for v in f]
    P = [v / T for v in P]
    loss = Fraction(alpha) * sum(a * b for a, b in zip(f, P))
    return f, P, loss


@pytest.mark.parametrize("T,E,k", [(1, 3, 1), (5, 6, 2), (9, 8, 3)])
def test_balance_stats_match_exact_rationals(T, E, k):
    rng = np.random.default_rng(100 + T)
    s = rng.uniform(0.01, 1.0, (T, E)).astype(np.float32)
    idx = _random_routing(rng, T, E, k)
    out = O.balance_stats(_cfg(E, k), s, idx, 0.0625)
    f, P, loss = _exact_stats(s, idx, 0.0625)
    assert np.allclose(out["f"], [float(v) for v in f], rtol=0, atol=1e-15)
    assert np.allclose(out["P"], [float(v) for v in P], rtol=1e-14, atol=0)
    assert abs(out["loss"] - float(loss)) <= 1e-14 * abs(float(loss))


@pytest.mark.parametrize("T,E,k", [(64, 16, 4), (512, 256, 8)])
def test_balance_stats_closed_forms(T, E, k):
    rng = np.random.default_rng(T)
    idx = _random_routing(rng, T, E, k)
    s = rng.uniform(0.01, 1.0, (T, E)).astype(np.float32)
    out = O.balance_stats(_cfg(E, k), s, idx, 1.0)
    assert abs(out["f"].sum() - k) <= 1e-12          # each token picks k experts
    assert abs(out["P"].sum() - 1.0) <= 1e-12        # normalised affinities sum to 1
    # Equal scores: P_i = 1/E whatever the routing.
    u = O.balance_stats(_cfg(E, k), np.full((T, E), 0.3, np.float32), idx, 1.0)
    assert np.allclose(u["P"], 1.0 / E, rtol=1e-14, atol=0)
    # Perfectly balanced routing (token t picks experts t*k .. t*k+k-1 mod E,
    # T*k a multiple of E): f_i = k/E, so with equal scores L = alpha * k / E.
    bal = ((np.arange(T)[:, None] * k + np.arange(k)[None, :]) % E).astype(np.int32)
    b = O.balance_stats(_cfg(E, k), np.full((T, E), 0.3, np.float32), bal, 0.5)
    assert np.allclose(b["f"], k / E, rtol=0, atol=1e-15)
    assert abs(b["loss"] - 0.5 * k / E) <= 1e-14


def test_balance_P_is_invariant_to_scaling_a_token_scores():
    rng = np.random.default_rng(3)
    s = rng.uniform(0.01, 1.0, (20, 8)).astype(np.float32)
    idx = _random_routing(rng, 20, 8, 2)
    a = O.balance_stats(_cfg(8, 2), s, idx, 1.0)
    s2 = s.copy()
    s2[::2] *= np.float32(4.0)        # exact in fp32
    b = O.balance_stats(_cfg(8, 2), s2, idx, 1.0)
    assert np.allclose(a["P"], b["P"], rtol=1e-15, atol=0)
    assert np.array_equal(a["f"], b["f"])
