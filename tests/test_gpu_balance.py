"""GPU parity of the load statistics, through the C ABI: kt_moe_scores,
kt_moe_bias_update and kt_moe_balance_stats against the oracle.

The bias update is integer counting plus one fp32 addition per expert, so it
must be bit-exact. f_i = load_i / T is an exact count divided once in fp32, so
it is compared for equality with the oracle's value rounded to fp32. P_i and
the loss sum T fp32 quotients in blocks (at most 4 per warp chain, 8 warps, then
at most 512 chunks): the rounding bound is about (T / 512 + 12) * 2^-24
relative, under 1e-5 for every T here, so they are checked at rtol 2e-5.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.oracle as O
from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import oracle_gate

pytestmark = pytest.mark.gpu

ODD_E = W.BY_NAME["small_sig_bias"].with_(name="small_E30", n_experts=30, n_groups=3)


def _random_idx(rng, T, E, k):
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("layer", [W.BY_NAME["small_sig_bias"], W.BY_NAME["small_softmax_ragged"],
                                   ODD_E, W.V2_LITE, W.V3_DECODE], ids=lambda c: c.name)
def test_scores_match_oracle_and_reproduce_the_gate(layer):
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    T, E = layer.T, layer.n_experts
    ws = K.alloc_workspace(cfg, T)
    s = torch.full((T, E), float("nan"), device="cuda")
    K.kt_moe_scores(cfg, T, inp["x"], inp["w_gate"], s, ws)
    assert K.kt_moe_check(ws) == K.KT_OK
    og = oracle_gate(layer, inp)
    assert np.abs(s.cpu().numpy() - og["scores"]).max() <= 1e-4
    # Selecting from these scores is exactly the gate's own selection.
    idx_a = torch.empty((T, layer.topk), dtype=torch.int32, device="cuda")
    w_a = torch.empty((T, layer.topk), dtype=torch.float32, device="cuda")
    idx_b, w_b = torch.empty_like(idx_a), torch.empty_like(w_a)
    K.kt_moe_gate(cfg, T, inp["x"], inp["w_gate"], inp["bias"], None, idx_a, w_a, ws)
    K.kt_moe_gate(cfg, T, None, None, inp["bias"], s, idx_b, w_b, ws)
    assert torch.equal(idx_a, idx_b) and torch.equal(w_a, w_b)


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (37, 30, 3), (1000, 64, 6), (8192, 256, 8),
                                   (50000, 256, 8)])
def test_bias_update_is_bit_exact(T, E, k):
    rng = np.random.default_rng(T + E)
    idx = _random_idx(rng, T, E, k)
    bias = rng.normal(0, 0.1, E).astype(np.float32)
    cfg_l = W.BY_NAME["small_sig_bias"].with_(n_experts=E, n_groups=1, topk_groups=1, topk=k)
    cfg = K.config_for(cfg_l)
    b = torch.from_numpy(bias).cuda()
    load = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    K.kt_moe_bias_update(cfg, T, torch.from_numpy(idx).cuda(), b, 1e-3, load)
    torch.cuda.synchronize()
    want = O.bias_update(dict(n_experts=E, n_groups=1, topk_groups=1, topk=k, route_scale=1.0,
                              score_func=0, dim=8, inter=8, n_shared=0), idx, 1e-3, bias)
    assert np.array_equal(b.cpu().numpy(), want)
    assert np.array_equal(load.cpu().numpy(), np.bincount(idx.ravel(), minlength=E))


def _stats_gpu(cfg, T, s, idx, alpha):
    E = s.shape[1]
    ws = torch.empty(K.kt_moe_balance_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    f = torch.full((E,), float("nan"), device="cuda")
    P = torch.full((E,), float("nan"), device="cuda")
    loss = torch.full((1,), float("nan"), device="cuda")
    K.kt_moe_balance_stats(cfg, T, s, idx, alpha, f, P, loss, ws)
    torch.cuda.synchronize()
    return f.cpu().numpy(), P.cpu().numpy(), float(loss.item())


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (33, 30, 3), (1000, 64, 6), (8192, 256, 8),
                                   (40000, 256, 8)])
def test_balance_stats_match_oracle(T, E, k):
    rng = np.random.default_rng(7 * T + E)
    idx = _random_idx(rng, T, E, k)
    s = rng.uniform(0.01, 1.0, (T, E)).astype(np.float32)
    layer = W.BY_NAME["small_sig_bias"].with_(n_experts=E, n_groups=1, topk_groups=1, topk=k)
    cfg = K.config_for(layer)
    sd, idd = torch.from_numpy(s).cuda(), torch.from_numpy(idx).cuda()
    f, P, loss = _stats_gpu(cfg, T, sd, idd, 1e-3)
    want = O.balance_stats(dict(n_experts=E, n_groups=1, topk_groups=1, topk=k, route_scale=1.0,
                                score_func=0, dim=8, inter=8, n_shared=0), s, idx, 1e-3)
    assert np.array_equal(f, want["f"].astype(np.float32))
    np.testing.assert_allclose(P, want["P"], rtol=2e-5, atol=0)
    assert abs(loss - want["loss"]) <= 2e-5 * abs(want["loss"])
    # Deterministic: a second call gives the same bits.
    f2, P2, loss2 = _stats_gpu(cfg, T, sd, idd, 1e-3)
    assert np.array_equal(f, f2) and np.array_equal(P, P2) and loss == loss2


def test_balance_stats_of_a_real_routing():
    """Scores and routing from the V3 prefill layer's own gate (Zipf-skewed load)."""
    layer = W.V3_PREFILL
    inp = W.make_gate_inputs(layer, "cuda")
    cfg = K.config_for(layer)
    T, E, k = layer.T, layer.n_experts, layer.topk
    ws = K.alloc_workspace(cfg, T)
    s = torch.empty((T, E), device="cuda")
    K.kt_moe_scores(cfg, T, inp["x"], inp["w_gate"], s, ws)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    K.kt_moe_gate(cfg, T, None, None, inp["bias"], s, idx, w, ws)
    f, P, loss = _stats_gpu(cfg, T, s, idx, 1e-4)
    sn, idn = s.cpu().numpy(), idx.cpu().numpy()
    want = O.balance_stats(layer.kernel_fields(), sn, idn, 1e-4)
    assert np.array_equal(f, want["f"].astype(np.float32))
    np.testing.assert_allclose(P, want["P"], rtol=2e-5, atol=0)
    assert abs(loss - want["loss"]) <= 2e-5 * abs(want["loss"])
    assert abs(float(f.sum()) - k) <= 1e-4


def test_repeated_bias_updates_even_out_the_load():
    """The mechanism of the page: gate, update the bias from the routing, repeat.
    Starting from a bias that sends most tokens to a few experts, the largest
    expert load falls."""
    layer = W.BY_NAME["small_sig_bias"].with_(T=2048, seed=4242)
    inp = W.make_gate_inputs(layer, "cuda")
    cfg = K.config_for(layer)
    T, E, k = layer.T, layer.n_experts, layer.topk
    bias = torch.linspace(0.3, -0.3, E, device="cuda").contiguous()
    ws = K.alloc_workspace(cfg, T)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    load = torch.empty((E,), dtype=torch.int32, device="cuda")
    peaks = []
    for _ in range(60):
        K.kt_moe_gate(cfg, T, inp["x"], inp["w_gate"], bias, None, idx, w, ws)
        K.kt_moe_bias_update(cfg, T, idx, bias, 0.01, load)
        peaks.append(int(load.max().item()))
    mean = T * k / E
    assert peaks[0] > 2 * mean
    assert peaks[-1] < 0.6 * peaks[0]
