"""Gate parity on the GPU, through the C ABI (kt_moe_gate).

Selection fed the oracle's fp32 scores must reproduce the oracle's indices and
weights exactly; the full gate from x may differ only at near ties (the
oracle's k-th vs (k+1)-th key, or TG-th vs (TG+1)-th group score, within 1e-5).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.oracle as O
from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import NEAR_TIE, oracle_gate

pytestmark = pytest.mark.gpu

# bf16 with E % 4 != 0 and T > 64: the register-tiled SIMT logits path.
ODD_E = W.BY_NAME["small_sig_bias"].with_(name="small_E30_simt_logits", n_experts=30, n_groups=3)
LAYERS = W.NAMED + W.SMALL + [ODD_E] + [c for c in W.LIMITS if c.dtype != "mxfp8"]


def _gpu_gate(layer, inp, scores_in=None):
    cfg = K.config_for(layer)
    T = inp["x"].shape[0]
    ws = K.alloc_workspace(cfg, T)
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device="cuda")
    w = torch.empty((T, layer.topk), dtype=torch.float32, device="cuda")
    K.kt_moe_gate(cfg, T, inp["x"], inp["w_gate"], inp["bias"], scores_in, idx, w, ws)
    assert K.kt_moe_check(ws) == K.KT_OK
    lay = K.kt_moe_workspace_layout(cfg, T)
    # the first [T, E] slot of the logits region holds the logits after the call
    logits = ws[lay["logits"]: lay["logits"] + T * layer.n_experts * 4].view(torch.float32)
    logits = logits.view(T, layer.n_experts).cpu().numpy()
    return idx.cpu().numpy(), w.cpu().numpy(), logits


@pytest.mark.parametrize("layer", LAYERS, ids=lambda c: c.name)
def test_selection_from_oracle_scores_is_exact(layer):
    inp = W.make_gate_inputs(layer, "cuda")
    og = oracle_gate(layer, inp)
    s = torch.from_numpy(og["scores"]).cuda()
    idx, w, _ = _gpu_gate(layer, inp, scores_in=s)
    assert np.array_equal(idx, og["idx"])
    assert np.array_equal(w, og["w"])


@pytest.mark.parametrize("layer", LAYERS, ids=lambda c: c.name)
def test_gate_from_tokens_matches_up_to_near_ties(layer):
    inp = W.make_gate_inputs(layer, "cuda")
    og = oracle_gate(layer, inp)
    idx, w, logits = _gpu_gate(layer, inp)
    # fp32 logits against the double-accumulated oracle
    scale = np.abs(og["logits"]).max()
    assert np.abs(logits - og["logits"]).max() <= 1e-5 * max(scale, 1.0)
    diff = np.where((idx != og["idx"]).any(1))[0]
    near = (og["kth_margin"] <= NEAR_TIE) | (og["grp_margin"] <= NEAR_TIE)
    assert near[diff].all(), f"routing differs away from a near tie at tokens {diff[~near[diff]]}"
    same = np.setdiff1d(np.arange(layer.T), diff)
    # The weights inherit the fp32 logits' accumulation error (about 1e-5 at
    # d = 7168) through the score function.
    np.testing.assert_allclose(w[same], og["w"][same], rtol=1e-4, atol=1e-6)
    print(f"{layer.name}: {len(diff)} near-tie routing differences, {near.sum()} near ties")


def test_selection_ties_resolve_to_lower_index():
    """Scores on a coarse grid (many exact ties), fed through scores_in."""
    layer = W.BY_NAME["small_sig_bias"]
    rng = np.random.default_rng(0)
    s = (rng.integers(1, 5, (layer.T, layer.n_experts)) / 8).astype(np.float32)
    bias = torch.from_numpy((rng.integers(-2, 3, layer.n_experts) / 16).astype(np.float32)).cuda()
    inp = dict(x=None, w_gate=None, bias=bias)
    og = O.select(layer.kernel_fields(), s, bias.cpu().numpy())
    idx, w, _ = _gpu_gate(layer, dict(inp, x=torch.empty(layer.T, 8, device="cuda")),
                          scores_in=torch.from_numpy(s).cuda())
    assert np.array_equal(idx, og["idx"]) and np.array_equal(w, og["w"])


def test_gate_worked_examples_on_gpu():
    import json
    import os
    doc = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                      "gate_worked_examples.json")))
    for ex in doc["examples"]:
        c = ex["cfg"]
        cfg = K.make_config(dtype=K.KT_DTYPE_BF16, **c)
        s = torch.tensor([ex["scores"]], dtype=torch.float32, device="cuda")
        b = None if ex["bias"] is None else torch.tensor(ex["bias"], dtype=torch.float32, device="cuda")
        ws = K.alloc_workspace(cfg, 1)
        idx = torch.empty((1, c["topk"]), dtype=torch.int32, device="cuda")
        w = torch.empty((1, c["topk"]), dtype=torch.float32, device="cuda")
        K.kt_moe_gate(cfg, 1, None, None, b, s, idx, w, ws)
        assert idx[0].tolist() == ex["idx"], ex["name"]
        assert w[0].tolist() == ex["w"], ex["name"]
