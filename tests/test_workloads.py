"""The synthetic workloads carry the pages' constants and the stated load shapes (CPU)."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle.oracle as O
from mixture_experts_layer_34_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_named_layers_carry_page_constants():
    pc = json.load(open(os.path.join(GOLDEN, "page_constants.json")))
    v3 = pc["v3"]
    for c in (W.V3_DECODE, W.V3_PREFILL):
        assert (c.dim, c.n_experts, c.n_shared, c.topk, c.n_groups, c.topk_groups) == \
            (v3["dim"], v3["n_routed"], v3["n_shared"], v3["topk"], v3["n_groups"], v3["topk_groups"])
        assert c.route_scale == v3["route_scale"] and c.score_func == W.SIGMOID
        assert c.bias != "none" and c.dim == pc["v3_bias"]["dim_with_bias"]
    v2 = pc["v2"]
    assert (W.V2.dim, W.V2.n_experts, W.V2.topk, W.V2.n_shared) == \
        (v2["dim"], v2["n_routed"], v2["topk"], v2["n_shared"])
    for c in (W.V2, W.V2_LITE):
        assert c.bias == "none"   # only the dim=7168 model carries a bias


def test_generators_are_seeded_and_shaped():
    c = W.BY_NAME["small_sig_bias"]
    a = W.make_layer(c)
    b = W.make_layer(c)
    for k in ("x", "w_gate", "bias", "w1", "w3", "w2"):
        assert torch.equal(a[k], b[k])
    n = c.n_experts + c.n_shared
    assert a["w1"].shape == (n, c.inter, c.dim) and a["w2"].shape == (n, c.dim, c.inter)
    assert a["x"].dtype == torch.bfloat16 and a["bias"].dtype == torch.float32
    t = W.make_layer(W.TINY)
    assert t["x"].dtype == torch.float32
    # fan-in init of the tiny layer: std of W2 rows ~ inter^-1/2
    assert abs(float(t["w2"].std()) - W.TINY.inter ** -0.5) < 0.01


@pytest.fixture(scope="module")
def v3_prefill_gate():
    c = W.V3_PREFILL
    gi = W.make_gate_inputs(c)
    return gi, O.gate(c.kernel_fields(), gi["x"], gi["w_gate"], gi["bias"])


def test_zipf_prefill_load_shape(v3_prefill_gate):
    gi, g = v3_prefill_gate
    c = W.V3_PREFILL
    load = np.bincount(g["idx"].ravel(), minlength=c.n_experts)
    assert load.sum() == c.T * c.topk
    assert load.max() >= 10 * load.mean()          # some experts > 10x mean
    assert (load == 0).sum() >= 1                    # some experts get no token
    nz = np.sort(load[load > 0])[::-1]
    rk = np.arange(1, len(nz) + 1)
    sel = (rk >= 5) & (rk <= len(nz) - 5)
    slope = np.polyfit(np.log(rk[sel]), np.log(nz[sel]), 1)[0]
    assert -1.3 < slope < -0.9, slope                # Zipf(1.1) rank-frequency
    stored = json.load(open(W.ZIPF_BIAS_FILE))
    assert stored["load"] == load.tolist()           # the fixture still describes this workload
