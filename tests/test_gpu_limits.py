"""The library at its limits, through the C ABI, against the oracle.

Configs at the largest expert count, group count, top-k and shared-expert count
the boundary accepts (E = 512, G = 32, k = 32, S = 8) in bf16, fp32 and MXFP8;
a single token; top-1 over 512 experts; every expert selected (k = E); one
routed expert and no shared one; and 65,536 tokens (589,824 hidden rows).
Same bounds as the other parity tests: max|dy| <= 2e-2 * RMS(y_ref) (bf16,
MXFP8; on the fp32 output) and 1e-4 * RMS(y_ref) (fp32), routing differences
only at near ties.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import (compare_outputs, oracle_gate, oracle_outputs, routing_agreement, run_forward,
                    tolerance)

pytestmark = pytest.mark.gpu


def _check(layer, toks):
    inp = W.make_layer(layer, "cuda")
    out = run_forward(layer, inp, y_fp32=True)
    og = oracle_gate(layer, inp)
    diff, near = routing_agreement(layer, og, out["idx"].cpu().numpy())
    assert near[diff].all(), f"routing differs away from near ties: {diff[~near[diff]]}"
    keep = [t for t in toks if t not in set(diff.tolist())]
    y_ref = oracle_outputs(layer, inp, og, keep)
    res = compare_outputs(layer, out["y"], y_ref, keep)
    print(f"{layer.name}: rel err {res['rel']:.3e} over {len(keep)} tokens")
    assert res["rel"] <= tolerance(layer), res
    return inp, out


@pytest.mark.parametrize("name", ["limits_E512_k32_S8", "limits_T1", "limits_E512_k1_softmax",
                                  "limits_E512_k32_S8_f32", "limits_k_equals_E",
                                  "limits_one_expert"])
def test_limit_layers_every_token(name):
    layer = W.BY_NAME[name]
    inp, out = _check(layer, list(range(layer.T)))
    if layer.dtype == "bf16":
        y16 = run_forward(layer, inp)["y"]
        assert torch.equal(y16, out["y"].to(torch.bfloat16))


def test_many_tokens_sampled_and_row_counts():
    layer = W.BY_NAME["limits_T65536"]
    rng = np.random.default_rng(31)
    toks = sorted(rng.choice(layer.T, 24, replace=False).tolist()) + [0, layer.T - 1]
    inp, out = _check(layer, sorted(set(toks)))
    lay = K.kt_moe_workspace_layout(K.config_for(layer, y_fp32=True), layer.T)
    ws = out["ws"]
    E, S, T, k = layer.n_experts, layer.n_shared, layer.T, layer.topk
    counts = ws[lay["counts"]: lay["counts"] + 4 * (E + S)].view(torch.int32).cpu().numpy()
    hist = np.bincount(out["idx"].cpu().numpy().ravel(), minlength=E)
    assert np.array_equal(counts[:E], hist)
    assert (counts[E:] == T).all() and counts[:E].sum() == T * k
    assert not torch.isnan(out["y"]).any()


def test_mxfp8_at_the_limits():
    from test_gpu_mxfp8 import _check as check_mxfp8
    layer = W.BY_NAME["limits_E512_k32_S8_mxfp8"]
    check_mxfp8(layer, list(range(layer.T)))
