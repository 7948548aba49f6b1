"""The forward as a CUDA graph (kt_moe_graph_*), through the C ABI: every
launch gives bitwise the output of kt_moe_forward on the inputs as they are at
launch time."""
from __future__ import annotations

import pytest
import torch

from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import run_forward

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layer", [W.V3_DECODE, W.BY_NAME["small_sig_bias"],
                                   W.BY_NAME["small_odd_dims"], W.TINY], ids=lambda c: c.name)
def test_graph_launches_match_the_direct_forward(layer):
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    T = layer.T
    ws = K.alloc_workspace(cfg, T)
    y = torch.full((T, layer.dim), float("nan"), dtype=inp["x"].dtype, device="cuda")
    idx = torch.full((T, layer.topk), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, layer.topk), float("nan"), device="cuda")
    x = inp["x"].clone()
    g = K.KtMoeGraph(cfg, T, x, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"], y,
                     idx, w, ws)
    try:
        side = torch.cuda.Stream()
        for step in range(3):
            # New tokens in the bound input buffer each step, as a decode loop does.
            gen = torch.Generator(device="cpu").manual_seed(77 + step)
            x.copy_(torch.randn(x.shape, generator=gen).to(x.dtype))
            stream = side if step == 1 else torch.cuda.current_stream()
            if step == 1:
                side.wait_stream(torch.cuda.current_stream())
            g.launch(stream)
            if step == 1:
                torch.cuda.current_stream().wait_stream(side)
            assert K.kt_moe_check(ws) == K.KT_OK
            ref = run_forward(layer, dict(inp, x=x))
            assert torch.equal(idx, ref["idx"]), step
            assert torch.equal(w, ref["w"]), step
            assert torch.equal(y, ref["y"]), step
    finally:
        g.destroy()


def test_graph_create_rejects_bad_arguments_without_leaving_a_handle():
    layer = W.BY_NAME["small_sig_bias"]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    ws = K.alloc_workspace(cfg, layer.T)
    y = torch.empty((layer.T, layer.dim), dtype=inp["x"].dtype, device="cuda")
    with pytest.raises(K.KtMoeError):
        K.KtMoeGraph(cfg, layer.T, inp["x"], inp["w_gate"], inp["bias"], inp["w1"], inp["w3"],
                     inp["w2"], y, None, None, ws[:-1])
