"""The forward as a CUDA graph (kt_moe_graph_*), through the C ABI: every
launch gives bitwise the output of kt_moe_forward on the inputs as they are at
launch time, and matches the oracle on those inputs."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import (compare_outputs, oracle_gate, oracle_outputs, routing_agreement, run_forward,
                    tolerance)
import mx_parity as MX
from test_gpu_mxfp8 import _oracle_weights as _oracle_weights_mx
from test_gpu_mxfp8 import _oracle_y as _oracle_y_mx

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


@pytest.mark.parametrize("name", ["v3_decode_T8_mxfp8", "small_sig_bias_mxfp8"])
def test_mxfp8_graph_launches_match_the_direct_forward(name):
    layer = W.BY_NAME[name]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    T = layer.T
    q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    ws = K.alloc_workspace(cfg, T)
    y = torch.full((T, layer.dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((T, layer.topk), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, layer.topk), float("nan"), device="cuda")
    x = inp["x"].clone()
    g = K.KtMoeGraph.mxfp8(cfg, T, x, inp["w_gate"], inp["bias"], q, y, idx, w, ws)
    try:
        for step in range(2):
            gen = torch.Generator(device="cpu").manual_seed(91 + step)
            x.copy_(torch.randn(x.shape, generator=gen).to(x.dtype))
            g.launch()
            assert K.kt_moe_check(ws) == K.KT_OK
            ws2 = K.alloc_workspace(cfg, T)
            y2 = torch.empty_like(y)
            idx2, w2 = torch.empty_like(idx), torch.empty_like(w)
            K.kt_moe_forward_mxfp8(cfg, T, x, inp["w_gate"], inp["bias"], q["w1q"], q["w3q"],
                                   q["w2q"], q["sf_up"], q["sf_down"], y2, idx2, w2, ws2)
            torch.cuda.synchronize()
            assert torch.equal(idx, idx2) and torch.equal(w, w2) and torch.equal(y, y2), step
    finally:
        g.destroy()


@pytest.mark.parametrize("name", ["v3_decode_T8", "v3_decode_T8_mxfp8"])
def test_graph_replays_match_the_oracle(name):
    """Replays of the captured V3 decode step, new tokens written into the bound
    input buffer before each, against the oracle on every token: routing equal
    except at near ties, routing weights within 1e-4 relative, outputs (fp32
    form) within the layer's bound (MXFP8: the hidden rows against the oracle's
    codes and the outputs within the two-part bound of mx_parity). A replay that read a stale pointer or tensor
    map would fail this even where it agreed with a direct forward sharing the
    same fault."""
    layer = W.BY_NAME[name]
    mx = layer.dtype in ("mxfp8", "mxfp4")
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer, y_fp32=True)
    T = layer.T
    ws = K.alloc_workspace(cfg, T)
    y = torch.full((T, layer.dim), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, layer.topk), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, layer.topk), float("nan"), device="cuda")
    x = inp["x"].clone()
    if mx:
        q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
        g = K.KtMoeGraph.mxfp8(cfg, T, x, inp["w_gate"], inp["bias"], q, y, idx, w, ws)
    else:
        g = K.KtMoeGraph(cfg, T, x, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                         y, idx, w, ws)
    try:
        for step in range(2):
            gen = torch.Generator(device="cpu").manual_seed(131 + step)
            x.copy_(torch.randn(x.shape, generator=gen).to(x.dtype))
            g.launch()
            assert K.kt_moe_check(ws) == K.KT_OK
            cur = dict(inp, x=x.clone())
            og = oracle_gate(layer, cur)
            diff, near = routing_agreement(layer, og, idx.cpu().numpy())
            assert near[diff].all(), (step, diff)
            keep = [t for t in range(T) if t not in set(diff.tolist())]
            wg, wo = w.cpu().numpy()[keep], og["w"][keep]
            assert np.allclose(wg, wo, rtol=1e-4, atol=0), step
            if mx:
                # hidden rows of this replay (in the graph's workspace) against
                # the oracle's codes, outputs within the two-part bound
                qw = _oracle_weights_mx(layer, cur, og, keep)
                y_ref = _oracle_y_mx(layer, cur, og, keep, qw)
                st = MX.check_forward(layer, cur, y, ws, og, keep, y_ref, qw, cfg)
                print(f"{name} replay {step}: {st}")
            else:
                y_ref = oracle_outputs(layer, cur, og, keep)
                res = compare_outputs(layer, y, y_ref, keep)
                print(f"{name} replay {step}: max|dy|/RMS {res['rel']:.3e} over {len(keep)} tokens")
                assert res["rel"] <= tolerance(layer), (step, res)
    finally:
        g.destroy()
