"""kt_moe_forward_static: the layer forward without any caller allocation.

Some callers cannot allocate device memory at all: engines whose device memory
is entirely owned by their own pool, latency-critical loops in which cudaMalloc
and cudaFree would synchronise the device, and plugin hosts that hand out no
workspace. kt_moe_forward_static serves them with scratch from a fixed 32 MiB
device array inside the library. These tests call it through the
C ABI and compare it with kt_moe_forward (caller workspace) on the same inputs,
on two calls in a row, since the shared scratch keeps the previous call's
contents; and they check that oversized calls are refused before any work.

This file is collected last on purpose (test_zz_...).
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import run_forward, tolerance

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layer", [W.BY_NAME["small_sig_bias"], W.V3_DECODE, W.TINY],
                         ids=lambda c: c.name)
def test_static_scratch_forward_matches_workspace_forward(layer):
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    T = layer.T
    assert K.kt_moe_workspace_size(cfg, T) <= K.KT_STATIC_SCRATCH_BYTES
    ref = run_forward(layer, inp)            # the existing entry point, caller workspace
    rms = ref["y"].float().pow(2).mean().sqrt().item()
    for call in range(2):                    # the second call reuses the same scratch
        y = torch.full_like(ref["y"], float("nan"))
        idx = torch.full_like(ref["idx"], -1)
        w = torch.full_like(ref["w"], float("nan"))
        K.kt_moe_forward_static(cfg, T, inp["x"], inp["w_gate"], inp["bias"], inp["w1"],
                                inp["w3"], inp["w2"], y, idx, w)
        scratch = K.kt_moe_static_scratch()
        assert scratch != 0
        assert K.kt_moe_check(scratch) == K.KT_OK
        assert torch.equal(idx, ref["idx"]), f"call {call}: routing differs"
        err = (y.float() - ref["y"].float()).abs().max().item()
        assert err <= tolerance(layer) * rms, f"call {call}: max |dy| {err:.3e}, RMS {rms:.3e}"
        torch.testing.assert_close(w, ref["w"], rtol=0, atol=0)


def test_static_scratch_refuses_calls_beyond_its_size():
    """The V3 prefill layer (T=8192) needs about 2.3 GB of scratch: refused on the
    host with KT_ERR_SCRATCH_LIMIT, before any pointer is used or work enqueued."""
    cfg = K.config_for(W.V3_PREFILL)
    assert K.kt_moe_workspace_size(cfg, W.V3_PREFILL.T) > K.KT_STATIC_SCRATCH_BYTES
    rc = K.lib().kt_moe_forward_static(ctypes.byref(cfg), W.V3_PREFILL.T, *([None] * 9),
                                       ctypes.c_void_p(0))
    assert rc == K.KT_ERR_SCRATCH_LIMIT
    assert "static" in K.strerror(rc)
