"""The device-side failure path, made to fire without faulting the GPU.

kt_moe_selftest_timeout waits, through the GEMM kernels' bounded wait, on an
mbarrier that nothing arrives on (a flag that nothing sets). The wait must give
up after its limit, record the timeout in the workspace error word, and leave
the context usable: kt_moe_check reports KT_ERR_TIMEOUT, and the next forward
on the same workspace runs clean and gives the same output as before.
"""
from __future__ import annotations

import time

import pytest
import torch

from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

from parity import run_forward

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_stays_usable():
    layer = W.BY_NAME["small_sig_bias"]
    inp = W.make_layer(layer, "cuda")
    before = run_forward(layer, inp)
    ws = before["ws"]
    assert K.kt_moe_check(ws) == K.KT_OK
    limit = 20_000_000                       # 20 ms
    t = time.perf_counter()
    K.kt_moe_selftest_timeout(ws, limit)
    assert K.kt_moe_check(ws) == K.KT_ERR_TIMEOUT
    assert time.perf_counter() - t >= limit * 1e-9
    after = run_forward(layer, inp, ws=ws)   # asserts kt_moe_check == KT_OK itself
    assert torch.equal(after["y"], before["y"])
    assert torch.equal(after["idx"], before["idx"])
