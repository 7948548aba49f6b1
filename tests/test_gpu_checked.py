"""The checked build (libktmoe_checked.so, -DKT_CHECKED) on the GPU.

In that build every index a kernel takes from another kernel's output (expert
ids, the row maps, the GEMM chunk and tile lists, chunk counts, token ids) is
range-checked where it is used. On valid inputs no check may fire
(kt_moe_check == KT_OK) and every output must equal the release build's, bit
for bit: the checks only guard accesses, they change no arithmetic.

The binding loads one library per process, so the checked runs happen in a
child process (KTMOE_LIB=checked) that saves its outputs; the release runs
happen here, on the same seeded inputs.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mixture_experts_layer_34_b200 import ep  # noqa: E402
from mixture_experts_layer_34_b200 import ktmoe as K  # noqa: E402
from mixture_experts_layer_34_b200 import workloads as W  # noqa: E402

CASES = ["small_sig_bias", "small_softmax_ragged", "small_odd_dims", "small_amax_groups",
         "small_fp32_groups", "small_sig_bias_mxfp8", "limits_E512_k32_S8", "limits_T1",
         "limits_k_equals_E", "limits_one_expert", "limits_E512_k32_S8_f32",
         "limits_E512_k32_S8_mxfp8", "v3_shape_T2048_E32_profile",
         "v3_shape_T2048_E32_profile_mxfp8", "small_sig_bias_mxfp4", "limits_E512_k32_S8_mxfp4"]
EP_CASES = ["small_sig_bias", "limits_E512_k32_S8"]


def _forward(layer, inp, q, y_fp32):
    T = layer.T
    cfg = K.config_for(layer, y_fp32=y_fp32)
    ws = K.alloc_workspace(cfg, T)
    dt = torch.float32 if y_fp32 or layer.dtype == "f32" else torch.bfloat16
    y = torch.full((T, layer.dim), float("nan"), dtype=dt, device="cuda")
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device="cuda")
    w = torch.empty((T, layer.topk), dtype=torch.float32, device="cuda")
    if q is None:
        K.kt_moe_forward(cfg, T, inp["x"], inp["w_gate"], inp["bias"], inp["w1"], inp["w3"],
                         inp["w2"], y, idx, w, ws)
    else:
        K.kt_moe_forward_mxfp8(cfg, T, inp["x"], inp["w_gate"], inp["bias"], q["w1q"], q["w3q"],
                               q["w2q"], q["sf_up"], q["sf_down"], y, idx, w, ws)
    return {"y": y.cpu(), "idx": idx.cpu(), "w": w.cpu(),
            "rc": torch.tensor(K.kt_moe_check(ws))}


def _ep_partials(layer, inp):
    """Each rank's fp32 partial of a 2-rank balanced placement and of a 3-rank
    contiguous split (rows of experts computed elsewhere are skipped)."""
    E, S, T = layer.n_experts, layer.n_shared, layer.T
    cfg = K.config_for(layer, y_fp32=True)
    ref = _forward(layer, inp, None, True)
    load = torch.bincount(ref["idx"].flatten().long(), minlength=E).tolist()
    out = {}
    for world, placement in ((2, ep.balanced_placement(load, 2)), (3, None)):
        for rank in range(world):
            m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"],
                                     inp["w2"], rank, world, placement=placement)
            part = torch.full((T, layer.dim), float("nan"), device="cuda")
            m.local(inp["x"], part)
            ws, _ = m.buffers(T, inp["x"].device)
            out[f"w{world}r{rank}"] = part.cpu()
            out[f"w{world}r{rank}_rc"] = torch.tensor(K.kt_moe_check(ws))
    return out


def run_cases() -> dict:
    torch.cuda.set_device(0)
    res = {}
    for name in CASES:
        layer = W.BY_NAME[name]
        inp = W.make_layer(layer, "cuda")
        q = None
        if layer.dtype in ("mxfp8", "mxfp4"):
            q = K.pack_mxfp8(K.config_for(layer), inp["w1"], inp["w3"], inp["w2"])
        for y_fp32 in (True, False):
            for key, v in _forward(layer, inp, q, y_fp32).items():
                res[f"{name}/{int(y_fp32)}/{key}"] = v
        if name in EP_CASES:
            for key, v in _ep_partials(layer, inp).items():
                res[f"{name}/ep/{key}"] = v
        del inp, q
        torch.cuda.empty_cache()
    return res


@pytest.mark.gpu
def test_checked_build_matches_release_bit_for_bit(tmp_path):
    assert not K.kt_moe_checked_build(), "run the parent on the release build"
    out = str(tmp_path / "checked.pt")
    env = dict(os.environ, KTMOE_LIB="checked")
    r = subprocess.run([sys.executable, os.path.abspath(__file__), out], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    checked = torch.load(out)
    release = run_cases()
    assert set(checked) == set(release)
    for key, v in release.items():
        if key.endswith("rc"):
            assert int(v) == K.KT_OK, (key, K.strerror(int(v)))
            rc = int(checked[key])
            assert rc == K.KT_OK, (key, "checked build:", K.strerror(rc))
        else:
            assert torch.equal(checked[key], v), key


if __name__ == "__main__":
    assert K.kt_moe_checked_build(), "KTMOE_LIB=checked must select the checked build"
    torch.save(run_cases(), sys.argv[1])
    print("checked run ok")
