"""Helpers for comparing the CUDA library with the oracle (test code only)."""
from __future__ import annotations

import numpy as np
import torch

import oracle.oracle as O
from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

NEAR_TIE = 1e-5
TOL_BF16 = 2e-2     # max |dy| <= TOL * RMS(y_ref), bf16 layers
TOL_F32 = 1e-4      # same form, fp32 layers


def tolerance(layer) -> float:
    """The output bound by dtype. Block-scaled (MXFP8 / MXFP4) layers get the
    bf16 form's bound here, for the tests that compare one output array only;
    their main parity tests (mx_parity.check_forward) hold the hidden rows to
    the oracle's codes and the outputs to 2e-4 of the RMS plus the effect of
    the hidden codes that sit on a rounding boundary."""
    return TOL_F32 if layer.dtype == "f32" else TOL_BF16


def coverage_tokens(idx: np.ndarray, n_experts: int, n_shared: int, chunk_rows: int,
                    total: int = 512, n_heavy: int = 8, n_light: int = 8,
                    seed: int = 0) -> list[int]:
    """Tokens whose outputs reach every GEMM chunk position of the heavy experts.

    The expert GEMMs take each expert's rows (its tokens in ascending order) in
    chunks of `chunk_rows`. From the routing `idx` (the oracle's), pick one
    random token from every chunk of the `n_heavy` most loaded experts and of the
    shared experts (all T tokens in order), plus the last token of each of those
    experts' final (partial) chunks, one token of each of the `n_light` least
    loaded experts that have a token (all of those with at most four tokens), and
    random tokens up to `total`."""
    rng = np.random.default_rng(seed)
    T = idx.shape[0]
    load = np.bincount(idx.ravel(), minlength=n_experts)
    pick: set[int] = set()

    def cover(toks):
        for c0 in range(0, len(toks), chunk_rows):
            part = toks[c0:c0 + chunk_rows]
            pick.add(int(part[rng.integers(len(part))]))
        if len(toks):
            pick.add(int(toks[-1]))

    for e in np.argsort(-load, kind="stable")[:n_heavy]:
        cover(np.where((idx == e).any(1))[0])
    if n_shared:
        cover(np.arange(T))
    used = [e for e in np.argsort(load, kind="stable") if load[e] > 0]
    for e in set(used[:n_light]) | {e for e in used if load[e] <= 4}:
        pick.add(int(np.where((idx == e).any(1))[0][0]))
    rest = np.setdiff1d(np.arange(T), np.fromiter(pick, np.int64))
    need = max(0, min(total, T) - len(pick))
    pick.update(int(t) for t in rng.choice(rest, min(need, len(rest)), replace=False))
    return sorted(pick)


def run_forward(layer, inp, T=None, ws=None, y_fp32=False):
    """One kt_moe_forward on the current stream; returns y, idx, w, workspace."""
    T = layer.T if T is None else T
    cfg = K.config_for(layer, y_fp32=y_fp32)
    dev = inp["x"].device
    ws = K.alloc_workspace(cfg, T, dev) if ws is None else ws
    ydt = torch.float32 if y_fp32 else inp["x"].dtype
    y = torch.empty((T, layer.dim), dtype=ydt, device=dev)
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device=dev)
    w = torch.empty((T, layer.topk), dtype=torch.float32, device=dev)
    K.kt_moe_forward(cfg, T, inp["x"], inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                     y, idx, w, ws)
    rc = K.kt_moe_check(ws)
    assert rc == K.KT_OK, K.strerror(rc)
    return dict(y=y, idx=idx, w=w, ws=ws)


def oracle_gate(layer, inp):
    bias = inp["bias"]
    return O.gate(layer.kernel_fields(), inp["x"], inp["w_gate"],
                  None if bias is None else bias.float().cpu().numpy())


def routing_agreement(layer, og, idx_gpu: np.ndarray):
    """Tokens whose routing differs, and whether each difference is a near tie."""
    diff = np.where((og["idx"] != idx_gpu).any(1))[0]
    near = (og["kth_margin"] <= NEAR_TIE) | (og["grp_margin"] <= NEAR_TIE)
    return diff, near


def oracle_outputs(layer, inp, og, tok_ids) -> np.ndarray:
    """The oracle's y for tok_ids, copying only the experts those tokens use."""
    E, S = layer.n_experts, layer.n_shared
    need = set(range(E, E + S))
    for t in tok_ids:
        need.update(int(e) for e in og["idx"][t])
    w1 = [inp["w1"][e].cpu() if e in need else None for e in range(E + S)]
    w3 = [inp["w3"][e].cpu() if e in need else None for e in range(E + S)]
    w2 = [inp["w2"][e].cpu() if e in need else None for e in range(E + S)]
    return O.forward(layer.kernel_fields(), inp["x"].cpu(), og["idx"], og["w"], w1, w3, w2,
                     tok_ids, inp["bias"] is not None)


def compare_outputs(layer, y_gpu: torch.Tensor, y_ref: np.ndarray, tok_ids) -> dict:
    yg = y_gpu[torch.as_tensor(np.asarray(tok_ids), device=y_gpu.device)].float().cpu().numpy()
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = float(np.abs(yg - y_ref).max())
    return dict(max_abs=err, rms=rms, rel=err / rms if rms > 0 else float("inf"))
