"""Fit the gate bias of the skewed V3 prefill layer.

The layer's expert load should follow Zipf(s=1.1) over its experts. A bias of
the plain form a*ln(p_r) cannot do that (top-k selection saturates), so the
bias is fitted instead: starting from that form, each expert's bias is nudged
by eta * (ln target - ln load), where the load comes from the oracle's gate on
the layer's seeded x and W_gate. This mirrors the load-driven bias adjustment
the DeepSeek-V3 notes describe ("V3 改进①：无辅助损失负载均衡": b_i moves with the
expert's load), run offline on synthetic inputs.

Writes mixture_experts_layer_34_b200/data/zipf_bias_v3_prefill.json.

Target: ranks r = 1..E-8 of a seeded permutation get load min(T, c * r^-1.1),
c chosen so the loads sum to T*k; the last 8 ranks get bias -4 and no token.

Calls only the oracle and the seeded input generator. Run from the repo root:
    python tests/golden/fit_zipf_bias.py
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle.oracle as O  # noqa: E402
from mixture_experts_layer_34_b200 import workloads as W  # noqa: E402

OUT = W.ZIPF_BIAS_FILE


def target_loads(n_active: int, total: int, cap: int, s: float) -> np.ndarray:
    r = np.arange(1, n_active + 1, dtype=np.float64)
    lo, hi = 0.0, float(total) * 10
    for _ in range(200):
        c = 0.5 * (lo + hi)
        tot = np.minimum(cap, c * r ** -s).sum()
        lo, hi = (c, hi) if tot < total else (lo, c)
    return np.minimum(cap, c * r ** -s)


def main():
    cfg = W.V3_PREFILL
    E, T, k = cfg.n_experts, cfg.T, cfg.topk
    gi = W.make_gate_inputs(cfg.with_(bias="none"))
    kf = cfg.kernel_fields()
    scores = O.scores(kf, O.gate_logits(kf, gi["x"], gi["w_gate"]))

    g = torch.Generator()
    g.manual_seed(cfg.seed + 7)
    rank = torch.randperm(E, generator=g).numpy()          # rank[e] in 0..E-1
    n_active = E - W.ZIPF_DEAD
    tgt_by_rank = target_loads(n_active, T * k, T, W.ZIPF_S)
    active = rank < n_active
    target = np.zeros(E)
    target[active] = tgt_by_rank[rank[active]]

    p = np.arange(1, E + 1, dtype=np.float64) ** -W.ZIPF_S
    b = (0.04 * np.log(p / p.sum()))[rank]
    b[~active] = W.ZIPF_DEAD_BIAS
    b = b.astype(np.float32)
    eta = 0.02
    for it in range(400):
        load = np.bincount(O.select(kf, scores, b)["idx"].ravel(), minlength=E)
        err = np.log(target[active]) - np.log(load[active] + 0.5)
        if it % 25 == 0:
            print(f"iter {it}: max |ln target - ln load| = {np.abs(err).max():.3f}")
        if np.abs(err).max() < 0.03:
            break
        b[active] = (b[active] + eta * err).astype(np.float32)
    load = np.bincount(O.select(kf, scores, b)["idx"].ravel(), minlength=E)
    print("final: max/mean %.1f, zero-load experts %d, top %s" %
          (load.max() / load.mean(), int((load == 0).sum()), np.sort(load)[::-1][:8]))
    doc = {
        "what": "gate bias [E] of the skewed V3 prefill layer (fp32), fitted so the expert "
                "load follows Zipf(1.1); written by tests/golden/fit_zipf_bias.py (oracle only)",
        "layer": cfg.name, "seed": cfg.seed, "zipf_s": W.ZIPF_S, "dead_experts": W.ZIPF_DEAD,
        "rank": rank.tolist(),
        "target_load": [float(v) for v in target],
        "bias": [float(v) for v in b],
        "load": [int(v) for v in load],
    }
    with open(OUT, "w") as f:
        json.dump(doc, f)
    print("wrote", OUT)


if __name__ == "__main__":
    main()
