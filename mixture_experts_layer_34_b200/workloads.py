"""Layer shapes and seeded synthetic inputs for the DeepSeekMoE layer forward.

This module serves both the CUDA path and the CPU oracle, so it holds NONE of
the layer's arithmetic: only shapes, seeds and random draws.

Shapes follow the pages: the V3 config table of the DeepSeek-V3 model.py notes
(73biji.xyz/llm_pp_dsv3, "DeepSeek-V3（model.py 配置，节选）": dim 7168, 256 routed
+ 1 shared, top-8, 8 groups keep 4, route_scale 2.5, sigmoid) and the
DeepSeek-V2 model card ("架构简图": dim 5120, 160 routed, top-6, 2 shared).
The token counts mirror the KTransformers DeepSeek page's serving runs
(chunked prefill of 512, at most 8 running requests).

Recipes (all seeded; seed = 1000 + index for the five named layers):
  x ~ N(0, 1). bf16 layers: every weight ~ N(0, 0.02), rounded to bf16.
  tiny fp32 layer: FFN weights ~ N(0, fan_in^-1/2) (std), gate ~ N(0, dim^-1/2).
  bias ~ N(0, 0.1) fp32 where the layer has one. The skewed-prefill layer uses
  a stored bias (data/zipf_bias_v3_prefill.json) fitted offline with the oracle
  so that its expert load follows Zipf(1.1) over a seeded rank order, the last
  8 ranks pinned to -4 (no token). See tests/golden/fit_zipf_bias.py.

x, W_gate and the bias are always drawn on the CPU generator (so routing is the
same on every device); the expert weights are drawn on the target device from a
second seeded stream (seed + 500), expert by expert.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass, asdict, replace

import torch

SIGMOID, SOFTMAX = 0, 1
GROUP_AUTO, GROUP_AMAX, GROUP_TOP2SUM = 0, 1, 2

# Zipf exponent and the pinned-dead experts of the skewed-prefill layer. Its load
# (max/mean >= 10, some experts with no token, rank-frequency slope near -1.1)
# is checked by tests/test_workloads.py with the oracle's gate.
ZIPF_S = 1.1
ZIPF_DEAD = 8
ZIPF_DEAD_BIAS = -4.0
ZIPF_BIAS_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "data",
                              "zipf_bias_v3_prefill.json")
WEIGHT_SEED_OFFSET = 500


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    dim: int
    n_experts: int
    n_groups: int
    topk_groups: int
    topk: int
    n_shared: int
    inter: int
    score_func: int
    route_scale: float
    norm_topk: int          # -1 auto (renormalise iff sigmoid), 0, 1
    group_score: int        # 0 auto, 1 amax, 2 top-2 sum
    dtype: str              # "f32", "bf16", "mxfp8" or "mxfp4" (bf16 tokens, MXFP8 / MXFP4
                            # expert weights)
    bias: str               # "none", "normal", "zipf"
    seed: int
    init: str = "std002"    # "std002" or "fan_in"
    add_residual: int = 0
    note: str = ""

    def as_dict(self) -> dict:
        return asdict(self)

    def kernel_fields(self) -> dict:
        """The fields of the layer config struct (and of the oracle's)."""
        return dict(n_experts=self.n_experts, n_groups=self.n_groups,
                    topk_groups=self.topk_groups, topk=self.topk,
                    route_scale=self.route_scale, score_func=self.score_func,
                    dim=self.dim, inter=self.inter, n_shared=self.n_shared,
                    norm_topk=self.norm_topk, group_score=self.group_score,
                    add_residual=self.add_residual)

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)


# The five named layers.
TINY = LayerConfig("tiny_fp32", T=64, dim=256, n_experts=16, n_groups=4, topk_groups=2,
                   topk=4, n_shared=1, inter=128, score_func=SIGMOID, route_scale=2.5,
                   norm_topk=-1, group_score=GROUP_AUTO, dtype="f32", bias="normal",
                   seed=1000, init="fan_in",
                   note="tiny DeepSeekMoE layer, fp32")
V2_LITE = LayerConfig("v2lite_T512", T=512, dim=2048, n_experts=64, n_groups=1, topk_groups=1,
                      topk=6, n_shared=2, inter=1408, score_func=SOFTMAX, route_scale=1.0,
                      norm_topk=0, group_score=GROUP_AUTO, dtype="bf16", bias="none",
                      seed=1001, note="DeepSeek-V2-Lite-shaped, one chunked-prefill chunk")
V2 = LayerConfig("v2_T4096", T=4096, dim=5120, n_experts=160, n_groups=8, topk_groups=3,
                 topk=6, n_shared=2, inter=1536, score_func=SOFTMAX, route_scale=1.0,
                 norm_topk=-1, group_score=GROUP_AMAX, dtype="bf16", bias="none",
                 seed=1002, note="DeepSeek-V2-shaped")
V3_DECODE = LayerConfig("v3_decode_T8", T=8, dim=7168, n_experts=256, n_groups=8,
                        topk_groups=4, topk=8, n_shared=1, inter=2048, score_func=SIGMOID,
                        route_scale=2.5, norm_topk=-1, group_score=GROUP_TOP2SUM,
                        dtype="bf16", bias="normal", seed=1003,
                        note="DeepSeek-V3-shaped decode step, 8 running requests")
V3_PREFILL = LayerConfig("v3_prefill_T8192_zipf", T=8192, dim=7168, n_experts=256, n_groups=8,
                         topk_groups=4, topk=8, n_shared=1, inter=2048, score_func=SIGMOID,
                         route_scale=2.5, norm_topk=-1, group_score=GROUP_TOP2SUM,
                         dtype="bf16", bias="zipf", seed=1004,
                         note="DeepSeek-V3-shaped prefill, Zipf(1.1) expert load")

NAMED = [TINY, V2_LITE, V2, V3_DECODE, V3_PREFILL]
BY_NAME = {c.name: c for c in NAMED}

# Smaller layers for element-by-element parity: several tiles and ragged tails
# in every dimension, finishing in seconds on the oracle.
SMALL = [
    LayerConfig("small_sig_bias", T=300, dim=512, n_experts=32, n_groups=4, topk_groups=2,
                topk=4, n_shared=1, inter=256, score_func=SIGMOID, route_scale=2.5,
                norm_topk=-1, group_score=GROUP_AUTO, dtype="bf16", bias="normal", seed=2001),
    LayerConfig("small_softmax_ragged", T=257, dim=384, n_experts=16, n_groups=1,
                topk_groups=1, topk=6, n_shared=2, inter=192, score_func=SOFTMAX,
                route_scale=1.0, norm_topk=0, group_score=GROUP_AUTO, dtype="bf16",
                bias="none", seed=2002),
    LayerConfig("small_amax_groups", T=129, dim=256, n_experts=24, n_groups=6, topk_groups=2,
                topk=3, n_shared=1, inter=136, score_func=SOFTMAX, route_scale=1.0,
                norm_topk=-1, group_score=GROUP_AMAX, dtype="bf16", bias="none", seed=2003),
    LayerConfig("small_odd_dims", T=77, dim=200, n_experts=8, n_groups=2, topk_groups=1,
                topk=2, n_shared=0, inter=72, score_func=SIGMOID, route_scale=1.5,
                norm_topk=-1, group_score=GROUP_AUTO, dtype="bf16", bias="normal",
                seed=2004, add_residual=1),
    LayerConfig("small_fp32_groups", T=100, dim=160, n_experts=12, n_groups=3, topk_groups=2,
                topk=3, n_shared=2, inter=96, score_func=SIGMOID, route_scale=2.5,
                norm_topk=-1, group_score=GROUP_AUTO, dtype="f32", bias="normal", seed=2005,
                init="fan_in"),
]
BY_NAME.update({c.name: c for c in SMALL})

# Reduced V3-shaped layer (d, I, k, S, groups of the V3 layer; 32 experts, about
# 3 GB of weights) for full ncu captures, which must stay a few GB on the device.
PROFILE = [
    LayerConfig("v3_shape_T2048_E32_profile", T=2048, dim=7168, n_experts=32, n_groups=8,
                topk_groups=4, topk=8, n_shared=1, inter=2048, score_func=SIGMOID,
                route_scale=2.5, norm_topk=-1, group_score=GROUP_TOP2SUM, dtype="bf16",
                bias="normal", seed=2101),
    # One routed expert, every token routed to it: the two expert GEMMs become
    # dense 8192 x 4096 x 7168 and 8192 x 7168 x 2048 GEMMs (main-loop efficiency
    # without the grouped structure).
    LayerConfig("dense_T8192_E1_profile", T=8192, dim=7168, n_experts=1, n_groups=1,
                topk_groups=1, topk=1, n_shared=0, inter=2048, score_func=SIGMOID,
                route_scale=1.0, norm_topk=-1, group_score=GROUP_AUTO, dtype="bf16",
                bias="none", seed=2102),
]
BY_NAME.update({c.name: c for c in PROFILE})

# MXFP8-expert forms (bf16 tokens and gate, expert weights packed to MXFP8 from
# the same seeded bf16 weights): the V3-shaped layers and two small parity
# layers (dims multiples of 128; ragged token counts; chunks of 224 rows).
MXFP8 = [
    V3_PREFILL.with_(name="v3_prefill_T8192_zipf_mxfp8", dtype="mxfp8"),
    V3_DECODE.with_(name="v3_decode_T8_mxfp8", dtype="mxfp8"),
    LayerConfig("small_sig_bias_mxfp8", T=300, dim=512, n_experts=32, n_groups=4, topk_groups=2,
                topk=4, n_shared=1, inter=256, score_func=SIGMOID, route_scale=2.5,
                norm_topk=-1, group_score=GROUP_AUTO, dtype="mxfp8", bias="normal", seed=2301),
    LayerConfig("small_softmax_mxfp8", T=500, dim=384, n_experts=16, n_groups=1, topk_groups=1,
                topk=3, n_shared=2, inter=384, score_func=SOFTMAX, route_scale=1.0,
                norm_topk=0, group_score=GROUP_AUTO, dtype="mxfp8", bias="none", seed=2302),
    PROFILE[0].with_(name="v3_shape_T2048_E32_profile_mxfp8", dtype="mxfp8"),
]
BY_NAME.update({c.name: c for c in MXFP8})

# The library's limits and degenerate sizes: the most experts, groups, top-k and
# shared experts a config may have (512, 32, 32, 8), a single token, top-1 over
# 512 experts, and a large token count (int32 row arithmetic over 589,824 rows).
LIMITS = [
    LayerConfig("limits_E512_k32_S8", T=67, dim=256, n_experts=512, n_groups=32, topk_groups=8,
                topk=32, n_shared=8, inter=128, score_func=SIGMOID, route_scale=2.5,
                norm_topk=-1, group_score=GROUP_AUTO, dtype="bf16", bias="normal", seed=2401),
    LayerConfig("limits_T1", T=1, dim=512, n_experts=64, n_groups=8, topk_groups=4, topk=8,
                n_shared=1, inter=256, score_func=SIGMOID, route_scale=2.5, norm_topk=-1,
                group_score=GROUP_AUTO, dtype="bf16", bias="normal", seed=2402),
    LayerConfig("limits_E512_k1_softmax", T=40, dim=128, n_experts=512, n_groups=1,
                topk_groups=1, topk=1, n_shared=0, inter=64, score_func=SOFTMAX, route_scale=1.0,
                norm_topk=0, group_score=GROUP_AUTO, dtype="bf16", bias="none", seed=2403),
    LayerConfig("limits_T65536", T=65536, dim=256, n_experts=64, n_groups=8, topk_groups=4,
                topk=8, n_shared=1, inter=128, score_func=SIGMOID, route_scale=2.5,
                norm_topk=-1, group_score=GROUP_AUTO, dtype="bf16", bias="normal", seed=2404),
    LayerConfig("limits_E512_k32_S8_f32", T=67, dim=256, n_experts=512, n_groups=32,
                topk_groups=8, topk=32, n_shared=8, inter=128, score_func=SIGMOID,
                route_scale=2.5, norm_topk=-1, group_score=GROUP_AUTO, dtype="f32",
                bias="normal", seed=2405, init="fan_in"),
    # Degenerate routing: every expert selected (k = E), and a single routed
    # expert with no shared one (the layer is one dense SwiGLU FFN).
    LayerConfig("limits_k_equals_E", T=40, dim=128, n_experts=8, n_groups=1, topk_groups=1,
                topk=8, n_shared=1, inter=128, score_func=SIGMOID, route_scale=1.0,
                norm_topk=-1, group_score=GROUP_AUTO, dtype="bf16", bias="normal", seed=2407),
    LayerConfig("limits_one_expert", T=70, dim=256, n_experts=1, n_groups=1, topk_groups=1,
                topk=1, n_shared=0, inter=128, score_func=SOFTMAX, route_scale=1.0,
                norm_topk=0, group_score=GROUP_AUTO, dtype="bf16", bias="none", seed=2408),
    LayerConfig("limits_E512_k32_S8_mxfp8", T=67, dim=256, n_experts=512, n_groups=32,
                topk_groups=8, topk=32, n_shared=8, inter=128, score_func=SIGMOID,
                route_scale=2.5, norm_topk=-1, group_score=GROUP_AUTO, dtype="mxfp8",
                bias="normal", seed=2406),
]
BY_NAME.update({c.name: c for c in LIMITS})

# MXFP4-expert forms: every MXFP8 layer above with its expert weights packed to
# MXFP4 instead (E2M1 codes, two per byte, and a scale per 32), from the same
# seeded bf16 weights; tokens and hidden rows stay MXFP8.
MXFP4 = [c.with_(name=c.name.replace("_mxfp8", "_mxfp4"), dtype="mxfp4")
         for c in MXFP8 + [BY_NAME["limits_E512_k32_S8_mxfp8"]]]
BY_NAME.update({c.name: c for c in MXFP4})


def torch_dtype(cfg: LayerConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, g, device, dtype):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)


def zipf_bias(n_experts: int) -> torch.Tensor:
    """The stored, oracle-fitted bias of the skewed-prefill layer."""
    with open(ZIPF_BIAS_FILE) as f:
        doc = json.load(f)
    b = torch.tensor(doc["bias"], dtype=torch.float32)
    if b.numel() != n_experts:
        raise ValueError(f"stored Zipf bias has {b.numel()} experts, layer has {n_experts}")
    return b


def make_gate_inputs(cfg: LayerConfig, device="cpu", seed: int | None = None) -> dict:
    """x [T, d], w_gate [E, d] and bias [E] (fp32, or None), drawn on the CPU."""
    seed = cfg.seed if seed is None else seed
    g = _gen("cpu", seed)
    dt = torch_dtype(cfg)
    x = _normal((cfg.T, cfg.dim), 1.0, g, "cpu", dt)
    gstd = cfg.dim ** -0.5 if cfg.init == "fan_in" else 0.02
    w_gate = _normal((cfg.n_experts, cfg.dim), gstd, g, "cpu", dt)
    if cfg.bias == "none":
        bias = None
    elif cfg.bias == "normal":
        bias = _normal((cfg.n_experts,), 0.1, g, "cpu", torch.float32)
    elif cfg.bias == "zipf":
        bias = zipf_bias(cfg.n_experts)
    else:
        raise ValueError(cfg.bias)
    out = dict(x=x, w_gate=w_gate, bias=bias)
    if str(device) != "cpu":
        out = {k: (v.to(device) if v is not None else None) for k, v in out.items()}
    return out


def make_layer(cfg: LayerConfig, device="cpu", seed: int | None = None) -> dict:
    """All inputs of one layer: x, w_gate, bias, and stacked expert weights.

    w1, w3: [E+S, I, d] (gate and up projections, nn.Linear [out, in]);
    w2: [E+S, d, I] (down projection). Routed experts 0..E-1, shared E..E+S-1.
    Drawn expert by expert so the peak host/device footprint stays at the
    stacked tensors themselves.
    """
    seed = cfg.seed if seed is None else seed
    out = make_gate_inputs(cfg, device, seed)
    g = _gen(device, seed + WEIGHT_SEED_OFFSET)
    dt = torch_dtype(cfg)
    n_all = cfg.n_experts + cfg.n_shared
    s13 = cfg.dim ** -0.5 if cfg.init == "fan_in" else 0.02
    s2 = cfg.inter ** -0.5 if cfg.init == "fan_in" else 0.02
    w1 = torch.empty((n_all, cfg.inter, cfg.dim), dtype=dt, device=device)
    w3 = torch.empty_like(w1)
    w2 = torch.empty((n_all, cfg.dim, cfg.inter), dtype=dt, device=device)
    for e in range(n_all):
        w1[e] = _normal((cfg.inter, cfg.dim), s13, g, device, dt)
        w3[e] = _normal((cfg.inter, cfg.dim), s13, g, device, dt)
        w2[e] = _normal((cfg.dim, cfg.inter), s2, g, device, dt)
    out.update(w1=w1, w3=w3, w2=w2)
    return out


def flops_per_token(cfg: LayerConfig) -> int:
    """6 d I (k + S) for the expert GEMMs plus 2 d E for the gate logits."""
    return 6 * cfg.dim * cfg.inter * (cfg.topk + cfg.n_shared) + 2 * cfg.dim * cfg.n_experts


def expert_bytes(cfg: LayerConfig) -> int:
    """Bytes of one expert's W1, W3 and W2."""
    es = 4 if cfg.dtype == "f32" else 2
    return 3 * cfg.dim * cfg.inter * es
