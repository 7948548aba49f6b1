"""MXFP8 expert weights on the GPU, through the C ABI, against the oracle.

Quantisation (kt_moe_mxfp8_quantize, kt_moe_mxfp8_pack) is integer work decided
by the same rule on both sides from the same bf16 inputs, so codes and scales
must be bit-exact; the packed scale layout is checked through the formula the
header documents.

The forward is compared with the oracle's MXFP8 forward, which quantises the
same bf16 weights and tokens by the same rule (identical codes) and runs the
literal loop in double. What differs: fp32 accumulation on the tensor cores
and the hidden rows, which the GPU quantises from fp32 sums and the oracle
from double sums, so a hidden code can differ by one E4M3 step (1/8 relative)
where a value sits at a rounding boundary. Both sides quantise identically, so
the bound is set from what these two differences measure (1e-5 to 6e-4 of the
RMS) with a margin: max|dy| <= 2e-3 * RMS(y_ref) on the fp32 output (y_fp32),
and the bf16 output must be exactly its rounding. A wrong block scale (one
32-feature block of one expert off by a factor of two) moves the output by 1-2%
of its RMS, ten times the bound.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.oracle as O
from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

import mx_parity as MX
from parity import coverage_tokens, oracle_gate, routing_agreement

pytestmark = pytest.mark.gpu



@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 256), (300, 7168), (2048, 2048)])
def test_quantize_is_bit_exact(rows, cols):
    g = torch.Generator().manual_seed(rows * cols)
    a = torch.randn(rows, cols, generator=g) * torch.exp2(torch.randint(-20, 20, (rows, 1),
                                                                        generator=g).float())
    a[0, :32] = 0.0                       # an all-zero block
    if rows > 1:
        a[1, :16] = 448.0                 # a block whose maximum is exactly representable
    a = a.to(torch.bfloat16)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, cols // 32, dtype=torch.uint8, device="cuda")
    K.kt_moe_mxfp8_quantize(rows, cols, a.cuda(), codes, scales)
    torch.cuda.synchronize()
    oc, os_ = O.mx_quantize(a)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(scales.cpu().numpy(), os_)


def _unpack_scales(sf, layer, down):
    """Row-major scale bytes of every expert from the packed layout (the
    header's formula)."""
    NG, d, I = layer.n_experts + layer.n_shared, layer.dim, layer.inter
    sf = sf.cpu().numpy()
    if not down:
        out = np.zeros((2, NG, I, d // 32), np.uint8)     # [W1 / W3][g][row][block]
        g, f, b = np.meshgrid(np.arange(NG), np.arange(I), np.arange(d // 32), indexing="ij")
        ft, h = f // 128, (f % 128) // 64
        for which in range(2):
            m = f % 64 + 64 * which
            blk = ((g * (I // 128) + ft) * 2 + h) * (d // 128) + b // 4
            out[which] = sf[blk * 512 + 16 * (m % 32) + 4 * (m // 32) + b % 4]
        return out
    nft = (d + 255) // 256
    g, o, b = np.meshgrid(np.arange(NG), np.arange(d), np.arange(I // 32), indexing="ij")
    ft, h, m = o // 256, (o % 256) // 128, o % 128
    blk = ((g * nft + ft) * 2 + h) * (I // 128) + b // 4
    return sf[blk * 512 + 16 * (m % 32) + 4 * (m // 32) + b % 4]


@pytest.mark.parametrize("name", ["small_sig_bias_mxfp8", "small_softmax_mxfp8"])
def test_pack_is_bit_exact_in_the_documented_layout(name):
    layer = W.BY_NAME[name]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    torch.cuda.synchronize()
    up = _unpack_scales(q["sf_up"], layer, False)
    dn = _unpack_scales(q["sf_down"], layer, True)
    for e in range(layer.n_experts + layer.n_shared):
        for which, key in ((0, "w1"), (1, "w3")):
            oc, os_ = O.mx_quantize(inp[key][e].cpu())
            assert np.array_equal(q[key + "q"][e].cpu().numpy(), oc), (e, key)
            assert np.array_equal(up[which, e], os_), (e, key)
        oc, os_ = O.mx_quantize(inp["w2"][e].cpu())
        assert np.array_equal(q["w2q"][e].cpu().numpy(), oc), e
        assert np.array_equal(dn[e], os_), e


def _forward(layer, inp, q, y_fp32, T=None, ws=None):
    T = layer.T if T is None else T
    cfg = K.config_for(layer, y_fp32=y_fp32)
    ws = K.alloc_workspace(cfg, T) if ws is None else ws
    y = torch.full((T, layer.dim), float("nan"), device="cuda",
                   dtype=torch.float32 if y_fp32 else torch.bfloat16)
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device="cuda")
    w = torch.empty((T, layer.topk), dtype=torch.float32, device="cuda")
    K.kt_moe_forward_mxfp8(cfg, T, inp["x"], inp["w_gate"], inp["bias"], q["w1q"], q["w3q"],
                           q["w2q"], q["sf_up"], q["sf_down"], y, idx, w, ws)
    assert K.kt_moe_check(ws) == K.KT_OK
    return y, idx, w


def _oracle_weights(layer, inp, og, toks):
    """The oracle's MXFP8 (codes, scales) of W1, W3, W2 of every expert the
    tokens use."""
    E, S = layer.n_experts, layer.n_shared
    need = set(range(E, E + S))
    for t in toks:
        need.update(int(e) for e in og["idx"][t])
    return {e: tuple(O.mx_quantize(inp[k][e].cpu()) for k in ("w1", "w3", "w2")) for e in need}


def _oracle_y(layer, inp, og, toks, qw=None):
    E, S = layer.n_experts, layer.n_shared
    qw = _oracle_weights(layer, inp, og, toks) if qw is None else qw
    pick = lambda j: [qw[e][j] if e in qw else None for e in range(E + S)]
    return O.forward_mxfp8(layer.kernel_fields(), inp["x"].cpu(), og["idx"], og["w"], pick(0),
                           pick(1), pick(2), toks, inp["bias"] is not None)


def _check(layer, toks):
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    cfg32 = K.config_for(layer, y_fp32=True)
    ws = K.alloc_workspace(cfg32, layer.T)
    y32, idx, w = _forward(layer, inp, q, True, ws=ws)
    y16, idx16, _ = _forward(layer, inp, q, False)
    assert torch.equal(idx, idx16)
    assert torch.equal(y16, y32.to(torch.bfloat16)), "bf16 y is not round(fp32 y)"
    og = oracle_gate(layer, inp)
    diff, near = routing_agreement(layer, og, idx.cpu().numpy())
    assert near[diff].all(), f"routing differs away from near ties: {diff[~near[diff]]}"
    keep = [t for t in toks if t not in set(diff.tolist())]
    qw = _oracle_weights(layer, inp, og, keep)
    y_ref = _oracle_y(layer, inp, og, keep, qw)
    st = MX.check_forward(layer, inp, y32, ws, og, keep, y_ref, qw, cfg32)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err16 = float(np.abs(y16[torch.as_tensor(keep, device="cuda")].float().cpu().numpy()
                         - y_ref).max())
    print(f"{layer.name}: max|dy| / RMS = {st['max_rel']:.3e} (fp32 output; "
          f"{st['max_rel_unexplained']:.3e} beyond the flip allowance), {err16 / rms:.3e} (bf16 "
          f"output) over {len(keep)} tokens; hidden: {st['hidden_flips']} flips, "
          f"{st['hidden_near']} near a boundary of {st['hidden_checked']}, "
          f"{st['tokens_with_flips']} tokens with flips")
    return inp, q, y32


@pytest.mark.parametrize("name", ["small_sig_bias_mxfp8", "small_softmax_mxfp8"])
def test_small_layers_every_token(name):
    layer = W.BY_NAME[name]
    _check(layer, list(range(layer.T)))


def test_v3_decode_every_token():
    layer = W.BY_NAME["v3_decode_T8_mxfp8"]
    _check(layer, list(range(layer.T)))


def test_v3_prefill_chunk_coverage():
    """At least 512 tokens: one from every 224-row GEMM chunk of the 8 heaviest
    experts and of the shared expert (about 180 chunks), the last row of their
    partial chunks, the lightest experts' tokens and random ones."""
    layer = W.BY_NAME["v3_prefill_T8192_zipf_mxfp8"]
    og = oracle_gate(layer, W.make_gate_inputs(layer))
    toks = coverage_tokens(og["idx"], layer.n_experts, layer.n_shared, 224, total=512, seed=17)
    assert len(toks) >= 512
    _check(layer, toks)


def test_forward_is_deterministic():
    layer = W.BY_NAME["small_sig_bias_mxfp8"]
    inp = W.make_layer(layer, "cuda")
    q = K.pack_mxfp8(K.config_for(layer), inp["w1"], inp["w3"], inp["w2"])
    a, _, _ = _forward(layer, inp, q, True)
    b, _, _ = _forward(layer, inp, q, True)
    assert torch.equal(a, b)


def test_bf16_entry_point_rejects_mxfp8_configs():
    layer = W.BY_NAME["small_sig_bias_mxfp8"]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer)
    ws = K.alloc_workspace(cfg, layer.T)
    y = torch.empty((layer.T, layer.dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(K.KtMoeError):
        K.kt_moe_forward(cfg, layer.T, inp["x"], inp["w_gate"], inp["bias"], inp["w1"], inp["w3"],
                         inp["w2"], y, None, None, ws)


@pytest.mark.parametrize("name", ["small_sig_bias_mxfp8", "small_softmax_mxfp8"])
def test_output_does_not_depend_on_workspace_contents(name):
    """Scale bytes 0xFF are NaN in E8M0: a forward that read any workspace byte
    it did not write first would turn NaN (or change) with this fill."""
    layer = W.BY_NAME[name]
    inp = W.make_layer(layer, "cuda")
    cfg = K.config_for(layer, y_fp32=True)
    q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    outs = []
    for fill in (0x00, 0xFF):
        ws = K.alloc_workspace(cfg, layer.T)
        ws.fill_(fill)
        y = torch.empty((layer.T, layer.dim), device="cuda")
        K.kt_moe_forward_mxfp8(cfg, layer.T, inp["x"], inp["w_gate"], inp["bias"], q["w1q"],
                               q["w3q"], q["w2q"], q["sf_up"], q["sf_down"], y, None, None, ws)
        assert K.kt_moe_check(ws) == K.KT_OK
        outs.append(y)
    assert not torch.isnan(outs[1]).any()
    assert torch.equal(outs[0], outs[1])


def test_tokens_with_distinct_scales():
    """x ~ N(0,1) gives almost every 32-block the same exponent, which would hide
    a kernel reading another token's scale; scaling token t by 2^(t mod 7 - 3)
    makes every token's scales distinct. Hidden rows against the oracle's codes,
    outputs within the two-part bound."""
    layer = W.BY_NAME["small_softmax_mxfp8"]
    inp = W.make_layer(layer, "cuda")
    sc = torch.exp2((torch.arange(layer.T) % 7 - 3).float()).cuda()
    inp["x"] = (inp["x"].float() * sc[:, None]).to(torch.bfloat16)
    cfg = K.config_for(layer)
    q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
    cfg32 = K.config_for(layer, y_fp32=True)
    ws = K.alloc_workspace(cfg32, layer.T)
    y32, idx, _ = _forward(layer, inp, q, True, ws=ws)
    og = oracle_gate(layer, inp)
    diff, near = routing_agreement(layer, og, idx.cpu().numpy())
    assert near[diff].all()
    toks = [t for t in range(0, layer.T, 3) if t not in set(diff.tolist())]
    qw = _oracle_weights(layer, inp, og, toks)
    y_ref = _oracle_y(layer, inp, og, toks, qw)
    st = MX.check_forward(layer, inp, y32, ws, og, toks, y_ref, qw, cfg32)
    print(f"{layer.name} distinct scales: {st}")


@pytest.mark.parametrize("T", [1, 17, 64, 65, 225])
def test_token_counts_every_token(T):
    """Token counts around the gate's split-K / tensor-core switch (64) and the
    224-row MXFP8 chunk, each token against the oracle."""
    layer = W.BY_NAME["small_sig_bias_mxfp8"].with_(name=f"small_sig_bias_mxfp8_T{T}", T=T)
    _check(layer, list(range(T)))
