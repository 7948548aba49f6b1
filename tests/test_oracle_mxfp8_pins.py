"""Pins of the oracle's MXFP8 arithmetic (CPU only).

E4M3 encoding and decoding are pinned to torch's float8_e4m3fn conversion (an
independent library routine) over every code, every rounding midpoint and many
random values; the block scale rule to its closed form; quantise-dequantise to
the format's rounding bound; the FP8 forward to the pinned double forward run
on dequantised operands (exactly, with the hidden quantisation off) and to the
hidden rounding bound (with it on).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.oracle as O


def _torch_encode(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(v, np.float64)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def _finite_values() -> np.ndarray:
    c = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(c)
    return np.unique(v[np.isfinite(v)])


def test_decode_every_code_matches_torch():
    c = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(c)
    th = torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(th))
    assert np.array_equal(ours[~np.isnan(ours)], th[~np.isnan(th)])


def test_encode_round_trips_every_finite_value():
    v = _finite_values()
    assert np.array_equal(O.e4m3_decode(O.e4m3_encode(v)), v)
    assert v.max() == 448.0 and v[v > 0].min() == 2.0 ** -9


def test_encode_midpoints_round_to_even_like_torch():
    v = _finite_values()
    mids = (v[:-1] + v[1:]) / 2          # exact in double
    assert np.array_equal(O.e4m3_encode(mids), _torch_encode(mids))
    # Half-way cases go to the code with an even mantissa.
    codes = O.e4m3_encode(mids[mids > 0])
    assert np.all((codes & 1) == 0)


def test_encode_random_values_like_torch():
    rng = np.random.default_rng(0)
    v = rng.normal(0, 1, 200000) * np.exp2(rng.integers(-14, 9, 200000))
    v = v[np.abs(v) <= 448]
    assert np.array_equal(O.e4m3_encode(v), _torch_encode(v))


def test_encode_saturates_above_448():
    assert O.e4m3_encode(np.array([464.0, 1e6, -500.0])).tolist() == [0x7E, 0x7E, 0xFE]


@pytest.mark.parametrize("seed", range(4))
def test_scale_rule_closed_form(seed):
    """e is the smallest integer with amax <= 448 * 2^e."""
    rng = np.random.default_rng(seed)
    a = rng.normal(0, 1, (64, 128)) * np.exp2(rng.integers(-30, 30, (64, 1)))
    _, s = O.mx_quantize(a)
    e = s.astype(np.int64) - 127
    amax = np.abs(a).reshape(64, 4, 32).max(-1)
    assert np.all(amax <= 448.0 * np.exp2(e))
    assert np.all(amax > 448.0 * np.exp2(e - 1))


def test_scale_rule_edge_cases():
    a = np.zeros((3, 32))
    a[1, 5] = 448.0            # exactly representable at e = 0
    a[2, 0] = 448.0 * 2 ** 3   # e = 3
    codes, s = O.mx_quantize(a)
    assert s[:, 0].tolist() == [0, 127, 130]
    assert not codes[0].any()
    assert O.mx_dequantize(codes, s)[1, 5] == 448.0
    assert O.mx_dequantize(codes, s)[2, 0] == 448.0 * 8


@pytest.mark.parametrize("src", ["f64", "f32", "bf16"])
def test_quantize_dequantize_error_bound(src):
    rng = np.random.default_rng(11)
    a = rng.normal(0, 1, (50, 256)) * np.exp2(rng.integers(-8, 8, (50, 1)))
    if src == "f32":
        a = a.astype(np.float32)
        ref = a.astype(np.float64)
        codes, s = O.mx_quantize(a)
    elif src == "bf16":
        t = torch.from_numpy(a).to(torch.bfloat16)
        ref = t.to(torch.float64).numpy()
        codes, s = O.mx_quantize(t)
    else:
        ref = a
        codes, s = O.mx_quantize(a)
    dq = O.mx_dequantize(codes, s)
    e = np.repeat(s.astype(np.int64) - 127, 32, axis=1)
    bound = np.maximum(np.abs(ref) * 2.0 ** -4, np.exp2(e - 10.0))
    assert np.all(np.abs(dq - ref) <= bound)


def test_quantize_rejects_ragged_k():
    with pytest.raises(ValueError):
        O.mx_quantize(np.zeros((2, 40)))


def _cfg(**kw):
    base = dict(n_experts=6, n_groups=1, topk_groups=1, topk=2, route_scale=1.0, score_func=0,
                dim=64, inter=96, n_shared=1, norm_topk=-1, group_score=0, add_residual=0)
    base.update(kw)
    return base


def _fp8_layer(rng, cfg, T):
    E, S, d, I = cfg["n_experts"], cfg["n_shared"], cfg["dim"], cfg["inter"]
    x = torch.from_numpy(rng.normal(0, 1, (T, d))).to(torch.bfloat16)
    q = []
    for _ in range(E + S):
        w1 = O.mx_quantize(rng.normal(0, 0.05, (I, d)))
        w3 = O.mx_quantize(rng.normal(0, 0.05, (I, d)))
        w2 = O.mx_quantize(rng.normal(0, 0.05, (d, I)))
        q.append((w1, w3, w2))
    idx = np.stack([rng.choice(E, cfg["topk"], replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1.0, (T, cfg["topk"])).astype(np.float32)
    return x, q, idx, w


def test_forward_without_hidden_quantisation_is_the_double_forward_on_dequantised_operands():
    rng = np.random.default_rng(5)
    cfg = _cfg()
    T = 7
    x, q, idx, w = _fp8_layer(rng, cfg, T)
    y8 = O.forward_mxfp8(cfg, x, idx, w, [e[0] for e in q], [e[1] for e in q],
                         [e[2] for e in q], range(T), False, quantize_hidden=False)
    xq = O.mx_dequantize(*O.mx_quantize(x)).astype(np.float32)     # exact in fp32
    deq = lambda p: torch.from_numpy(O.mx_dequantize(*p).astype(np.float32))
    y = O.forward(cfg, torch.from_numpy(xq), idx, w, [deq(e[0]) for e in q],
                  [deq(e[1]) for e in q], [deq(e[2]) for e in q], range(T), False)
    assert np.allclose(y8, y, rtol=1e-12, atol=1e-14)


def test_forward_hidden_quantisation_stays_within_its_rounding_bound():
    rng = np.random.default_rng(6)
    cfg = _cfg()
    T = 5
    x, q, idx, w = _fp8_layer(rng, cfg, T)
    args = (cfg, x, idx, w, [e[0] for e in q], [e[1] for e in q], [e[2] for e in q], range(T),
            False)
    y_off = O.forward_mxfp8(*args, quantize_hidden=False)
    y_on = O.forward_mxfp8(*args, quantize_hidden=True)
    xq = O.mx_dequantize(*O.mx_quantize(x)).astype(np.float32)
    E, S = cfg["n_experts"], cfg["n_shared"]
    for n in range(T):
        bound = np.zeros(cfg["dim"])
        experts = [(E + s, 1.0) for s in range(S)] + [(int(idx[n, j]), float(w[n, j]))
                                                      for j in range(cfg["topk"])]
        for e, wt in experts:
            w1 = torch.from_numpy(O.mx_dequantize(*q[e][0]).astype(np.float32))
            w3 = torch.from_numpy(O.mx_dequantize(*q[e][1]).astype(np.float32))
            h = O.expert_hidden(cfg, torch.from_numpy(xq), w1, w3, [n])[0]
            hb = np.maximum(np.abs(h) * 2.0 ** -4, 2.0 ** -10 * np.repeat(
                np.exp2(O.mx_quantize(h[None, :])[1][0].astype(np.float64) - 127), 32))
            bound += abs(wt) * (np.abs(O.mx_dequantize(*q[e][2])) @ hb)
        assert np.all(np.abs(y_on[n] - y_off[n]) <= bound * (1 + 1e-9) + 1e-12)
    assert not np.array_equal(y_on, y_off)
