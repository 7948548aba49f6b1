"""Pins of the oracle's MXFP4 arithmetic (CPU only).

E2M1 encoding and decoding are pinned to ml_dtypes' float4_e2m1fn conversion
(an independent library routine) over every code, every rounding midpoint and
many random values, and to the format's published magnitudes (0, 0.5, 1, 1.5,
2, 3, 4, 6); the block scale rule to its closed form and its edge cases; the
elements of a quantised block to the library's rounding of v / 2^e; the 4-bit
forward to the 8-bit forward on weights that both formats hold exactly.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle.oracle as O

ml_dtypes = pytest.importorskip("ml_dtypes")
F4 = ml_dtypes.float4_e2m1fn


def _lib_encode(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, np.float32).astype(F4).view(np.uint8) & 0xF


def test_decode_every_code_matches_the_library():
    c = np.arange(16, dtype=np.uint8)
    ours = O.e2m1_decode(c)
    lib = c.view(F4).astype(np.float64)
    assert np.array_equal(ours, lib)
    assert np.array_equal(np.signbit(ours), np.signbit(lib))


def test_magnitudes_are_the_published_ones():
    mags = O.e2m1_decode(np.arange(8, dtype=np.uint8))
    assert mags.tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(O.e2m1_decode(np.arange(8, 16, dtype=np.uint8)), -mags)


def test_encode_round_trips_every_value():
    v = O.e2m1_decode(np.arange(16, dtype=np.uint8))
    assert np.array_equal(O.e2m1_encode(v), np.arange(16, dtype=np.uint8))


def test_midpoints_round_to_even_like_the_library():
    v = O.e2m1_decode(np.arange(8, dtype=np.uint8))
    mids = (v[:-1] + v[1:]) / 2
    mids = np.concatenate([mids, -mids])
    codes = O.e2m1_encode(mids)
    assert np.array_equal(codes, _lib_encode(mids))
    assert np.all((codes & 1) == 0)          # the even mantissa wins a tie


def test_random_values_like_the_library():
    rng = np.random.default_rng(4)
    v = rng.uniform(-6, 6, 200000).astype(np.float32).astype(np.float64)
    assert np.array_equal(O.e2m1_encode(v), _lib_encode(v))


def test_encode_saturates_above_six():
    assert O.e2m1_encode([6.5, 7.0, 100.0, -9.0, -1e30]).tolist() == [7, 7, 7, 15, 15]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_scale_rule_closed_form(seed):
    rng = np.random.default_rng(seed)
    a = rng.normal(0, 1, (64, 256)) * np.exp2(rng.integers(-20, 20, (64, 1)))
    _, s = O.mx4_quantize(a)
    amax = np.abs(a.reshape(64, 8, 32)).max(-1)
    e = s.astype(np.int64) - 127
    assert np.all(amax <= 6.0 * np.exp2(e))              # no element saturates
    assert np.all(amax > 6.0 * np.exp2(e - 1))           # and e is the smallest such


def test_scale_rule_edge_cases():
    def scale(amax):
        row = np.zeros((1, 32))
        row[0, 5] = amax
        return int(O.mx4_quantize(row)[1][0, 0]) - 127
    assert scale(0.0) == -127
    assert scale(6.0) == 0 and scale(np.nextafter(6.0, 7.0)) == 1
    assert scale(1.5) == -2 and scale(np.nextafter(1.5, 2.0)) == -1
    assert scale(6.0 * 2.0 ** 40) == 40
    assert scale(2.0 ** -200) == -127                  # clamped below


@pytest.mark.parametrize("seed", [0, 1])
def test_elements_are_the_library_rounding_of_the_scaled_block(seed):
    rng = np.random.default_rng(10 + seed)
    a = rng.normal(0, 1, (32, 128)).astype(np.float32)
    c, s = O.mx4_quantize(a)
    e = np.repeat(s.astype(np.int64) - 127, 32, axis=1)
    want = _lib_encode(np.ldexp(a.astype(np.float64), -e))
    assert np.array_equal(c, want)
    assert np.array_equal(O.mx4_dequantize(c, s), O.e2m1_decode(c) * np.exp2(e))


def test_quantize_rejects_ragged_k():
    with pytest.raises(ValueError):
        O.mx4_quantize(np.zeros((2, 40)))


def test_e2m1_values_are_e4m3_values():
    c = np.arange(16, dtype=np.uint8)
    assert np.array_equal(O.e4m3_decode(O.e2m1_as_e4m3(c)), O.e2m1_decode(c))


def _grid_weights(rng, rows, cols):
    """Rows whose every 32-block is E2M1 values times one power of two (held
    exactly by both MXFP4 and MXFP8)."""
    grid = O.e2m1_decode(np.arange(16, dtype=np.uint8))
    v = grid[rng.integers(0, 16, (rows, cols))]
    v[:, ::32] = 6.0                                  # a full-range element per block
    return v * np.exp2(rng.integers(-9, -5, (rows, cols // 32))).repeat(32, axis=1)


def test_forward_equals_the_fp8_forward_on_weights_both_hold_exactly():
    import torch
    rng = np.random.default_rng(7)
    cfg = dict(n_experts=4, n_groups=1, topk_groups=1, topk=2, route_scale=1.0, score_func=0,
               dim=64, inter=64, n_shared=1, norm_topk=-1, group_score=0, add_residual=0)
    T, E, S, d, I = 5, 4, 1, 64, 64
    x = torch.from_numpy(rng.normal(0, 1, (T, d)).astype(np.float32)).to(torch.bfloat16)
    idx = np.array([[0, 1], [2, 3], [1, 3], [0, 2], [3, 0]], np.int32)
    w = rng.uniform(0.1, 1.0, (T, 2)).astype(np.float32)
    f4 = {k: [] for k in ("w1", "w3", "w2")}
    f8 = {k: [] for k in ("w1", "w3", "w2")}
    for _ in range(E + S):
        for k, shape in (("w1", (I, d)), ("w3", (I, d)), ("w2", (d, I))):
            a = _grid_weights(rng, *shape)
            c4, s4 = O.mx4_quantize(a)
            assert np.array_equal(O.mx4_dequantize(c4, s4), a)      # held exactly
            c8, s8 = O.mx_quantize(a)
            assert np.array_equal(O.mx_dequantize(c8, s8), a)
            f4[k].append((c4, s4))
            f8[k].append((c8, s8))
    y4 = O.forward_mxfp4(cfg, x, idx, w, f4["w1"], f4["w3"], f4["w2"], range(T), False)
    y8 = O.forward_mxfp8(cfg, x, idx, w, f8["w1"], f8["w3"], f8["w2"], range(T), False)
    assert np.array_equal(y4, y8)
    assert np.abs(y4).max() > 0
