"""Parity of the block-scaled (MXFP8 / MXFP4 weight) forwards, hidden rows
included (test code only).

Both sides quantise the same bf16 weights and tokens by the same rule, so
their codes are identical (checked bit for bit elsewhere). What remains
different is fp32 accumulation on the tensor cores against fp64 in the oracle,
and the one place where that can move a code: the SwiGLU hidden row h, which
each side quantises (E4M3, a power-of-two scale per 32 features) from its own
sum. Where the oracle's h sits next to a rounding boundary, the GPU may round
the other way; one such flip moves one hidden element by one E4M3 step (up to
1/8 of it), and the output by that step times one column of W2, which can
reach a few thousandths of the output's RMS.

So the check has two parts:
  hidden rows: every GPU hidden value (code x 2^scale, read from the
    workspace) equals the oracle's quantisation of its fp64 h, except at
    elements the oracle itself marks as near a boundary (the quantisation of
    h x (1 - delta) or h x (1 + delta) differs from that of h, or the block's
    scale does), where it may be one step away;
  outputs: |y_gpu - y_oracle| <= TOL_BASE * RMS(y_oracle) + allowance, per
    element, where the allowance is the sum over the flipped hidden elements
    of |routing weight x W2 column x flip| (oracle weights, and each flip
    already checked to be one step at an oracle-marked element).
A wrong scale anywhere (a token's, a weight block's or a hidden block's) moves
whole 32-element blocks by a factor of two and fails the first part; the
second part, with no flips, holds the output to TOL_BASE.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle.oracle as O
from mixture_experts_layer_34_b200 import ktmoe as K

# Half-width of the interval around the oracle's fp64 h inside which the GPU's
# fp32 h may fall: DELTA_REL x |h| + DELTA_BLOCK x (the block's max |h|). The
# fp32 sums of g and u leave h an error that is absolute rather than relative
# (small elements of a block are sums with cancellation); measured on the V3
# prefill layers at most 3.1e-7 of the block maximum, 1e-5 of |h| for the
# large elements.
DELTA_REL = 1e-5
DELTA_BLOCK = 2e-6
# Output bound with no flipped hidden element: fp32 against fp64 accumulation.
TOL_BASE = 2e-4


def quantizer(layer):
    """(quantise, dequantise) of the layer's expert-weight format."""
    if layer.dtype == "mxfp4":
        return O.mx4_quantize, O.mx4_dequantize
    return O.mx_quantize, O.mx_dequantize


def _ws_slice(ws, off, nbytes):
    return ws[off: off + nbytes]


def hidden_reader(layer, cfg, ws):
    """A function giving the GPU hidden values (decoded codes x 2^scale,
    float64 [n, I]) of (token, slot) pairs: slot s < S is shared expert s, slot
    S + j the token's j-th routed expert. Rows and scales are located through
    the workspace's row map and GEMM chunk list, by the layout the header
    documents (read once here)."""
    T, k, S, I = layer.T, layer.topk, layer.n_shared, layer.inter
    lay = K.kt_moe_workspace_layout(cfg, T)
    R = T * (k + S)
    row_of = _ws_slice(ws, lay["row_of"], T * k * 4).view(torch.int32).cpu().numpy().reshape(T, k)
    n_chunks = int(_ws_slice(ws, lay["meta"], 4).view(torch.int32).item())
    chunks = _ws_slice(ws, lay["chunks"], n_chunks * 16).view(torch.int32).cpu().numpy()
    chunks = chunks.reshape(n_chunks, 4)
    chunk_of = np.full(R, -1, np.int64)
    m_of = np.zeros(R, np.int64)
    for c, (_, row0, nrows, _) in enumerate(chunks):
        chunk_of[row0: row0 + nrows] = c
        m_of[row0: row0 + nrows] = np.arange(nrows)
    nslab = I // 128
    sf = _ws_slice(ws, lay["hid_sf"], n_chunks * nslab * 1024).cpu().numpy()
    hid = _ws_slice(ws, lay["hidden"], R * I).view(R, I)

    def read(pairs):
        rows = np.array([T * k + s * T + t if s < S else row_of[t, s - S] for t, s in pairs],
                        np.int64)
        assert (chunk_of[rows] >= 0).all()
        codes = hid[torch.as_tensor(rows, device=ws.device)].cpu().numpy()
        c, m = chunk_of[rows][:, None], m_of[rows][:, None]
        b = np.arange(I // 32)[None, :]
        off = ((c * nslab + b // 4) * 1024 + (m // 128) * 512 + 16 * (m % 32) +
               4 * ((m // 32) % 4) + b % 4)
        scales = sf[off].astype(np.int64) - 127
        return O.e4m3_decode(codes) * np.exp2(np.repeat(scales, 32, axis=1).astype(np.float64))

    return read


def hidden_check(h_ref: np.ndarray, v_gpu: np.ndarray) -> dict:
    """Compare GPU hidden values with the oracle's quantisation of its fp64 h
    (rows [n, I]); returns the flips (v_gpu - v_ref, zero where equal) after
    asserting that each is at most one E4M3 step at an element the oracle marks
    as near a boundary: its quantisation changes somewhere in [h - w, h + w]
    (w = DELTA_REL |h| + DELTA_BLOCK x block max), or the block's scale changes
    for a block maximum moved by as much."""
    n, I = h_ref.shape
    deq = lambda a: O.mx_dequantize(*O.mx_quantize(a))
    c0, s0 = O.mx_quantize(h_ref)
    v_ref = O.mx_dequantize(c0, s0)
    amax = np.abs(h_ref).reshape(n, I // 32, 32).max(axis=2)
    w = DELTA_REL * np.abs(h_ref) + DELTA_BLOCK * np.repeat(amax, 32, axis=1)
    lo, hi = h_ref - w, h_ref + w
    # scales of each block's maximum moved up and down by its own half-width
    grow = np.zeros((n * (I // 32), 32))
    grow[:, 0] = (amax * (1 + DELTA_REL + DELTA_BLOCK)).ravel()
    s_up = O.mx_quantize(grow)[1][:, 0].reshape(n, I // 32)
    grow[:, 0] = (amax * (1 - DELTA_REL - DELTA_BLOCK)).ravel()
    s_dn = O.mx_quantize(grow)[1][:, 0].reshape(n, I // 32)
    block_near = (s_up != s0) | (s_dn != s0)
    near = (deq(lo) != v_ref) | (deq(hi) != v_ref) | np.repeat(block_near, 32, axis=1)
    dv = v_gpu - v_ref
    flip = dv != 0
    # one E4M3 step at the larger scale the block may take
    e_max = np.maximum(s0, s_up).astype(np.float64) - 127
    step = np.abs(v_ref) * 2.0 ** -3 + np.repeat(np.exp2(e_max - 9), 32, axis=1)
    bad = flip & (~near | (np.abs(dv) > step * (1 + 1e-12)))
    if bad.any():
        i, f = np.argwhere(bad)[0]
        raise AssertionError(
            f"{int(bad.sum())} hidden values differ from the oracle away from a rounding boundary "
            f"or by more than one step; first at row {i}, feature {f}: h {h_ref[i, f]:.9e}, "
            f"oracle {v_ref[i, f]:.9e}, GPU {v_gpu[i, f]:.9e}, block max {amax[i, f // 32]:.6e}")
    return {"flips": int(flip.sum()), "near": int(near.sum()), "dv": np.where(flip, dv, 0.0)}


def check_forward(layer, inp, y32, ws, og, keep, y_ref, qw, cfg) -> dict:
    """The two-part check on the tokens `keep` (routed as the oracle routes
    them). qw: {expert: (w1 codes/scales, w3 ..., w2 ...)} in the layer's format.
    Returns the statistics the caller prints."""
    _, dequant = quantizer(layer)
    k, S, E = layer.topk, layer.n_shared, layer.n_experts
    kf = layer.kernel_fields()
    xq = torch.from_numpy(O.mx_dequantize(*O.mx_quantize(inp["x"].cpu())).astype(np.float32))
    keep = list(keep)
    pos = {t: i for i, t in enumerate(keep)}
    by_expert: dict[int, list] = {}
    for t in keep:
        for s in range(S):
            by_expert.setdefault(E + s, []).append((t, s, 1.0))
        for j in range(k):
            by_expert.setdefault(int(og["idx"][t, j]), []).append((t, S + j, float(og["w"][t, j])))
    allow = np.zeros((len(keep), layer.dim))
    flips = near = checked = 0
    read = hidden_reader(layer, cfg, ws)
    for e, items in sorted(by_expert.items()):
        toks = [t for t, _, _ in items]
        w1 = torch.from_numpy(dequant(*qw[e][0]).astype(np.float32))
        w3 = torch.from_numpy(dequant(*qw[e][1]).astype(np.float32))
        h_ref = O.expert_hidden(kf, xq, w1, w3, toks)
        del w1, w3
        v_gpu = read([(t, s) for t, s, _ in items])
        r = hidden_check(h_ref, v_gpu)
        flips += r["flips"]
        near += r["near"]
        checked += h_ref.size
        if r["flips"]:
            w2 = np.abs(dequant(*qw[e][2]))
            for i, (t, _, wt) in enumerate(items):
                f = np.nonzero(r["dv"][i])[0]
                if len(f):
                    allow[pos[t]] += abs(wt) * (w2[:, f] @ np.abs(r["dv"][i, f]))
    yg = y32[torch.as_tensor(keep, device=y32.device)].cpu().numpy()
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(yg - y_ref)
    over = err > TOL_BASE * rms + allow * (1 + 1e-9)
    assert not over.any(), (f"{int(over.sum())} outputs beyond {TOL_BASE} x RMS plus the flip "
                            f"allowance; worst excess {float((err - allow).max() / rms):.3e} x RMS")
    return {"max_rel": float(err.max() / rms), "max_rel_unexplained": float(
        np.maximum(err - allow, 0).max() / rms), "hidden_checked": checked,
            "hidden_flips": flips, "hidden_near": near,
            "tokens_with_flips": int((allow.max(axis=1) > 0).sum())}
