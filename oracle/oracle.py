"""Oracle for the DeepSeekMoE layer forward — TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper around ``moe_oracle.cpp`` (plain C++17, fp64, OpenMP).
Only ``tests/``, the package's ``smoke()`` entry and ``bench.py``'s CPU-baseline
leg may import this module. It imports nothing from the CUDA package and the
CUDA package imports nothing from here; the two meet only through the seeded
input generators, which hold none of the method's arithmetic.

What each function computes, and the page passage it follows, is stated in the
C++ source. Parity pins for every function are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

SIGMOID, SOFTMAX = 0, 1
AMAX, TOP2SUM = 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (IEEE arithmetic: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["g++", "-std=c++17", "-O2", "-fopenmp", "-fPIC", "-shared",
               "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("n_experts", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("route_scale", ctypes.c_float), ("score_func", ctypes.c_int32),
                ("dim", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("norm_topk", ctypes.c_int32),
                ("group_score", ctypes.c_int32), ("add_residual", ctypes.c_int32)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            CP = ctypes.POINTER(_Cfg)
            lib.oracle_gate_logits.argtypes = [CP, I64, ctypes.c_int, P, P, P]
            lib.oracle_scores.argtypes = [CP, I64, P, P]
            lib.oracle_select.argtypes = [CP, I64, P, P, P, P, P, P, P, P]
            lib.oracle_forward.argtypes = [CP, I64, ctypes.c_int, P, P, P, P, P, P, I64, P, P]
            lib.oracle_expert_hidden.argtypes = [CP, I64, ctypes.c_int, P, P, P, I64, P, P]
            lib.oracle_expert_load.argtypes = [CP, I64, P, P]
            lib.oracle_bias_update.argtypes = [CP, I64, P, ctypes.c_float, P]
            lib.oracle_balance_stats.argtypes = [CP, I64, P, P, ctypes.c_double, P, P, P]
            lib.oracle_e4m3_encode.argtypes = [I64, P, P]
            lib.oracle_e4m3_decode.argtypes = [I64, P, P]
            lib.oracle_mx_quantize.argtypes = [I64, I64, ctypes.c_int, P, P, P]
            lib.oracle_mx_dequantize.argtypes = [I64, I64, P, P, P]
            lib.oracle_e2m1_encode.argtypes = [I64, P, P]
            lib.oracle_e2m1_decode.argtypes = [I64, P, P]
            lib.oracle_mx4_quantize.argtypes = [I64, I64, ctypes.c_int, P, P, P]
            lib.oracle_mx4_dequantize.argtypes = [I64, I64, P, P, P]
            lib.oracle_forward_mxfp8.argtypes = [CP, I64, P, P, P, P, P, P, P, P, P, ctypes.c_int,
                                                 I64, P, P]
            lib.oracle_forward_part.argtypes = [CP, I64, ctypes.c_int, P, P, P, P, P, P,
                                                ctypes.c_int, ctypes.c_int, I64, P, P, P]
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def resolve(cfg: dict, has_bias: bool) -> dict:
    """Resolve the config's automatic choices.

    norm_topk = -1: renormalise iff sigmoid scoring (the V3 gate renormalises;
    the V2-style softmax configs do not). group_score = 0 (auto): the sum of the
    top-2 keys when a bias exists, else the group max ("Gate 选专家流程", step 2).
    """
    out = dict(cfg)
    if out.get("norm_topk", -1) < 0:
        out["norm_topk"] = 1 if out["score_func"] == SIGMOID else 0
    if out.get("group_score", 0) == 0:
        out["group_score"] = TOP2SUM if has_bias else AMAX
    out.setdefault("add_residual", 0)
    return out


def _cfg_struct(cfg: dict) -> _Cfg:
    return _Cfg(int(cfg["n_experts"]), int(cfg["n_groups"]), int(cfg["topk_groups"]),
                int(cfg["topk"]), float(cfg["route_scale"]), int(cfg["score_func"]),
                int(cfg["dim"]), int(cfg["inter"]), int(cfg["n_shared"]),
                int(cfg["norm_topk"]), int(cfg["group_score"]), int(cfg.get("add_residual", 0)))


def _as_raw(a):
    """Return (contiguous numpy array, dtype code): 0 = fp32, 1 = bf16 bits."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach()
            if a.device.type != "cpu":
                a = a.cpu()
            a = a.contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), 1
            if a.dtype == torch.float32:
                return a.numpy(), 0
            raise TypeError(f"unsupported dtype {a.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.uint16:
        return a, 1
    raise TypeError(f"unsupported dtype {a.dtype}")


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def gate_logits(cfg: dict, x, w_gate) -> np.ndarray:
    """fp32 logits [T, E] = x W_g^T, accumulated in double."""
    xa, dt = _as_raw(x)
    wa, dt2 = _as_raw(w_gate)
    assert dt == dt2
    T = xa.shape[0]
    out = np.empty((T, cfg["n_experts"]), np.float32)
    c = _cfg_struct(resolve(cfg, False))
    _load().oracle_gate_logits(ctypes.byref(c), T, dt, _ptr(xa), _ptr(wa), _ptr(out))
    return out


def scores(cfg: dict, logits: np.ndarray) -> np.ndarray:
    logits = np.ascontiguousarray(logits, np.float32)
    out = np.empty_like(logits)
    c = _cfg_struct(resolve(cfg, False))
    _load().oracle_scores(ctypes.byref(c), logits.shape[0], _ptr(logits), _ptr(out))
    return out


def select(cfg: dict, s: np.ndarray, bias=None) -> dict:
    """Gate steps 2-5 from fp32 scores [T, E]; bias [E] fp32 or None."""
    s = np.ascontiguousarray(s, np.float32)
    T, E = s.shape
    rc = resolve(cfg, bias is not None)
    G, k = rc["n_groups"], rc["topk"]
    b = None if bias is None else np.ascontiguousarray(_as_raw(bias)[0], np.float32)
    out = dict(keys=np.empty((T, E), np.float32), gsc=np.empty((T, G), np.float32),
               idx=np.empty((T, k), np.int32), w=np.empty((T, k), np.float32),
               kth_margin=np.empty(T, np.float32), grp_margin=np.empty(T, np.float32))
    c = _cfg_struct(rc)
    _load().oracle_select(ctypes.byref(c), T, _ptr(s), _ptr(b), _ptr(out["keys"]),
                          _ptr(out["gsc"]), _ptr(out["idx"]), _ptr(out["w"]),
                          _ptr(out["kth_margin"]), _ptr(out["grp_margin"]))
    return out


def gate(cfg: dict, x, w_gate, bias=None) -> dict:
    """The whole gate: logits, scores, keys, group scores, idx, w and margins."""
    l = gate_logits(cfg, x, w_gate)
    s = scores(cfg, l)
    out = select(cfg, s, bias)
    out["logits"] = l
    out["scores"] = s
    return out


def forward(cfg: dict, x, idx: np.ndarray, w: np.ndarray, w1, w3, w2, tok_ids,
            has_bias: bool) -> np.ndarray:
    """Literal loop for the tokens in ``tok_ids``; returns y [n, d] float64.

    w1/w3/w2 are sequences of E+S per-expert weights (None where unused) or
    stacked [E+S, ...] tensors.
    """
    xa, dt = _as_raw(x)
    T = xa.shape[0]
    rc = resolve(cfg, has_bias)
    n_all = rc["n_experts"] + rc["n_shared"]
    keep = []

    def ptrs(ws):
        arr = (ctypes.c_void_p * n_all)()
        for e in range(n_all):
            we = ws[e]
            if we is None:
                arr[e] = None
                continue
            a, d2 = _as_raw(we)
            assert d2 == dt, "weights and activations must share a dtype"
            keep.append(a)
            arr[e] = a.ctypes.data
        return arr

    p1, p3, p2 = ptrs(w1), ptrs(w3), ptrs(w2)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    tok = np.ascontiguousarray(np.asarray(tok_ids, np.int64))
    y = np.empty((tok.shape[0], rc["dim"]), np.float64)
    c = _cfg_struct(rc)
    rcode = _load().oracle_forward(ctypes.byref(c), T, dt, _ptr(xa), _ptr(idx), _ptr(w),
                                   p1, p3, p2, tok.shape[0], _ptr(tok), _ptr(y))
    if rcode != 0:
        raise ValueError("oracle_forward: bad token id or missing expert weights")
    return y


def expert_hidden(cfg: dict, x, w1_e, w3_e, tok_ids) -> np.ndarray:
    """h = silu(W1 u) * W3 u for one expert, [n, I] float64."""
    xa, dt = _as_raw(x)
    a1, _ = _as_raw(w1_e)
    a3, _ = _as_raw(w3_e)
    tok = np.ascontiguousarray(np.asarray(tok_ids, np.int64))
    h = np.empty((tok.shape[0], cfg["inter"]), np.float64)
    c = _cfg_struct(resolve(cfg, False))
    rcode = _load().oracle_expert_hidden(ctypes.byref(c), xa.shape[0], dt, _ptr(xa), _ptr(a1),
                                         _ptr(a3), tok.shape[0], _ptr(tok), _ptr(h))
    if rcode != 0:
        raise ValueError("oracle_expert_hidden: bad token id")
    return h


def expert_load(cfg: dict, idx: np.ndarray) -> np.ndarray:
    """Picks per routed expert (histogram of idx [T, k]), int64 [E]."""
    idx = np.ascontiguousarray(idx, np.int32)
    out = np.empty(cfg["n_experts"], np.int64)
    c = _cfg_struct(resolve(dict(cfg, topk=idx.shape[1]), False))
    if _load().oracle_expert_load(ctypes.byref(c), idx.shape[0], _ptr(idx), _ptr(out)) != 0:
        raise ValueError("oracle_expert_load: expert index out of range")
    return out


def bias_update(cfg: dict, idx: np.ndarray, gamma: float, bias) -> np.ndarray:
    """Aux-loss-free bias update: returns the new fp32 bias [E]."""
    idx = np.ascontiguousarray(idx, np.int32)
    b = np.array(_as_raw(bias)[0], np.float32, copy=True)
    c = _cfg_struct(resolve(dict(cfg, topk=idx.shape[1]), False))
    if _load().oracle_bias_update(ctypes.byref(c), idx.shape[0], _ptr(idx), ctypes.c_float(gamma),
                                  _ptr(b)) != 0:
        raise ValueError("oracle_bias_update: expert index out of range")
    return b


def balance_stats(cfg: dict, s: np.ndarray, idx: np.ndarray, alpha: float) -> dict:
    """f [E], P [E] and L_Bal = alpha * sum f P, float64, from fp32 scores [T, E]."""
    s = np.ascontiguousarray(s, np.float32)
    idx = np.ascontiguousarray(idx, np.int32)
    E = s.shape[1]
    f, P, loss = np.empty(E, np.float64), np.empty(E, np.float64), np.empty(1, np.float64)
    c = _cfg_struct(resolve(dict(cfg, n_experts=E, topk=idx.shape[1]), False))
    if _load().oracle_balance_stats(ctypes.byref(c), s.shape[0], _ptr(s), _ptr(idx),
                                    ctypes.c_double(alpha), _ptr(f), _ptr(P), _ptr(loss)) != 0:
        raise ValueError("oracle_balance_stats: expert index out of range")
    return dict(f=f, P=P, loss=float(loss[0]))


# ----------------------------------------------------------------------------
# MXFP8 (E4M3 elements, one power-of-two scale per 32 along K)
# ----------------------------------------------------------------------------
def e4m3_encode(v) -> np.ndarray:
    """E4M3 codes (uint8) of float64 values, round to nearest even, saturating at 448."""
    v = np.ascontiguousarray(np.asarray(v, np.float64))
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e4m3_encode(v.size, _ptr(v), _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(c, np.uint8))
    out = np.empty(c.shape, np.float64)
    _load().oracle_e4m3_decode(c.size, _ptr(c), _ptr(out))
    return out


def mx_quantize(a) -> tuple[np.ndarray, np.ndarray]:
    """[rows, K] (fp32, bf16 tensor or float64) -> (codes [rows, K] uint8,
    biased scale exponents [rows, K/32] uint8)."""
    if isinstance(a, np.ndarray) and a.dtype == np.float64:
        raw, dt = np.ascontiguousarray(a), 2
    else:
        raw, dt = _as_raw(a)
    rows, K = raw.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    if _load().oracle_mx_quantize(rows, K, dt, _ptr(raw), _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("mx_quantize: K must be a multiple of 32")
    return codes, scales


def mx_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    _load().oracle_mx_dequantize(rows, K, _ptr(codes), _ptr(scales), _ptr(out))
    return out


def forward_mxfp8(cfg: dict, x, idx, w, w1, w3, w2, tok_ids, has_bias: bool,
                  quantize_hidden: bool = True) -> np.ndarray:
    """The literal loop with MXFP8 expert weights. w1/w3/w2: sequences of E+S
    (codes, scales) pairs (None where unused); x bf16 [T, d]. Returns y [n, d]."""
    xa, dt = _as_raw(x)
    assert dt == 1, "the FP8 form takes bf16 tokens"
    T = xa.shape[0]
    rc = resolve(cfg, has_bias)
    n_all = rc["n_experts"] + rc["n_shared"]
    keep = []

    def ptrs(ws, part):
        arr = (ctypes.c_void_p * n_all)()
        for e in range(n_all):
            if ws[e] is None:
                arr[e] = None
                continue
            a = np.ascontiguousarray(ws[e][part], np.uint8)
            keep.append(a)
            arr[e] = a.ctypes.data
        return arr

    tok = np.ascontiguousarray(np.asarray(tok_ids, np.int64))
    y = np.empty((tok.shape[0], rc["dim"]), np.float64)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    c = _cfg_struct(rc)
    code = _load().oracle_forward_mxfp8(
        ctypes.byref(c), T, _ptr(xa), _ptr(idx), _ptr(w), ptrs(w1, 0), ptrs(w1, 1), ptrs(w3, 0),
        ptrs(w3, 1), ptrs(w2, 0), ptrs(w2, 1), int(bool(quantize_hidden)), tok.shape[0], _ptr(tok),
        _ptr(y))
    if code != 0:
        raise ValueError("oracle_forward_mxfp8: bad token id, missing weights or dims not multiples of 32")
    return y


# ----------------------------------------------------------------------------
# MXFP4 (E2M1 elements, one power-of-two scale per 32 along K)
# ----------------------------------------------------------------------------
def e2m1_encode(v) -> np.ndarray:
    """E2M1 codes (uint8 0..15, sign in bit 3) of float64 values, round to
    nearest even, saturating at 6."""
    v = np.ascontiguousarray(np.asarray(v, np.float64))
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e2m1_encode(v.size, _ptr(v), _ptr(out))
    return out


def e2m1_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(c, np.uint8))
    out = np.empty(c.shape, np.float64)
    _load().oracle_e2m1_decode(c.size, _ptr(c), _ptr(out))
    return out


def mx4_quantize(a) -> tuple[np.ndarray, np.ndarray]:
    """[rows, K] (fp32, bf16 tensor or float64) -> (codes [rows, K] uint8, one
    E2M1 code per byte; biased scale exponents [rows, K/32] uint8)."""
    if isinstance(a, np.ndarray) and a.dtype == np.float64:
        raw, dt = np.ascontiguousarray(a), 2
    else:
        raw, dt = _as_raw(a)
    rows, K = raw.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    if _load().oracle_mx4_quantize(rows, K, dt, _ptr(raw), _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("mx4_quantize: K must be a multiple of 32")
    return codes, scales


def mx4_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    _load().oracle_mx4_dequantize(rows, K, _ptr(codes), _ptr(scales), _ptr(out))
    return out


def e2m1_as_e4m3(codes: np.ndarray) -> np.ndarray:
    """The E4M3 code of each E2M1 code's value (every E2M1 value is an E4M3
    value, so this loses nothing)."""
    table = e4m3_encode(e2m1_decode(np.arange(16, dtype=np.uint8)))
    return table[np.asarray(codes, np.uint8)]


def forward_mxfp4(cfg: dict, x, idx, w, w1, w3, w2, tok_ids, has_bias: bool) -> np.ndarray:
    """The literal loop with MXFP4 expert weights (tokens and hidden vectors in
    MXFP8, as in the 8-bit form). w1/w3/w2: sequences of E+S (E2M1 codes, scales)
    pairs (None where unused). The weights' values are those of E4M3 codes with
    the same scales, so this is forward_mxfp8 on the re-encoded codes."""
    conv = lambda ws: [None if q is None else (e2m1_as_e4m3(q[0]), q[1]) for q in ws]
    return forward_mxfp8(cfg, x, idx, w, conv(w1), conv(w3), conv(w2), tok_ids, has_bias)


def forward_part(cfg: dict, x, idx, w, w1, w3, w2, tok_ids, has_bias: bool, expert_begin: int,
                 expert_end: int, shared: bool = True) -> tuple[np.ndarray, np.ndarray | None]:
    """One rank's part of the expert-parallel forward: (y_routed over experts
    [expert_begin, expert_end), y_shared or None), each [n, d] float64."""
    xa, dt = _as_raw(x)
    T = xa.shape[0]
    rc = resolve(cfg, has_bias)
    n_all = rc["n_experts"] + rc["n_shared"]
    keep = []

    def ptrs(ws):
        arr = (ctypes.c_void_p * n_all)()
        for e in range(n_all):
            if ws[e] is None:
                arr[e] = None
                continue
            a, d2 = _as_raw(ws[e])
            assert d2 == dt
            keep.append(a)
            arr[e] = a.ctypes.data
        return arr

    tok = np.ascontiguousarray(np.asarray(tok_ids, np.int64))
    yr = np.empty((tok.shape[0], rc["dim"]), np.float64)
    ys = np.empty((tok.shape[0], rc["dim"]), np.float64) if shared else None
    c = _cfg_struct(rc)
    code = _load().oracle_forward_part(
        ctypes.byref(c), T, dt, _ptr(xa), _ptr(np.ascontiguousarray(idx, np.int32)),
        _ptr(np.ascontiguousarray(w, np.float32)), ptrs(w1), ptrs(w3), ptrs(w2),
        int(expert_begin), int(expert_end), tok.shape[0], _ptr(tok), _ptr(yr), _ptr(ys))
    if code != 0:
        raise ValueError("oracle_forward_part: bad token id or missing expert weights")
    return yr, ys
