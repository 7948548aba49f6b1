"""Python binding of libktmoe.so (include/ktmoe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module only
turns torch tensors into pointers, picks the current CUDA stream, and raises on
error codes. There is no fallback: if the library is missing or fails to load,
importing the entry points raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
# KTMOE_LIB=checked loads the checked build (libktmoe_checked.so: every index
# a kernel takes from another kernel's output is range-checked; same entry
# points and results); anything else, or unset, the release build.
LIB_NAMES = {"release": "libktmoe.so", "checked": "libktmoe_checked.so"}
LIB_PATH = os.path.join(HERE, LIB_NAMES.get(os.environ.get("KTMOE_LIB", "release"), "libktmoe.so"))

KT_SCORE_SIGMOID, KT_SCORE_SOFTMAX = 0, 1
KT_GROUP_AUTO, KT_GROUP_AMAX, KT_GROUP_TOP2SUM = 0, 1, 2
KT_OK = 0
KT_ERR_INVALID_CONFIG, KT_ERR_NULL, KT_ERR_WORKSPACE, KT_ERR_ALIGN = -1, -2, -3, -4
KT_ERR_CUDA, KT_ERR_TIMEOUT, KT_ERR_UNSUPPORTED, KT_ERR_SCRATCH_LIMIT = -5, -6, -7, -8
KT_ERR_BOUNDS = -9
KT_STATIC_SCRATCH_BYTES = 32 << 20
KT_DTYPE_F32, KT_DTYPE_BF16, KT_DTYPE_MXFP8, KT_DTYPE_MXFP4 = 0, 1, 2, 3

# Every symbol include/ktmoe.h declares.
EXPORTS = ("kt_moe_validate", "kt_moe_workspace_size", "kt_moe_gate", "kt_moe_forward",
           "kt_moe_forward_profiled", "kt_moe_forward_static", "kt_moe_static_scratch",
           "kt_moe_check", "kt_moe_workspace_layout", "kt_moe_strerror", "kt_moe_version",
           "kt_moe_scores", "kt_moe_bias_update", "kt_moe_balance_workspace_size",
           "kt_moe_balance_stats", "kt_moe_graph_create", "kt_moe_graph_launch",
           "kt_moe_graph_destroy", "kt_moe_mxfp8_quantize", "kt_moe_mxfp8_scale_bytes",
           "kt_moe_mxfp8_pack", "kt_moe_forward_mxfp8", "kt_moe_graph_create_mxfp8",
           "kt_moe_forward_local", "kt_moe_forward_local_mxfp8", "kt_moe_ep_finish",
           "kt_moe_mxfp8_scale_bytes_local", "kt_moe_mxfp8_pack_local", "kt_moe_forward_placed",
           "kt_moe_forward_placed_mxfp8", "kt_moe_selftest_timeout", "kt_moe_checked_build",
           "kt_moe_mxfp4_quantize")


class kt_moe_config(ctypes.Structure):
    _fields_ = [("n_experts", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("route_scale", ctypes.c_float), ("score_func", ctypes.c_int32),
                ("dim", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("norm_topk", ctypes.c_int32),
                ("group_score", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("add_residual", ctypes.c_int32), ("y_fp32", ctypes.c_int32)]


class kt_moe_ws_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("error_word", "logits", "logits_splits", "counts", "offsets",
                                              "row_of", "tok_of", "row_weight", "hidden",
                                              "expert_out", "meta", "chunks", "tiles_up",
                                              "tiles_down", "total", "xq", "xs", "xperm",
                                              "tok_sf", "hid_sf")]


class KtMoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {strerror(code)} (code {code})")
        self.code = code


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libktmoe.so (raises OSError if it is missing: no fallback path)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise OSError(f"{LIB_PATH} not found: build it with "
                              "`python -m mixture_experts_layer_34_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I64, CP = ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(kt_moe_config)
            L.kt_moe_validate.argtypes = [CP, I64, ctypes.c_int]
            L.kt_moe_validate.restype = ctypes.c_int
            L.kt_moe_workspace_size.argtypes = [CP, I64]
            L.kt_moe_workspace_size.restype = ctypes.c_size_t
            L.kt_moe_gate.argtypes = [CP, I64, P, P, P, P, P, P, P, ctypes.c_size_t, P]
            L.kt_moe_gate.restype = ctypes.c_int
            L.kt_moe_forward.argtypes = [CP, I64, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
            L.kt_moe_forward.restype = ctypes.c_int
            L.kt_moe_forward_profiled.argtypes = [CP, I64, P, P, P, P, P, P, P, P, P, P,
                                                  ctypes.c_size_t, P, ctypes.POINTER(P)]
            L.kt_moe_forward_profiled.restype = ctypes.c_int
            L.kt_moe_forward_static.argtypes = [CP, I64, P, P, P, P, P, P, P, P, P, P]
            L.kt_moe_forward_static.restype = ctypes.c_int
            L.kt_moe_static_scratch.argtypes = []
            L.kt_moe_static_scratch.restype = ctypes.c_void_p
            L.kt_moe_check.argtypes = [P, P]
            L.kt_moe_check.restype = ctypes.c_int
            L.kt_moe_workspace_layout.argtypes = [CP, I64, ctypes.POINTER(kt_moe_ws_layout)]
            L.kt_moe_workspace_layout.restype = ctypes.c_int
            L.kt_moe_strerror.argtypes = [ctypes.c_int]
            L.kt_moe_strerror.restype = ctypes.c_char_p
            L.kt_moe_scores.argtypes = [CP, I64, P, P, P, P, ctypes.c_size_t, P]
            L.kt_moe_scores.restype = ctypes.c_int
            L.kt_moe_bias_update.argtypes = [CP, I64, P, P, ctypes.c_float, P, P]
            L.kt_moe_bias_update.restype = ctypes.c_int
            L.kt_moe_balance_workspace_size.argtypes = [CP, I64]
            L.kt_moe_balance_workspace_size.restype = ctypes.c_size_t
            L.kt_moe_balance_stats.argtypes = [CP, I64, P, P, ctypes.c_float, P, P, P, P,
                                               ctypes.c_size_t, P]
            L.kt_moe_balance_stats.restype = ctypes.c_int
            L.kt_moe_graph_create.argtypes = [CP, I64, P, P, P, P, P, P, P, P, P, P,
                                              ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p)]
            L.kt_moe_graph_create.restype = ctypes.c_int
            L.kt_moe_graph_create_mxfp8.argtypes = [CP, I64, P, P, P, P, P, P, P, P, P, P, P, P,
                                                    ctypes.c_size_t,
                                                    ctypes.POINTER(ctypes.c_void_p)]
            L.kt_moe_graph_create_mxfp8.restype = ctypes.c_int
            L.kt_moe_graph_launch.argtypes = [P, P]
            L.kt_moe_graph_launch.restype = ctypes.c_int
            L.kt_moe_graph_destroy.argtypes = [P]
            L.kt_moe_graph_destroy.restype = None
            L.kt_moe_mxfp8_quantize.argtypes = [I64, I64, P, P, P, P]
            L.kt_moe_mxfp8_quantize.restype = ctypes.c_int
            L.kt_moe_mxfp4_quantize.argtypes = [I64, I64, P, P, P, P]
            L.kt_moe_mxfp4_quantize.restype = ctypes.c_int
            L.kt_moe_mxfp8_scale_bytes.argtypes = [CP, ctypes.c_int]
            L.kt_moe_mxfp8_scale_bytes.restype = ctypes.c_size_t
            L.kt_moe_mxfp8_pack.argtypes = [CP, P, P, P, P, P, P, P, P, P]
            L.kt_moe_mxfp8_pack.restype = ctypes.c_int
            L.kt_moe_forward_mxfp8.argtypes = [CP, I64, P, P, P, P, P, P, P, P, P, P, P, P,
                                               ctypes.c_size_t, P, P]
            L.kt_moe_forward_mxfp8.restype = ctypes.c_int
            C = ctypes.c_int
            L.kt_moe_forward_local.argtypes = [CP, I64, P, P, P, C, C, I64, I64, P, P, P, P, P, P,
                                               P, ctypes.c_size_t, P]
            L.kt_moe_forward_local.restype = ctypes.c_int
            L.kt_moe_forward_local_mxfp8.argtypes = [CP, I64, P, P, P, C, C, I64, I64, P, P, P, P,
                                                     P, P, P, P, P, ctypes.c_size_t, P]
            L.kt_moe_forward_local_mxfp8.restype = ctypes.c_int
            L.kt_moe_forward_placed.argtypes = [CP, I64, P, P, P, P, I64, I64, P, P, P, P, P, P,
                                                P, ctypes.c_size_t, P]
            L.kt_moe_forward_placed.restype = ctypes.c_int
            L.kt_moe_forward_placed_mxfp8.argtypes = [CP, I64, P, P, P, P, I64, I64, P, P, P, P, P,
                                                      P, P, P, P, ctypes.c_size_t, P]
            L.kt_moe_forward_placed_mxfp8.restype = ctypes.c_int
            L.kt_moe_ep_finish.argtypes = [CP, I64, P, P, P, P]
            L.kt_moe_ep_finish.restype = ctypes.c_int
            L.kt_moe_mxfp8_scale_bytes_local.argtypes = [CP, C, C, C]
            L.kt_moe_mxfp8_scale_bytes_local.restype = ctypes.c_size_t
            L.kt_moe_mxfp8_pack_local.argtypes = [CP, C, C, P, P, P, P, P, P, P, P, P]
            L.kt_moe_mxfp8_pack_local.restype = ctypes.c_int
            L.kt_moe_selftest_timeout.argtypes = [P, I64, P]
            L.kt_moe_selftest_timeout.restype = ctypes.c_int
            L.kt_moe_version.argtypes = []
            L.kt_moe_version.restype = ctypes.c_int
            L.kt_moe_checked_build.argtypes = []
            L.kt_moe_checked_build.restype = ctypes.c_int
            _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().kt_moe_strerror(int(code)).decode()


def make_config(n_experts, n_groups, topk_groups, topk, route_scale, score_func, dim, inter,
                n_shared, norm_topk=-1, group_score=KT_GROUP_AUTO, dtype=KT_DTYPE_BF16,
                add_residual=0, y_fp32=0) -> kt_moe_config:
    return kt_moe_config(int(n_experts), int(n_groups), int(topk_groups), int(topk),
                         float(route_scale), int(score_func), int(dim), int(inter), int(n_shared),
                         int(norm_topk), int(group_score), int(dtype), int(add_residual),
                         int(y_fp32))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def kt_moe_validate(cfg: kt_moe_config, T: int, has_bias: bool) -> int:
    return lib().kt_moe_validate(ctypes.byref(cfg), int(T), int(bool(has_bias)))


def kt_moe_workspace_size(cfg: kt_moe_config, T: int) -> int:
    return int(lib().kt_moe_workspace_size(ctypes.byref(cfg), int(T)))


def kt_moe_workspace_layout(cfg: kt_moe_config, T: int) -> dict:
    out = kt_moe_ws_layout()
    rc = lib().kt_moe_workspace_layout(ctypes.byref(cfg), int(T), ctypes.byref(out))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_workspace_layout", rc)
    return {n: getattr(out, n) for n, _ in kt_moe_ws_layout._fields_}


def kt_moe_gate(cfg, T, x, w_gate, bias, scores_in, topk_idx, topk_w, workspace, stream=None):
    rc = lib().kt_moe_gate(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
                           _ptr(scores_in), _ptr(topk_idx), _ptr(topk_w), _ptr(workspace),
                           _nbytes(workspace), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_gate", rc)


def kt_moe_scores(cfg, T, x, w_gate, scores_out, workspace, stream=None):
    rc = lib().kt_moe_scores(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(scores_out),
                             _ptr(workspace), _nbytes(workspace), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_scores", rc)


def kt_moe_bias_update(cfg, T, topk_idx, bias, gamma, load_out=None, stream=None):
    rc = lib().kt_moe_bias_update(ctypes.byref(cfg), int(T), _ptr(topk_idx), _ptr(bias),
                                  ctypes.c_float(gamma), _ptr(load_out), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_bias_update", rc)


def kt_moe_balance_workspace_size(cfg: kt_moe_config, T: int) -> int:
    return int(lib().kt_moe_balance_workspace_size(ctypes.byref(cfg), int(T)))


def kt_moe_balance_stats(cfg, T, scores, topk_idx, alpha, f_out, P_out, loss_out, workspace,
                         stream=None):
    rc = lib().kt_moe_balance_stats(ctypes.byref(cfg), int(T), _ptr(scores), _ptr(topk_idx),
                                    ctypes.c_float(alpha), _ptr(f_out), _ptr(P_out),
                                    _ptr(loss_out), _ptr(workspace), _nbytes(workspace),
                                    _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_balance_stats", rc)


def kt_moe_forward(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out, workspace,
                   stream=None):
    rc = lib().kt_moe_forward(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
                              _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y), _ptr(topk_idx_out),
                              _ptr(topk_w_out), _ptr(workspace), _nbytes(workspace),
                              _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward", rc)


class KtMoeGraph:
    """A captured kt_moe_forward (kt_moe_graph_create); launch() replays it.

    Holds references to every tensor bound into the graph so that none is freed
    while the graph exists."""

    def __init__(self, cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out,
                 workspace):
        self._keep = (x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out, workspace)
        h = ctypes.c_void_p(0)
        rc = lib().kt_moe_graph_create(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate),
                                       _ptr(bias), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y),
                                       _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace),
                                       _nbytes(workspace), ctypes.byref(h))
        if rc != KT_OK:
            raise KtMoeError("kt_moe_graph_create", rc)
        self._h = h

    @classmethod
    def mxfp8(cls, cfg, T, x, w_gate, bias, q, y, topk_idx_out, topk_w_out, workspace):
        """A captured kt_moe_forward_mxfp8; q holds the packed weights (pack_mxfp8)."""
        self = cls.__new__(cls)
        self._keep = (x, w_gate, bias, q, y, topk_idx_out, topk_w_out, workspace)
        h = ctypes.c_void_p(0)
        rc = lib().kt_moe_graph_create_mxfp8(
            ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias), _ptr(q["w1q"]),
            _ptr(q["w3q"]), _ptr(q["w2q"]), _ptr(q["sf_up"]), _ptr(q["sf_down"]), _ptr(y),
            _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace), _nbytes(workspace),
            ctypes.byref(h))
        if rc != KT_OK:
            raise KtMoeError("kt_moe_graph_create_mxfp8", rc)
        self._h = h
        return self

    def launch(self, stream=None):
        rc = lib().kt_moe_graph_launch(self._h, _stream(stream))
        if rc != KT_OK:
            raise KtMoeError("kt_moe_graph_launch", rc)

    def destroy(self):
        if self._h:
            lib().kt_moe_graph_destroy(self._h)
            self._h = ctypes.c_void_p(0)
            self._keep = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def kt_moe_mxfp8_quantize(rows, K, src, codes, scales, stream=None):
    rc = lib().kt_moe_mxfp8_quantize(int(rows), int(K), _ptr(src), _ptr(codes), _ptr(scales),
                                     _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_mxfp8_quantize", rc)


def kt_moe_mxfp4_quantize(rows, K, src, codes, scales, stream=None):
    """bf16 [rows, K] -> packed E2M1 codes [rows, K/2] and scale bytes [rows, K/32]."""
    rc = lib().kt_moe_mxfp4_quantize(int(rows), int(K), _ptr(src), _ptr(codes), _ptr(scales),
                                     _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_mxfp4_quantize", rc)


def _code_shape(cfg, shape) -> tuple:
    """Shape of the weight codes: one byte per element (MXFP8), or two 4-bit
    codes per byte along K (MXFP4)."""
    shape = tuple(shape)
    return shape[:-1] + (shape[-1] // 2,) if cfg.dtype == KT_DTYPE_MXFP4 else shape


def kt_moe_mxfp8_scale_bytes(cfg: kt_moe_config, down: bool) -> int:
    return int(lib().kt_moe_mxfp8_scale_bytes(ctypes.byref(cfg), int(bool(down))))


def kt_moe_mxfp8_pack(cfg, w1, w3, w2, w1q, w3q, w2q, sf_up, sf_down, stream=None):
    rc = lib().kt_moe_mxfp8_pack(ctypes.byref(cfg), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(w1q),
                                 _ptr(w3q), _ptr(w2q), _ptr(sf_up), _ptr(sf_down), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_mxfp8_pack", rc)


def pack_mxfp8(cfg, w1, w3, w2, stream=None) -> dict:
    """Allocate the MXFP8 (or, for an MXFP4 config, packed 4-bit) codes (W1 and
    W3 as the two halves of one buffer) and the packed scales for bf16 weights,
    and pack them."""
    import torch
    w13 = torch.empty((2,) + _code_shape(cfg, w1.shape), dtype=torch.uint8, device=w1.device)
    out = dict(w1q=w13[0], w3q=w13[1],      # W1's codes below W3's, as the forward needs
               w2q=torch.empty(_code_shape(cfg, w2.shape), dtype=torch.uint8, device=w2.device),
               sf_up=torch.empty(kt_moe_mxfp8_scale_bytes(cfg, False), dtype=torch.uint8,
                                 device=w1.device),
               sf_down=torch.empty(kt_moe_mxfp8_scale_bytes(cfg, True), dtype=torch.uint8,
                                   device=w1.device))
    kt_moe_mxfp8_pack(cfg, w1, w3, w2, out["w1q"], out["w3q"], out["w2q"], out["sf_up"],
                      out["sf_down"], stream)
    return out


def kt_moe_forward_mxfp8(cfg, T, x, w_gate, bias, w1q, w3q, w2q, sf_up, sf_down, y, topk_idx_out,
                         topk_w_out, workspace, stream=None, stage_events=None):
    ev = None
    if stage_events is not None:
        ev = (ctypes.c_void_p * KT_STAGE_EVENTS)(*[ctypes.c_void_p(e.cuda_event)
                                                   if e is not None else None
                                                   for e in stage_events])
    rc = lib().kt_moe_forward_mxfp8(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
                                    _ptr(w1q), _ptr(w3q), _ptr(w2q), _ptr(sf_up), _ptr(sf_down),
                                    _ptr(y), _ptr(topk_idx_out), _ptr(topk_w_out),
                                    _ptr(workspace), _nbytes(workspace), _stream(stream), ev)
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward_mxfp8", rc)


def kt_moe_forward_local(cfg, T, x, w_gate, bias, expert_begin, expert_end, shared_begin,
                         shared_end, w1, w3, w2, y_part, topk_idx_out, topk_w_out, workspace,
                         stream=None):
    """One rank's part of the expert-parallel forward: fp32 y_part from routed
    experts [expert_begin, expert_end) (local weight slots, then the shared
    experts) and the shared experts on tokens [shared_begin, shared_end)."""
    rc = lib().kt_moe_forward_local(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
                                    int(expert_begin), int(expert_end), int(shared_begin),
                                    int(shared_end), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y_part),
                                    _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace),
                                    _nbytes(workspace), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward_local", rc)


def kt_moe_forward_local_mxfp8(cfg, T, x, w_gate, bias, expert_begin, expert_end, shared_begin,
                               shared_end, w1q, w3q, w2q, sf_up, sf_down, y_part, topk_idx_out,
                               topk_w_out, workspace, stream=None):
    rc = lib().kt_moe_forward_local_mxfp8(
        ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias), int(expert_begin),
        int(expert_end), int(shared_begin), int(shared_end), _ptr(w1q), _ptr(w3q), _ptr(w2q),
        _ptr(sf_up), _ptr(sf_down), _ptr(y_part), _ptr(topk_idx_out), _ptr(topk_w_out),
        _ptr(workspace), _nbytes(workspace), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward_local_mxfp8", rc)


def _slot_array(expert_slot):
    arr = (ctypes.c_int32 * len(expert_slot))(*[int(v) for v in expert_slot])
    return arr


def kt_moe_forward_placed(cfg, T, x, w_gate, bias, expert_slot, shared_begin, shared_end, w1, w3,
                          w2, y_part, topk_idx_out, topk_w_out, workspace, stream=None):
    """kt_moe_forward_local with any placement: expert_slot[e] = the weight slot
    of routed expert e on this rank, or -1 (a sequence of n_experts ints)."""
    tab = _slot_array(expert_slot)
    rc = lib().kt_moe_forward_placed(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
                                     ctypes.cast(tab, ctypes.c_void_p), int(shared_begin),
                                     int(shared_end), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y_part),
                                     _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace),
                                     _nbytes(workspace), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward_placed", rc)


def kt_moe_forward_placed_mxfp8(cfg, T, x, w_gate, bias, expert_slot, shared_begin, shared_end,
                                w1q, w3q, w2q, sf_up, sf_down, y_part, topk_idx_out, topk_w_out,
                                workspace, stream=None):
    tab = _slot_array(expert_slot)
    rc = lib().kt_moe_forward_placed_mxfp8(
        ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
        ctypes.cast(tab, ctypes.c_void_p), int(shared_begin), int(shared_end), _ptr(w1q),
        _ptr(w3q), _ptr(w2q), _ptr(sf_up), _ptr(sf_down), _ptr(y_part), _ptr(topk_idx_out),
        _ptr(topk_w_out), _ptr(workspace), _nbytes(workspace), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward_placed_mxfp8", rc)


def kt_moe_ep_finish(cfg, T, y_sum, x, y, stream=None):
    """y = y_sum (+ x with the residual) in y's type, after the sum over ranks."""
    rc = lib().kt_moe_ep_finish(ctypes.byref(cfg), int(T), _ptr(y_sum), _ptr(x), _ptr(y),
                                _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_ep_finish", rc)


def kt_moe_mxfp8_scale_bytes_local(cfg, expert_begin, expert_end, down) -> int:
    return int(lib().kt_moe_mxfp8_scale_bytes_local(ctypes.byref(cfg), int(expert_begin),
                                                    int(expert_end), int(bool(down))))


def kt_moe_mxfp8_pack_local(cfg, expert_begin, expert_end, w1, w3, w2, w1q, w3q, w2q, sf_up,
                            sf_down, stream=None):
    rc = lib().kt_moe_mxfp8_pack_local(ctypes.byref(cfg), int(expert_begin), int(expert_end),
                                       _ptr(w1), _ptr(w3), _ptr(w2), _ptr(w1q), _ptr(w3q),
                                       _ptr(w2q), _ptr(sf_up), _ptr(sf_down), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_mxfp8_pack_local", rc)


def pack_mxfp8_local(cfg, expert_begin, expert_end, w1, w3, w2, stream=None) -> dict:
    """pack_mxfp8 for one rank's local stacks (routed experts [expert_begin,
    expert_end), then the shared ones)."""
    import torch
    w13 = torch.empty((2,) + _code_shape(cfg, w1.shape), dtype=torch.uint8, device=w1.device)
    sb = lambda down: kt_moe_mxfp8_scale_bytes_local(cfg, expert_begin, expert_end, down)
    out = dict(w1q=w13[0], w3q=w13[1],
               w2q=torch.empty(_code_shape(cfg, w2.shape), dtype=torch.uint8, device=w2.device),
               sf_up=torch.empty(sb(False), dtype=torch.uint8, device=w1.device),
               sf_down=torch.empty(sb(True), dtype=torch.uint8, device=w1.device))
    kt_moe_mxfp8_pack_local(cfg, expert_begin, expert_end, w1, w3, w2, out["w1q"], out["w3q"],
                            out["w2q"], out["sf_up"], out["sf_down"], stream)
    return out


KT_STAGE_EVENTS = 6
STAGES = ("gate", "permute", "up_gemm", "down_gemm", "combine")


def kt_moe_forward_profiled(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out,
                            workspace, events, stream=None):
    """kt_moe_forward recording `events` (6 torch.cuda.Event, created with
    enable_timing=True) at the stage boundaries on the launch stream."""
    if len(events) != KT_STAGE_EVENTS:
        raise ValueError(f"need {KT_STAGE_EVENTS} events")
    arr = (ctypes.c_void_p * KT_STAGE_EVENTS)(*[ctypes.c_void_p(e.cuda_event) if e is not None
                                                 else None for e in events])
    rc = lib().kt_moe_forward_profiled(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
                                       _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y), _ptr(topk_idx_out),
                                       _ptr(topk_w_out), _ptr(workspace), _nbytes(workspace),
                                       _stream(stream), arr)
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward_profiled", rc)


def kt_moe_forward_static(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out,
                          stream=None):
    """kt_moe_forward with the library's static device scratch: no workspace,
    no allocation (see include/ktmoe.h for its limit and sharing rules)."""
    rc = lib().kt_moe_forward_static(ctypes.byref(cfg), int(T), _ptr(x), _ptr(w_gate), _ptr(bias),
                                     _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y), _ptr(topk_idx_out),
                                     _ptr(topk_w_out), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_forward_static", rc)


def kt_moe_static_scratch() -> int:
    """Device address of the current device's static scratch (0 on error)."""
    return lib().kt_moe_static_scratch() or 0


def kt_moe_check(workspace, stream=None) -> int:
    """Synchronise the stream and read the workspace's device error word."""
    return lib().kt_moe_check(_ptr(workspace), _stream(stream))


def kt_moe_selftest_timeout(workspace, limit_ns: int, stream=None):
    """Run the bounded-wait diagnostic (see include/ktmoe.h); kt_moe_check then
    reports KT_ERR_TIMEOUT."""
    rc = lib().kt_moe_selftest_timeout(_ptr(workspace), int(limit_ns), _stream(stream))
    if rc != KT_OK:
        raise KtMoeError("kt_moe_selftest_timeout", rc)


def kt_moe_version() -> int:
    return lib().kt_moe_version()


def kt_moe_checked_build() -> bool:
    return bool(lib().kt_moe_checked_build())


def config_for(layer, y_fp32: bool = False) -> kt_moe_config:
    """kt_moe_config of a workloads.LayerConfig."""
    dt = {"f32": KT_DTYPE_F32, "bf16": KT_DTYPE_BF16, "mxfp8": KT_DTYPE_MXFP8,
          "mxfp4": KT_DTYPE_MXFP4}[layer.dtype]
    return make_config(dtype=dt, y_fp32=int(y_fp32), **layer.kernel_fields())


def alloc_workspace(cfg: kt_moe_config, T: int, device="cuda"):
    """A byte tensor of kt_moe_workspace_size bytes (torch's allocator aligns to 512 B)."""
    import torch
    n = kt_moe_workspace_size(cfg, T)
    if n == 0:
        raise KtMoeError("kt_moe_workspace_size", KT_ERR_INVALID_CONFIG)
    return torch.empty(n, dtype=torch.uint8, device=device)
