"""The C-ABI library: loads, exports what include/ktmoe.h declares, and rejects bad
calls on the host before any CUDA call (CPU; also safe where a GPU is present)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

from mixture_experts_layer_34_b200 import ktmoe as K
from mixture_experts_layer_34_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "ktmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kt_moe_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = K.lib()
    declared = _declared_functions()
    assert declared, "no declarations found"
    assert set(declared) == set(K.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_checked_library_exports_every_declared_symbol():
    """The checked build (-DKT_CHECKED) has the same ABI and says which it is;
    loaded in a fresh process, as the binding picks one library per process."""
    import subprocess
    import sys
    code = ("from mixture_experts_layer_34_b200 import ktmoe as K; "
            "L = K.lib(); assert K.LIB_PATH.endswith('libktmoe_checked.so'), K.LIB_PATH; "
            "missing = [n for n in K.EXPORTS if not hasattr(L, n)]; assert not missing, missing; "
            "assert K.kt_moe_checked_build(); print('ok')")
    env = dict(os.environ, KTMOE_LIB="checked")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT,
                       env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr
    if os.environ.get("KTMOE_LIB", "release") != "checked":
        assert not K.kt_moe_checked_build()


def test_library_links_no_torch():
    # The library is plain C ABI: it must not need libtorch / libc10 to load.
    import subprocess
    r = subprocess.run(["ldd", K.LIB_PATH], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "torch" not in r.stdout and "c10" not in r.stdout, r.stdout


def test_config_struct_layout_matches_header():
    assert ctypes.sizeof(K.kt_moe_config) == 14 * 4
    assert ctypes.sizeof(K.kt_moe_ws_layout) == 20 * 8


@pytest.mark.parametrize("layer", W.NAMED + W.SMALL, ids=lambda c: c.name)
def test_named_configs_validate(layer):
    cfg = K.config_for(layer)
    assert K.kt_moe_validate(cfg, layer.T, layer.bias != "none") == K.KT_OK
    ws = K.kt_moe_workspace_size(cfg, layer.T)
    assert ws > 0 and ws % 1024 == 0
    lay = K.kt_moe_workspace_layout(cfg, layer.T)
    assert lay["total"] == ws and lay["error_word"] == 0
    for key in ("hidden", "expert_out"):
        assert lay[key] % 1024 == 0
    # workspace grows with T
    assert K.kt_moe_workspace_size(cfg, layer.T * 2) > ws


BAD = [
    dict(n_experts=0), dict(n_experts=513), dict(n_groups=3),            # E % G != 0 for E=16
    dict(topk_groups=5), dict(n_groups=1, topk_groups=2), dict(topk=0),
    dict(topk=9),                                                         # > TG * E/G = 8
    dict(n_shared=-1), dict(n_shared=9), dict(route_scale=0.0), dict(route_scale=float("inf")),
    dict(route_scale=float("nan")), dict(score_func=2), dict(dtype=4), dict(dim=12),
    dict(dtype=2, dim=192), dict(dtype=3, inter=64),                     # MX: multiples of 128
    dict(inter=4), dict(norm_topk=2), dict(group_score=3), dict(add_residual=2), dict(y_fp32=2),
    dict(n_experts=16, n_groups=16, topk_groups=4, topk=4, group_score=2),  # top-2 of 1 expert
]


@pytest.mark.parametrize("bad", BAD)
def test_invalid_configs_rejected(bad):
    base = dict(n_experts=16, n_groups=4, topk_groups=2, topk=4, route_scale=2.5, score_func=0,
                dim=256, inter=128, n_shared=1, norm_topk=-1, group_score=0, dtype=K.KT_DTYPE_BF16,
                add_residual=0)
    base.update(bad)
    cfg = K.make_config(**base)
    assert K.kt_moe_validate(cfg, 64, True) == K.KT_ERR_INVALID_CONFIG
    assert K.kt_moe_workspace_size(cfg, 64) == 0


def test_token_count_limits():
    cfg = K.config_for(W.TINY)
    assert K.kt_moe_validate(cfg, 0, True) == K.KT_ERR_INVALID_CONFIG
    assert K.kt_moe_validate(cfg, 1, True) == K.KT_OK
    assert K.kt_moe_validate(cfg, 1 << 20, True) == K.KT_OK
    assert K.kt_moe_validate(cfg, (1 << 20) + 1, True) == K.KT_ERR_INVALID_CONFIG


def _call_forward(cfg, T, ptrs, ws_ptr, ws_bytes):
    L = K.lib()
    return L.kt_moe_forward(ctypes.byref(cfg), T, *[ctypes.c_void_p(p) if p else None for p in ptrs],
                            ctypes.c_void_p(ws_ptr) if ws_ptr else None, ws_bytes, None)


def test_host_side_errors_return_before_any_device_work():
    """Fake (never dereferenced) pointer values: every case must be rejected on
    the host, so this is safe with or without a GPU."""
    cfg = K.config_for(W.BY_NAME["small_sig_bias"])
    T = 300
    need = K.kt_moe_workspace_size(cfg, T)
    good = [0x10000 * (i + 1) for i in range(9)]   # x wg bias w1 w3 w2 y idx w, 16-B aligned
    ws = 0x7000000
    # NULL required pointer
    p = list(good)
    p[0] = 0
    assert _call_forward(cfg, T, p, ws, need) == K.KT_ERR_NULL
    # workspace missing / too small
    assert _call_forward(cfg, T, good, 0, need) == K.KT_ERR_WORKSPACE
    assert _call_forward(cfg, T, good, ws, need - 1) == K.KT_ERR_WORKSPACE
    # misaligned tensor and workspace
    p = list(good)
    p[3] += 8
    assert _call_forward(cfg, T, p, ws, need) == K.KT_ERR_ALIGN
    assert _call_forward(cfg, T, good, ws + 128, need) == K.KT_ERR_ALIGN
    # output aliasing the input
    p = list(good)
    p[6] = p[0]
    assert _call_forward(cfg, T, p, ws, need) == K.KT_ERR_INVALID_CONFIG
    # invalid config
    bad = K.make_config(**{**{f: getattr(cfg, f) for f, _ in K.kt_moe_config._fields_}, "topk": 0})
    assert _call_forward(bad, T, good, ws, need) == K.KT_ERR_INVALID_CONFIG


def test_gate_host_side_errors():
    cfg = K.config_for(W.BY_NAME["small_sig_bias"])
    L = K.lib()
    need = K.kt_moe_workspace_size(cfg, 300)
    V = ctypes.c_void_p
    # scores_in absent and x missing
    rc = L.kt_moe_gate(ctypes.byref(cfg), 300, None, V(0x10000), None, None, V(0x20000),
                       V(0x30000), V(0x7000000), need, None)
    assert rc == K.KT_ERR_NULL
    # outputs missing
    rc = L.kt_moe_gate(ctypes.byref(cfg), 300, V(0x10000), V(0x20000), None, None, None,
                       V(0x30000), V(0x7000000), need, None)
    assert rc == K.KT_ERR_NULL


def test_load_statistics_host_side_errors():
    """kt_moe_scores / kt_moe_bias_update / kt_moe_balance_stats reject bad
    arguments on the host (fake pointers, never dereferenced)."""
    cfg = K.config_for(W.BY_NAME["small_sig_bias"])
    L = K.lib()
    V = ctypes.c_void_p
    T = 300
    f32 = ctypes.c_float
    # bias update: gamma must be finite and >= 0; idx and bias are required
    for g in (float("nan"), float("inf"), -1e-3):
        rc = L.kt_moe_bias_update(ctypes.byref(cfg), T, V(0x10000), V(0x20000), f32(g), None, None)
        assert rc == K.KT_ERR_INVALID_CONFIG, g
    assert L.kt_moe_bias_update(ctypes.byref(cfg), T, None, V(0x20000), f32(1e-3), None,
                                None) == K.KT_ERR_NULL
    assert L.kt_moe_bias_update(ctypes.byref(cfg), T, V(0x10002), V(0x20000), f32(1e-3), None,
                                None) == K.KT_ERR_ALIGN
    # balance statistics: workspace size, alpha, pointers
    need = K.kt_moe_balance_workspace_size(cfg, T)
    assert need > 0
    bad = K.make_config(**{**{f: getattr(cfg, f) for f, _ in K.kt_moe_config._fields_}, "topk": 0})
    assert K.kt_moe_balance_workspace_size(bad, T) == 0
    args = [V(0x10000), V(0x20000), f32(1.0), V(0x30000), V(0x40000), V(0x50000)]
    assert L.kt_moe_balance_stats(ctypes.byref(cfg), T, *args, V(0x7000000), need - 1,
                                  None) == K.KT_ERR_WORKSPACE
    a2 = list(args)
    a2[2] = f32(float("inf"))
    assert L.kt_moe_balance_stats(ctypes.byref(cfg), T, *a2, V(0x7000000), need,
                                  None) == K.KT_ERR_INVALID_CONFIG
    a2 = list(args)
    a2[0] = None
    assert L.kt_moe_balance_stats(ctypes.byref(cfg), T, *a2, V(0x7000000), need,
                                  None) == K.KT_ERR_NULL
    assert L.kt_moe_balance_stats(ctypes.byref(cfg), T, *args, V(0x7000080), need,
                                  None) == K.KT_ERR_ALIGN
    # scores: x required, workspace of the forward's size
    wneed = K.kt_moe_workspace_size(cfg, T)
    assert L.kt_moe_scores(ctypes.byref(cfg), T, None, V(0x20000), V(0x30000), V(0x7000000),
                           wneed, None) == K.KT_ERR_NULL
    assert L.kt_moe_scores(ctypes.byref(cfg), T, V(0x10000), V(0x20000), V(0x30000),
                           V(0x7000000), wneed - 1, None) == K.KT_ERR_WORKSPACE


def test_graph_create_host_side_errors():
    """kt_moe_graph_create runs the forward's host checks before any CUDA call
    and leaves the output handle NULL on failure."""
    cfg = K.config_for(W.BY_NAME["small_sig_bias"])
    L = K.lib()
    V = ctypes.c_void_p
    T = 300
    need = K.kt_moe_workspace_size(cfg, T)
    good = [V(0x10000 * (i + 1)) for i in range(9)]
    h = V(0x1234)
    rc = L.kt_moe_graph_create(ctypes.byref(cfg), T, *good, V(0x7000000), need - 1, ctypes.byref(h))
    assert rc == K.KT_ERR_WORKSPACE and not h.value
    p = list(good)
    p[0] = None
    h = V(0x1234)
    rc = L.kt_moe_graph_create(ctypes.byref(cfg), T, *p, V(0x7000000), need, ctypes.byref(h))
    assert rc == K.KT_ERR_NULL and not h.value
    assert L.kt_moe_graph_create(ctypes.byref(cfg), T, *good, V(0x7000000), need,
                                 None) == K.KT_ERR_NULL
    assert L.kt_moe_graph_launch(None, None) == K.KT_ERR_NULL
    L.kt_moe_graph_destroy(None)


def test_expert_parallel_host_side_errors():
    """kt_moe_forward_local / _mxfp8, kt_moe_ep_finish and the local pack check
    ranges, pointers and dtypes on the host (fake pointers, never dereferenced)."""
    layer = W.BY_NAME["small_sig_bias"]
    cfg = K.config_for(layer)
    L = K.lib()
    V = ctypes.c_void_p
    T, E = layer.T, layer.n_experts
    need = K.kt_moe_workspace_size(cfg, T)
    ptr = lambda i: V(0x10000 * (i + 1))

    def local(eb, ee, sb, se, ws_bytes=need, y=ptr(7), x=ptr(0)):
        return L.kt_moe_forward_local(ctypes.byref(cfg), T, x, ptr(1), ptr(2), eb, ee, sb, se,
                                      ptr(3), ptr(4), ptr(5), y, None, None, V(0x7000000),
                                      ws_bytes, None)

    for eb, ee, sb, se in ((-1, 4, 0, T), (5, 4, 0, T), (0, E + 1, 0, T), (0, E, -1, T),
                           (0, E, 10, 9), (0, E, 0, T + 1)):
        assert local(eb, ee, sb, se) == K.KT_ERR_INVALID_CONFIG, (eb, ee, sb, se)
    assert local(0, E, 0, T, ws_bytes=need - 1) == K.KT_ERR_WORKSPACE
    assert local(0, E, 0, T, y=None) == K.KT_ERR_NULL
    assert local(0, E, 0, T, x=None) == K.KT_ERR_NULL
    assert local(0, E, 0, T, y=V(0x80008)) == K.KT_ERR_ALIGN
    # y_part is fp32 [T, dim]: overlapping x over that size is rejected
    assert local(0, E, 0, T, y=V(0x10000 + 16)) == K.KT_ERR_INVALID_CONFIG
    # the bf16 entry rejects an MXFP8 config and the MXFP8 entry a bf16 one
    cf8 = K.config_for(W.BY_NAME["small_sig_bias_mxfp8"])
    need8 = K.kt_moe_workspace_size(cf8, 300)
    assert L.kt_moe_forward_local(ctypes.byref(cf8), 300, ptr(0), ptr(1), ptr(2), 0, 4, 0, 300,
                                  ptr(3), ptr(4), ptr(5), ptr(7), None, None, V(0x7000000),
                                  need8, None) == K.KT_ERR_INVALID_CONFIG
    f8 = lambda c, w1q, w3q: L.kt_moe_forward_local_mxfp8(
        ctypes.byref(c), 300, ptr(0), ptr(1), ptr(2), 0, 4, 0, 300, w1q, w3q, ptr(5), ptr(8),
        ptr(9), ptr(7), None, None, V(0x7000000), max(need, need8), None)
    assert f8(cfg, ptr(3), ptr(4)) == K.KT_ERR_INVALID_CONFIG
    assert f8(cf8, ptr(4), ptr(3)) == K.KT_ERR_INVALID_CONFIG     # W3 codes below W1's
    # finish: NULLs, alignment, overlap (in place only for fp32 y)
    fin = lambda c, ys, x, y: L.kt_moe_ep_finish(ctypes.byref(c), T, ys, x, y, None)
    assert fin(cfg, None, ptr(0), ptr(1)) == K.KT_ERR_NULL
    assert fin(cfg, ptr(2), ptr(0), V(0x30008)) == K.KT_ERR_ALIGN
    assert fin(cfg, ptr(2), ptr(0), ptr(2)) == K.KT_ERR_INVALID_CONFIG      # bf16 y in place
    res = K.config_for(W.BY_NAME["small_odd_dims"])                        # with the residual
    assert L.kt_moe_ep_finish(ctypes.byref(res), 77, ptr(2), None, ptr(1), None) == K.KT_ERR_NULL
    # local pack sizes follow the slot count; bad ranges give 0 / an error
    full = K.kt_moe_mxfp8_scale_bytes(cf8, False)
    n_all = 32 + 1
    assert K.kt_moe_mxfp8_scale_bytes_local(cf8, 0, 32, False) == full
    assert K.kt_moe_mxfp8_scale_bytes_local(cf8, 8, 16, False) == full // n_all * 9
    assert K.kt_moe_mxfp8_scale_bytes_local(cf8, 8, 16, True) == \
        K.kt_moe_mxfp8_scale_bytes(cf8, True) // n_all * 9
    assert K.kt_moe_mxfp8_scale_bytes_local(cf8, 16, 8, False) == 0
    assert K.kt_moe_mxfp8_scale_bytes_local(cfg, 0, 8, False) == 0
    assert L.kt_moe_mxfp8_pack_local(ctypes.byref(cf8), 0, 33, *[ptr(i) for i in range(8)],
                                     None) == K.KT_ERR_INVALID_CONFIG


def test_placed_table_host_side_errors():
    """kt_moe_forward_placed validates the slot table on the host: every slot
    used is one of 0 .. n_local - 1, exactly once."""
    layer = W.BY_NAME["small_sig_bias"]          # E = 32
    cfg = K.config_for(layer)
    L = K.lib()
    V = ctypes.c_void_p
    T, E = layer.T, layer.n_experts
    need = K.kt_moe_workspace_size(cfg, T)
    ptr = lambda i: V(0x10000 * (i + 1))

    def placed(tab):
        arr = None if tab is None else (ctypes.c_int32 * E)(*tab)
        return L.kt_moe_forward_placed(ctypes.byref(cfg), T, ptr(0), ptr(1), ptr(2),
                                       None if arr is None else ctypes.cast(arr, V), 0, T,
                                       ptr(3), ptr(4), ptr(5), ptr(7), None, None, V(0x7000000),
                                       need, None)

    base = [-1] * E
    dup = list(base); dup[3] = 0; dup[9] = 0            # slot 0 twice
    gap = list(base); gap[3] = 0; gap[9] = 2            # slots 0 and 2: 1 missing
    low = list(base); low[4] = -2
    high = list(base); high[4] = E
    for tab in (dup, gap, low, high):
        assert placed(tab) == K.KT_ERR_INVALID_CONFIG, tab
    assert placed(None) == K.KT_ERR_NULL


def test_selftest_host_side_errors():
    L = K.lib()
    V = ctypes.c_void_p
    assert L.kt_moe_selftest_timeout(None, 1000, None) == K.KT_ERR_WORKSPACE
    assert L.kt_moe_selftest_timeout(V(0x7000080), 1000, None) == K.KT_ERR_ALIGN
    for bad in (0, -5, 2_000_000_000):
        assert L.kt_moe_selftest_timeout(V(0x7000000), bad, None) == K.KT_ERR_INVALID_CONFIG


def test_strerror_covers_codes():
    for code in range(-9, 1):
        assert K.strerror(code) and K.strerror(code) != "unknown error code"
    assert K.strerror(-99) == "unknown error code"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_reports_cuda_error():
    cfg = K.config_for(W.TINY)
    n = K.kt_moe_workspace_size(cfg, 64)
    buf = torch.empty(n + 256, dtype=torch.uint8)
    ws_ptr = (buf.data_ptr() + 255) // 256 * 256
    x = torch.empty(64, 256)
    y = torch.empty(64, 256)      # its own allocation: must overlap neither x nor the workspace
    # Valid host-side arguments; the first CUDA call fails without a device.
    ptrs = [x.data_ptr()] * 6 + [y.data_ptr()] + [0, 0]
    rc = _call_forward(cfg, 64, ptrs, ws_ptr, n)
    assert rc in (K.KT_ERR_CUDA, K.KT_ERR_UNSUPPORTED)


def test_mxfp4_host_side_errors():
    """MXFP4 configs: dims must be multiples of 128; the packed 4-bit codes need
    32-byte alignment (their tensor maps); the quantize entry checks K, NULLs
    and alignment. Fake pointers, rejected on the host."""
    cfg4 = K.config_for(W.BY_NAME["small_sig_bias_mxfp4"])
    assert cfg4.dtype == K.KT_DTYPE_MXFP4
    assert K.kt_moe_validate(cfg4, 300, True) == K.KT_OK
    fields = {f: getattr(cfg4, f) for f, _ in K.kt_moe_config._fields_}
    assert K.kt_moe_validate(K.make_config(**{**fields, "dim": 448}), 300, True) == \
        K.KT_ERR_INVALID_CONFIG
    assert K.kt_moe_validate(K.make_config(**{**fields, "dtype": 4}), 300, True) == \
        K.KT_ERR_INVALID_CONFIG
    # Scale sizes are the MXFP8 ones (same layout).
    cfg8 = K.config_for(W.BY_NAME["small_sig_bias_mxfp8"])
    for down in (False, True):
        assert K.kt_moe_mxfp8_scale_bytes(cfg4, down) == K.kt_moe_mxfp8_scale_bytes(cfg8, down) > 0
    L = K.lib()
    T = 300
    need = K.kt_moe_workspace_size(cfg4, T)
    V = ctypes.c_void_p
    x, wg, bias, y = 0x100000, 0x200000, 0x300000, 0x400000
    w1q, w3q, w2q, sfu, sfd = 0x1000000, 0x1800000, 0x2000000, 0x2800000, 0x3000000
    ws = 0x7000000

    def fwd(c, a1, a3, a2):
        return L.kt_moe_forward_mxfp8(ctypes.byref(c), T, V(x), V(wg), V(bias), V(a1), V(a3),
                                      V(a2), V(sfu), V(sfd), V(y), None, None, V(ws), need, None,
                                      None)
    assert fwd(cfg4, w1q + 16, w3q + 16, w2q) == K.KT_ERR_ALIGN     # 16 but not 32 bytes
    assert fwd(cfg4, w1q, w3q + 16, w2q) == K.KT_ERR_ALIGN
    assert fwd(cfg4, w1q, w3q, w2q + 16) == K.KT_ERR_ALIGN
    assert fwd(cfg4, w3q, w1q, w2q) == K.KT_ERR_INVALID_CONFIG      # W3's codes below W1's
    # The same offsets pass the 8-bit checks (16-byte alignment suffices there);
    # without a GPU the call then fails at the first CUDA call instead.
    if not torch.cuda.is_available():
        assert fwd(cfg8, w1q + 16, w3q + 16, w2q) in (K.KT_ERR_CUDA, K.KT_ERR_UNSUPPORTED)
    q = L.kt_moe_mxfp4_quantize
    assert q(4, 48, V(x), V(w1q), V(sfu), None) == K.KT_ERR_INVALID_CONFIG
    assert q(4, 64, None, V(w1q), V(sfu), None) == K.KT_ERR_NULL
    assert q(4, 64, V(x + 8), V(w1q), V(sfu), None) == K.KT_ERR_ALIGN
