"""bench.py's host-side arithmetic and inputs (CPU only).

The algorithmic FLOPs and bytes behind every roofline line, against their
closed forms for a layer small enough to count by hand; the DRAM-traffic table
and the measured peaks the roofline reads; the flags of the multi-GPU and
expert-parallel runs.
"""
from __future__ import annotations

import os
import numpy as np
import pytest

import bench
from mixture_experts_layer_34_b200 import workloads as W


def test_algorithmic_counts_match_closed_forms():
    layer = W.BY_NAME["small_sig_bias"]          # T 300, d 512, E 32, k 4, S 1, I 256, bf16
    T, d, E, k, S, I = 300, 512, 32, 4, 1, 256
    idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))     # every token -> experts 0..3
    w = bench.algorithmic(layer, idx)
    R = T * (k + S)
    assert w["rows"] == R
    assert w["active_experts"] == k + S                      # 4 routed hit + 1 shared
    assert w["flops_up"] == 4 * d * I * R
    assert w["flops_down"] == 2 * d * I * R
    assert w["flops_layer"] == W.flops_per_token(layer) * T
    assert W.flops_per_token(layer) == 6 * d * I * (k + S) + 2 * d * E
    # bf16: weights 2 B per element; W_gate, x and y once
    assert w["bytes_layer"] == (k + S) * 3 * d * I * 2 + E * d * 2 + 2 * T * d * 2
    assert w["bytes_up"] == (k + S) * 2 * d * I * 2 + R * d * 2 + R * I * 2


def test_algorithmic_mxfp8_weight_bytes():
    layer = W.BY_NAME["small_sig_bias_mxfp8"]
    idx = np.tile(np.arange(4, dtype=np.int32), (layer.T, 1))
    w = bench.algorithmic(layer, idx)
    # one code byte per weight plus one scale byte per 32
    per_expert = 3 * layer.dim * layer.inter * (1 + 1 / 32)
    tok = layer.n_experts * layer.dim * 2 + 2 * layer.T * layer.dim * 2
    assert w["bytes_layer"] == pytest.approx(5 * per_expert + tok)


def test_traffic_table_is_read_per_kernel_and_workload():
    assert bench.traffic("up", "v3_prefill_T8192_zipf") > 1.5e10
    assert bench.traffic("down", "v3_decode_T8") > 1e9
    assert bench.traffic("up", "no_such_workload") is None


def test_peaks_come_from_the_measured_file():
    p = bench.load_peaks()
    assert p["source"] in ("measured", "fallback")
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    assert p["bf16_tflops_sustained"] <= p["bf16_tflops"]


def test_flags():
    a = bench.parse_args([])
    assert (a.gpus, a.parallel, a.ep_placement, a.ep_ranks) == (1, "dp", "balanced", 8)
    a = bench.parse_args(["--gpus", "4", "--parallel", "ep", "--ep-placement", "contiguous"])
    assert (a.gpus, a.parallel, a.ep_placement) == (4, "ep", "contiguous")
    with pytest.raises(SystemExit):
        bench.parse_args(["--parallel", "tp"])


def test_dump_arrays_round_trip_bit_for_bit():
    """--dump writes bf16 as its 16-bit patterns; reading back gives the same bits."""
    import torch
    g = torch.Generator().manual_seed(3)
    for t in (torch.randn(5, 7, generator=g).to(torch.bfloat16), torch.randn(4, 3, generator=g),
              torch.randint(-5, 9, (6, 2), generator=g, dtype=torch.int32)):
        a = bench._np_of(t)
        tag = "bf16" if t.dtype == torch.bfloat16 else str(t.dtype)
        back = bench._tensor_of(a, tag, "cpu")
        assert back.dtype == t.dtype and torch.equal(back, t)
    special = torch.tensor([float("inf"), -0.0, 1e-40, 3.0], dtype=torch.bfloat16)
    assert bench._np_of(special).tolist() == [0x7F80, 0x8000, special[2].view(torch.int16).item(),
                                              0x4040]


def test_dump_and_replay_flags():
    a = bench.parse_args(["--dump", "/tmp/d"])
    assert a.dump == "/tmp/d" and a.replay is None
    assert bench.parse_args(["--replay", "/tmp/d/x"]).replay == "/tmp/d/x"


def test_algorithmic_mxfp4_weight_bytes():
    layer = W.BY_NAME["small_sig_bias_mxfp4"]
    idx = np.tile(np.arange(4, dtype=np.int32), (layer.T, 1))
    w = bench.algorithmic(layer, idx)
    # half a byte per weight (two E2M1 codes per byte) plus one scale byte per 32
    per_expert = 3 * layer.dim * layer.inter * (0.5 + 1 / 32)
    tok = layer.n_experts * layer.dim * 2 + 2 * layer.T * layer.dim * 2
    assert w["bytes_layer"] == pytest.approx(5 * per_expert + tok)
    assert bench.parse_args(["--no-mxfp4"]).no_mxfp4


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """--impl reference on rank 0: one JSON line with the contract's keys, the
    oracle timed on a sample of the workload (here a small layer, on the CPU)."""
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    a = bench.parse_args(["--impl", "reference", "--workload", "small_sig_bias", "--steps", "1",
                          "--warmup", "3"])
    bench.run_reference(a)
    lines = [x for x in capsys.readouterr().out.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["config"]["workload"] == "small_sig_bias"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_clock_scaled_peak():
    assert bench.clock_scaled_peak(1666.8, 1965.0, 1965.0)[0] == 1666.8
    assert bench.clock_scaled_peak(1666.8, 1900.0, 1965.0)[0] == 1666.8     # within 5%
    p, rule = bench.clock_scaled_peak(1666.8, 1335.0, 1965.0)
    assert p == pytest.approx(1666.8 * 1335 / 1965) and "1335" in rule
    assert bench.clock_scaled_peak(100.0, None, None)[0] == 100.0


def test_smi_timestamps_parse_to_host_time():
    import datetime
    t = bench._smi_time("2026/12/02 16:43:10.250")
    assert t == pytest.approx(datetime.datetime(2026, 12, 2, 16, 43, 10, 250000).timestamp())
    assert bench._smi_time("[N/A]") is None


def test_extra_workloads_flag():
    assert bench.extra_workloads(bench.parse_args([])) == ["v2lite_T512", "v2_T4096"]
    assert bench.extra_workloads(bench.parse_args(["--workload", "small_sig_bias"])) == []
    assert bench.extra_workloads(bench.parse_args(["--extra-workloads", "none"])) == []
    assert bench.extra_workloads(bench.parse_args(["--extra-workloads", "v2_T4096"])) == \
        ["v2_T4096"]


def test_cpu_leg_reports_routing_and_output_agreement():
    """The CPU baseline leg's checks on a tiny layer, fed a 'GPU run' made from
    the oracle itself with one token's routing changed and one output element
    moved: exactly that token differs, and the moved element sets max|dy|."""
    import torch
    import oracle.oracle as O
    layer = W.TINY
    inp = W.make_layer(layer, "cpu")
    kf = layer.kernel_fields()
    g = O.gate(kf, inp["x"], inp["w_gate"], inp["bias"].numpy())
    n = layer.n_experts + layer.n_shared
    y = O.forward(kf, inp["x"], g["idx"], g["w"], [inp["w1"][e] for e in range(n)],
                  [inp["w3"][e] for e in range(n)], [inp["w2"][e] for e in range(n)],
                  range(layer.T), True)
    idx = g["idx"].copy()
    idx[5] = idx[5][::-1]                       # token 5 routed differently
    y32 = torch.tensor(y, dtype=torch.float32)
    rms = float(np.sqrt(np.mean(y ** 2)))
    y32[7, 3] += 0.01 * rms
    res = {"idx": idx, "y32": y32, "y16": y32.to(torch.bfloat16)}
    out = bench.cpu_baseline_leg(layer, inp, res, target_s=0.1, full=True)
    r = out["routing"]
    assert r["tokens"] == layer.T and r["differ_from_oracle"] == 1
    near5 = g["kth_margin"][5] <= 1e-5 or g["grp_margin"][5] <= 1e-5
    assert r["differ_away_from_near_ties"] == (0 if near5 else 1)
    p = out["parity"]
    assert p["tokens"] == layer.T - 1
    rms_keep = float(np.sqrt(np.mean(np.delete(y, 5, axis=0) ** 2)))
    assert p["max_abs_dy_over_rms_fp32"] == pytest.approx(0.01 * rms / rms_keep, rel=1e-3)
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["loop_tokens"] == layer.T and cb["value"] > 0


def test_coverage_tokens_reach_every_chunk():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from parity import coverage_tokens
    rng = np.random.default_rng(0)
    T, E, k = 2000, 16, 2
    # expert 0 in every token, expert 1 in 600, the rest random
    idx = np.stack([np.zeros(T, np.int32), rng.integers(2, E, T).astype(np.int32)], 1)
    idx[:600, 1] = 1
    toks = coverage_tokens(idx, E, 1, 256, total=100, n_heavy=2, seed=3)
    assert len(toks) == 100 and len(set(toks)) == 100
    for e in (0, 1):
        mine = np.where((idx == e).any(1))[0]
        for c0 in range(0, len(mine), 256):
            assert set(mine[c0:c0 + 256]) & set(toks), (e, c0)
        assert mine[-1] in toks


PEAKS = {"bf16_tflops": 1666.8, "bf16_tflops_sustained": 1391.0, "hbm_gbs": 6551.0,
         "source": "measured"}


def test_tensor_roofline_takes_the_clock_of_its_own_region():
    """achieved = FLOPs / event time; the peak is the burst figure scaled to the
    median clock of the kernel's region (the run's median when the region has no
    samples); the fraction can be recomputed from the entry alone."""
    clk = {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "regions": {"pre": {"sm_mhz": 1300.0}}}
    e = bench.tensor_roofline("up", 4.33e12, 4.5, PEAKS, clk, "pre")
    assert e["achieved"] == pytest.approx(4.33e12 / 4.5e-3 / 1e12, abs=0.05)
    assert e["peak"] == pytest.approx(1666.8 * 1300 / 1965, abs=0.05)
    assert e["peak_clock_mhz"] == 1300.0 and e["sm_max_mhz"] == 1965.0
    assert e["frac"] == pytest.approx(e["achieved"] / e["peak"], abs=1e-3)
    assert e["frac_of_sustained"] == pytest.approx(e["achieved"] / 1391.0, abs=1e-3)
    # no samples in the region: the run's median (within 5% of max: burst)
    e = bench.tensor_roofline("up", 4.33e12, 4.5, PEAKS, clk, "other")
    assert e["peak"] == pytest.approx(1666.8) and e["peak_clock_mhz"] == 1900.0
    # another dtype: its nominal ratio times the measured bf16 figure
    e = bench.tensor_roofline("up", 4.33e12, 4.5, PEAKS, clk, "other", mult=2.0)
    assert e["peak"] == pytest.approx(2 * 1666.8) and "x 2" in e["peak_source"]


def test_hbm_roofline_and_layer_fractions():
    e = bench.hbm_roofline("up", 2.64e9, 0.4, PEAKS, traffic_bytes=2645930837)
    assert e["achieved"] == pytest.approx(6600.0) and e["frac"] == pytest.approx(6600 / 6551, abs=1e-4)
    assert e["traffic"] == 2645930837 and e["unit"] == "GB/s"
    layer = W.BY_NAME["v3_prefill_T8192_zipf"]
    res = {"ms": 16.0, "work": {"flops_layer": 6.524e12, "bytes_layer": 22.6e9}}
    f = bench.layer_fracs(layer, res, 2, PEAKS, 1300.0, 1965.0)    # 8 ms per step
    assert f["layer_tflops"] == pytest.approx(6.524e12 / 8e-3 / 1e12, abs=0.05)
    assert f["layer_hbm_frac"] == pytest.approx(22.6e9 / 8e-3 / 1e9 / 6551, abs=1e-4)
    assert f["layer_tensor_frac"] == pytest.approx(
        6.524e12 / 8e-3 / 1e12 / (1666.8 * 1300 / 1965), abs=1e-4)
    mx = W.BY_NAME["v3_prefill_T8192_zipf_mxfp8"]
    g = bench.layer_fracs(mx, res, 2, PEAKS, 1965.0, 1965.0)
    assert g["layer_tensor_frac"] == pytest.approx(6.524e12 / 8e-3 / 1e12 / (2 * 1666.8), abs=1e-4)


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_sampler_assigns_samples_to_regions(tmp_path, monkeypatch):
    """stop() on a recorded nvidia-smi log: the median clock of the loaded
    samples, the throttle reasons seen, and per marked region the median of the
    samples stamped inside it (widened by one sampling period)."""
    import datetime
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    t0 = datetime.datetime(2026, 12, 2, 16, 0, 0)
    rows = []
    for i, (mhz, cap) in enumerate([(1965, "Not Active")] * 4 + [(1300, "Active")] * 5
                                   + [(1965, "Not Active")] * 3):
        ts = (t0 + datetime.timedelta(milliseconds=50 * i)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        rows.append(f"0, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, {cap}, {ts}")
    path = tmp_path / "clk.csv"
    path.write_text("\n".join(rows) + "\n")
    cs = bench.ClockSampler(0)
    cs.path, cs.proc = str(path), _DoneProc()
    base = t0.timestamp()
    cs.windows = {"capped": [base + 0.25, base + 0.40], "open": [base + 0.5, None]}
    out = cs.stop()
    assert out["sm_max_mhz"] == 1965.0 and out["samples"] == 12
    assert out["reasons"] == ["sw_power_cap"]
    assert out["sm_mhz"] == 1965.0              # 7 of 12 loaded samples at full clock
    reg = out["regions"]
    assert set(reg) == {"capped"}               # an unclosed window is dropped
    # [0.25, 0.40] s widened to [0.20, 0.45]: the five capped samples and one at full clock
    assert reg["capped"]["sm_mhz"] == 1300.0 and reg["capped"]["samples"] == 6
    assert not path.exists()
