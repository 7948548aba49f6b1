"""bench.py --dump / --replay on the GPU: a dumped step reruns bit for bit.

A short bench run on a small layer (bf16, MXFP8 and MXFP4 forms) dumps each
step's inputs and outputs; --replay redraws the expert weights from the seed, checks
the weight probe, reruns the forward on the dumped tokens and must reproduce
the routing and y exactly (the forward is deterministic: fixed sum orders, no
atomics in the arithmetic).
"""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def _run(args, timeout=900):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=timeout)
    return r


def test_dump_then_replay_is_bit_exact(tmp_path):
    d = str(tmp_path / "dump")
    r = _run(["--workload", "small_sig_bias", "--decode-workload", "none", "--ep-ranks", "0",
              "--no-cpu-baseline", "--steps", "2", "--warmup", "3", "--e2e-steps", "2",
              "--dump", d])
    assert r.returncode == 0, r.stderr[-4000:]
    # The run's one JSON line carries the contract's keys.
    line = json.loads([x for x in r.stdout.splitlines() if x.startswith("{")][-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks", "layer_hbm_frac", "mxfp8", "mxfp4"):
        assert key in line, key
    assert line["value"] > 0 and line["config"]["workload"] == "small_sig_bias"
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in line["roofline"], key
    assert line["e2e"]["h2d_bytes_per_step"] == 300 * 512 * 2
    steps = sorted(os.listdir(d))
    assert steps == ["small_sig_bias_mxfp4_rank0", "small_sig_bias_mxfp8_rank0",
                     "small_sig_bias_rank0"], steps
    for s in steps:
        files = set(os.listdir(os.path.join(d, s)))
        assert {"x.npy", "w_gate.npy", "bias.npy", "idx.npy", "w.npy", "y.npy", "w_probe.npy",
                "meta.json"} <= files, files
        meta = json.load(open(os.path.join(d, s, "meta.json")))
        assert meta["check"] == "ok" and meta["T"] == 300
        rr = _run(["--replay", os.path.join(d, s)])
        assert rr.returncode == 0, rr.stdout + rr.stderr[-4000:]
        out = json.loads(rr.stdout.strip().splitlines()[-1])
        assert out["match"] and out["weights_redrawn_identically"], out
        assert all(out["identical"].values()), out
