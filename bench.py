#!/usr/bin/env python
"""Throughput of the DeepSeekMoE layer forward on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one kt_moe_forward of the V3-shaped prefill layer (T = 8192 tokens,
Zipf(1.1) expert load, bf16) with inputs resident in HBM; the same run also
measures the V3-shaped decode step (T = 8) and prints it under "decode". With N
GPUs every rank runs its own replica on its own tokens (data parallel over
tokens, no collective on the data path): weak scaling, timed on the device as
the max over ranks.

Rank 0 prints one JSON line. `value` is tokens/s of the whole job, timed over
the forwards alone (stage times come from a separate pass of the same steps with
events at the stage boundaries: `stage_ms`, `staged_ms_per_step`); `e2e` is the
same metric with host buffers (pinned x copied in and y copied out every step,
serial with the compute), `e2e_pipelined` the same copies overlapped with the
neighbouring steps' compute on two copy streams; `roofline` is the dominant
kernel (the gate/up expert GEMM) and `roofline_down` the down GEMM, each against
the measured bf16 burst peak matched to the median SM clock of the timed region
(the burst figure when that median is within 5% of the maximum clock, else
scaled by median / maximum; `peak_clock_mhz` is the clock used); `routing` is
the expert-load summary and, from the CPU oracle's gate over all T tokens, how
many tokens the GPU routed differently (and how many of those away from the
oracle's near ties) and the oracle's own near-tie count; `parity` compares the
outputs of the CPU leg's tokens with the oracle's (fp32 form and bf16 output);
`cpu_baseline` is the CPU oracle timed on this host's cores (its gate on all T
tokens plus its expert loop on a sample, extrapolated to T; the decode layer in
full); "v2lite_T512" and "v2_T4096" time the V2-shaped layers the same way;
"mxfp8" and "mxfp4" repeat prefill and decode with MXFP8 and MXFP4 expert
weights.
`--impl reference` times the oracle alone (rank 0 only) in the same JSON form.

`--dump DIR` saves each timed step's inputs and outputs as .npy files under
DIR/<workload>_rank<r>/, also when a device error stops the run (before it
raises): x, w_gate, bias, the routing (idx, w), y, a probe of the expert
weights and meta.json. The expert weights themselves are not written: they are
redrawn from the workload's seed. `python bench.py --replay DIR/<dumped step>`
redraws them, checks the probe, reruns the forward on the dumped tokens and
compares the routing and y bit for bit.

"expert_parallel" (N = 1) times each rank's local step of the expert-parallel
layer over --ep-ranks ranks (its experts, all tokens through the gate, its
share of the shared experts' tokens) one rank after another on this GPU, for
contiguous expert ranges and for a placement balanced on another batch's load,
plus the finish kernel; the all-reduce (or, for a token-sharded output, the
reduce-scatter) between them is projected, not measured. With N > 1,
`--parallel ep` runs that layer for real over NCCL (the same T tokens on every
rank, strong scaling; --ep-placement, --ep-output).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_34_b200 import workloads as W  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
LAUNCHES_PER_FORWARD = 7   # logits, select, scan, scatter, up GEMM, down GEMM, combine


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=W.V3_PREFILL.name)
    ap.add_argument("--decode-workload", default=W.V3_DECODE.name, help="'none' to skip")
    ap.add_argument("--extra-workloads", default="auto",
                    help="comma-separated layers also timed (no graph, no CPU leg); 'auto' = "
                         "the V2-Lite and V2 layers when --workload is the V3 prefill; 'none'")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target wall time of the CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mxfp8", action="store_true", help="skip the MXFP8-weight lines")
    ap.add_argument("--no-mxfp4", action="store_true", help="skip the MXFP4-weight lines")
    ap.add_argument("--ep-ranks", type=int, default=8,
                    help="N=1: time each rank's local step of the expert-parallel layer over "
                         "this many ranks, one after another (0 to skip)")
    ap.add_argument("--parallel", choices=("dp", "ep"), default="dp",
                    help="N>1: dp = replicas on their own tokens (default); ep = experts "
                         "split over the ranks, one all-reduce per step")
    ap.add_argument("--ep-placement", choices=("contiguous", "balanced"), default="balanced",
                    help="--parallel ep: experts in contiguous ranges, or placed by the load "
                         "of another seeded batch")
    ap.add_argument("--ep-output", choices=("full", "sharded"), default="full",
                    help="--parallel ep: every rank gets all T output rows (all-reduce), or "
                         "its token share (reduce-scatter; T divisible by N)")
    ap.add_argument("--dump", default=None,
                    help="save each step's inputs and outputs (.npy) under this directory")
    ap.add_argument("--replay", default=None,
                    help="rerun a step saved by --dump and compare bit for bit, then exit")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


# ---------------------------------------------------------------------------
# Process group (only for barriers and the max-over-ranks of device times)
# ---------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=300))


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_tokens_seed(layer, rank: int) -> int:
    """Each rank routes its own tokens; weights and bias are the same everywhere."""
    return layer.seed * 1000 + rank


# ---------------------------------------------------------------------------
# Peaks, clocks
# ---------------------------------------------------------------------------
def traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of a kernel on a workload, from the
    ncu counters summarised in profiles/dram_traffic.txt, or None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        f = line.split()
        if len(f) == 3 and f[0] == kernel and f[1] == workload:
            return float(f[2])
    return None


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS)


class ClockSampler:
    """nvidia-smi clock/throttle samples every 50 ms while the timed work runs.
    mark(name) / unmark(name) bracket a timed region on the host clock; stop()
    gives the run's summary and the median SM clock inside each region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
             "timestamp")
    PERIOD_MS = 50

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.windows = {}

    def mark(self, name: str):
        self.windows[name] = [time.time(), None]

    def unmark(self, name: str):
        if name in self.windows:
            self.windows[name][1] = time.time()

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        power = [float(r[3]) if r[3].replace(".", "").isdigit() else 0.0 for r in rows]
        loaded = [s for s, p in zip(sm, power) if p > 0.3 * max(power)] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        out = {"sm_mhz": statistics.median(loaded), "sm_max_mhz": float(rows[0][2]),
               "reasons": reasons, "samples": len(rows)}
        stamps = [_smi_time(r[9]) if len(r) > 9 else None for r in rows]
        regions = {}
        for name, (t0, t1) in self.windows.items():
            if t1 is None:
                continue
            # samples taken inside the region, widened by one sampling period
            pad = self.PERIOD_MS / 1e3
            inside = [f for f, ts in zip(sm, stamps) if ts is not None and t0 - pad <= ts <= t1 + pad]
            regions[name] = {"sm_mhz": statistics.median(inside) if inside else None,
                             "samples": len(inside), "seconds": round(t1 - t0, 3)}
        if regions:
            out["regions"] = regions
        return out


def _smi_time(field: str):
    """nvidia-smi's timestamp ("2026/12/02 16:43:10.123") as host epoch seconds."""
    try:
        return datetime.datetime.strptime(field.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
    except ValueError:
        return None


def clock_scaled_peak(burst: float, sm_mhz, sm_max_mhz) -> tuple[float, str]:
    """The tensor peak that matches the SM clock a kernel ran at: the measured
    burst figure when the median clock of its timed region is within 5% of the
    maximum, else the burst figure scaled by median / maximum."""
    if not sm_mhz or not sm_max_mhz or sm_mhz >= 0.95 * sm_max_mhz:
        return burst, "burst (median SM clock within 5% of max)"
    return burst * sm_mhz / sm_max_mhz, f"burst x {sm_mhz:.0f} / {sm_max_mhz:.0f} MHz"


# ---------------------------------------------------------------------------
# Algorithmic work per launch: the bytes the method must move and the FLOPs it
# must do (activated experts only; no padding, no implementation buffers)
# ---------------------------------------------------------------------------
def algorithmic(layer, idx: np.ndarray) -> dict:
    T, d, I, k, S, E = layer.T, layer.dim, layer.inter, layer.topk, layer.n_shared, layer.n_experts
    es = 4 if layer.dtype == "f32" else 2
    # expert-weight bytes per element (MXFP8: one byte plus one scale byte per 32;
    # MXFP4: half a byte plus one scale byte per 32)
    ew = {"mxfp8": 1 + 1 / 32, "mxfp4": 0.5 + 1 / 32}.get(layer.dtype, es)
    R = T * (k + S)
    active = int((np.bincount(idx.ravel(), minlength=E) > 0).sum()) + S
    return {
        "rows": R,
        "active_experts": active,
        "flops_layer": W.flops_per_token(layer) * T,
        "flops_up": 4 * d * I * R,
        "flops_down": 2 * d * I * R,
        # bytes the method must move: activated experts' weights, W_gate, x, y
        "bytes_layer": active * 3 * d * I * ew + E * d * es + 2 * T * d * es,
        # gate/up GEMM: W1, W3 of active experts, the token rows in, hidden rows out
        "bytes_up": active * 2 * d * I * ew + R * d * es + R * I * es,
    }


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------
# All-reduce bus bandwidth of 8 B200s over NVSwitch at 1 GiB messages, measured
# on this pool (NCCL); used only to project the expert-parallel step's
# collective from one GPU.
ALLREDUCE_BUS_GBS = 725.0


def load_stats(layer, idx: np.ndarray) -> dict:
    """Expert-load summary of the routing the timed forward produced."""
    load = np.bincount(idx.ravel(), minlength=layer.n_experts)
    return {"load_max": int(load.max()), "load_mean": round(float(load.mean()), 2),
            "max_over_mean": round(float(load.max() / load.mean()), 2),
            "active_experts": int((load > 0).sum()), "zero_load_experts": int((load == 0).sum()),
            "load_top8": np.sort(load)[::-1][:8].tolist()}


def time_ep_ranks(layer, inp, dev, ranks, steps, warmup):
    """The expert-parallel layer's per-rank local step (the gate on all tokens,
    the rank's experts, its share of the shared experts' tokens), each rank
    timed on this GPU in turn, for two placements of the routed experts:
    contiguous ranges (kt_moe_forward_local) and a placement balanced on the
    expert load of another batch of the same workload (kt_moe_forward_placed);
    and the finish kernel."""
    from mixture_experts_layer_34_b200 import ep
    from mixture_experts_layer_34_b200 import ktmoe as K
    cfg = K.config_for(layer)
    T, E, S = layer.T, layer.n_experts, layer.n_shared
    ws = K.alloc_workspace(cfg, T, dev)
    part = torch.empty((T, layer.dim), dtype=torch.float32, device=dev)
    y = torch.empty((T, layer.dim), dtype=inp["x"].dtype, device=dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(run):
        for _ in range(warmup):
            run()
        torch.cuda.synchronize()
        t0.record()
        for _ in range(steps):
            run()
        t1.record()
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / steps

    load2 = expected_load(layer, inp, dev)
    placements = {"contiguous": ep.contiguous_placement(E, ranks),
                  "balanced": ep.balanced_placement(load2, ranks)}
    out = {}
    for name, placement in placements.items():
        rank_ms = []
        for r in range(ranks):
            sb, se = ep.token_range(T, ranks, r)
            experts = placement[r]
            w1, w3, w2 = (ep.local_stack_of(inp[k], E, S, experts) for k in ("w1", "w3", "w2"))
            if name == "contiguous":
                eb, ee = experts[0], experts[-1] + 1
                run = lambda: K.kt_moe_forward_local(cfg, T, inp["x"], inp["w_gate"], inp["bias"],
                                                     eb, ee, sb, se, w1, w3, w2, part, None, None,
                                                     ws)
            else:
                tab = ep.slot_table(experts, E)
                run = lambda: K.kt_moe_forward_placed(cfg, T, inp["x"], inp["w_gate"],
                                                      inp["bias"], tab, sb, se, w1, w3, w2, part,
                                                      None, None, ws)
            rank_ms.append(timed(run))
            del w1, w3, w2
        out[name] = rank_ms
    finish_ms = timed(lambda: K.kt_moe_ep_finish(cfg, T, part, inp["x"], y))
    rc = K.kt_moe_check(ws)
    if rc != K.KT_OK:
        raise RuntimeError(f"device error in the expert-parallel steps: {K.strerror(rc)}")
    msg = T * layer.dim * 4
    ar_ms = 2 * (ranks - 1) / ranks * msg / (ALLREDUCE_BUS_GBS * 1e9) * 1e3
    rs_ms = ar_ms / 2          # a reduce-scatter moves half an all-reduce's bytes
    torch.cuda.empty_cache()
    res = {"ranks": ranks, "workload": layer.name, "finish_ms": round(finish_ms, 4),
           "allreduce_bytes": msg, "allreduce_ms_projected": round(ar_ms, 4),
           "reduce_scatter_ms_projected": round(rs_ms, 4), "unit": "tokens/s"}
    for name, rank_ms in out.items():
        step_ms = max(rank_ms) + ar_ms + finish_ms
        # token-sharded output: reduce-scatter, and the finish on 1/ranks of the rows
        shard_ms = max(rank_ms) + rs_ms + finish_ms / ranks
        res[name] = {"rank_local_ms": [round(v, 4) for v in rank_ms],
                     "max_rank_local_ms": round(max(rank_ms), 4),
                     "step_ms_projected": round(step_ms, 4),
                     "value_projected": round(T / (step_ms / 1e3), 1),
                     "sharded_step_ms_projected": round(shard_ms, 4),
                     "sharded_value_projected": round(T / (shard_ms / 1e3), 1)}
    res["note"] = ("local steps and finish measured here, one rank after another on this GPU; "
                   "the fp32 all-reduce is projected at the measured 8-GPU NCCL bus bandwidth "
                   f"({ALLREDUCE_BUS_GBS:.0f} GB/s), not measured (one GPU); the balanced "
                   "placement is computed from the expert load of another seeded batch")
    return res


def expected_load(layer, inp, dev) -> np.ndarray:
    """Per-expert token counts of another seeded batch of the same workload (the
    tokens of rank 1 of a data-parallel run), routed by kt_moe_gate."""
    from mixture_experts_layer_34_b200 import ktmoe as K
    cfg = K.config_for(layer)
    T = layer.T
    g = torch.Generator(device="cpu").manual_seed(rank_tokens_seed(layer, 1))
    x2 = torch.randn(inp["x"].shape, generator=g).to(inp["x"].dtype).to(dev)
    ws = K.alloc_workspace(cfg, T, dev)
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device=dev)
    w = torch.empty((T, layer.topk), dtype=torch.float32, device=dev)
    K.kt_moe_gate(cfg, T, x2, inp["w_gate"], inp["bias"], None, idx, w, ws)
    return np.bincount(idx.cpu().numpy().ravel(), minlength=layer.n_experts)


def time_ep_layer(layer, dev, rank, world, steps, warmup, placement_kind="balanced",
                  output="full"):
    """N > 1, --parallel ep: the expert-parallel layer over the process group
    (NCCL all-reduce of the fp32 partials); the same T tokens on every rank.
    Every rank computes the same placement from the same seeded batch."""
    from mixture_experts_layer_34_b200 import ep
    from mixture_experts_layer_34_b200 import ktmoe as K
    inp = W.make_layer(layer, dev)
    cfg = K.config_for(layer)
    placement = None
    if placement_kind == "balanced":
        placement = ep.balanced_placement(expected_load(layer, inp, dev), world)
    m = ep.ExpertParallelMoE(cfg, inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                             rank, world, placement=placement)
    inp["w1"] = inp["w3"] = inp["w2"] = None
    torch.cuda.empty_cache()
    sb, se = m.shared_range(layer.T)
    rows = layer.T if output == "full" else se - sb
    y = torch.empty((rows, layer.dim), dtype=inp["x"].dtype, device=dev)
    step = (lambda: m.forward(inp["x"], y)) if output == "full" else \
        (lambda: m.forward_shard(inp["x"], y))
    for _ in range(warmup):
        step()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    rc = K.kt_moe_check(m.buffers(layer.T, dev)[0])
    if rc != K.KT_OK:
        raise RuntimeError(f"device error in the expert-parallel steps: {K.strerror(rc)}")
    return max_over_ranks(t0.elapsed_time(t1), world, dev)
def time_layer(layer, dev, rank, world, steps, warmup, e2e_steps, graph=False, dump=None,
               clocks=None, keep_y32=False):
    """Time one layer: the plain forward (the headline loop: nothing but the
    forwards between its two events), then a separate pass of the same steps
    with stage events (stage_ms), optionally a CUDA-graph replay, and the
    end-to-end loops with host buffers. keep_y32: also run one forward with an
    fp32 output (the sum before its bf16 rounding) and return it with the bf16
    output of the timed loop, for the comparison with the oracle."""
    from mixture_experts_layer_34_b200 import ktmoe as K
    inp = W.make_layer(layer, dev)
    if rank > 0:
        g = torch.Generator(device="cpu").manual_seed(rank_tokens_seed(layer, rank))
        inp["x"] = torch.randn(inp["x"].shape, generator=g).to(inp["x"].dtype).to(dev)
    probe = weight_probe(layer, inp) if dump else None
    cfg = K.config_for(layer)
    T = layer.T
    ws = K.alloc_workspace(cfg, T, dev)
    y = torch.empty((T, layer.dim), dtype=inp["x"].dtype, device=dev)
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device=dev)
    w = torch.empty((T, layer.topk), dtype=torch.float32, device=dev)
    fp8 = layer.dtype in ("mxfp8", "mxfp4")   # block-scaled expert weights
    if fp8:
        # MXFP8 form: pack the seeded bf16 expert weights once, then drop them.
        q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
        torch.cuda.synchronize()
        inp["w1"] = inp["w3"] = inp["w2"] = None
        torch.cuda.empty_cache()
    args = (cfg, T, inp["x"], inp["w_gate"], inp["bias"], inp["w1"], inp["w3"], inp["w2"], y, idx, w, ws)

    def fwd(x, events=None, y_out=None, c=None):
        yo = y if y_out is None else y_out
        c = cfg if c is None else c
        if fp8:
            K.kt_moe_forward_mxfp8(c, T, x, inp["w_gate"], inp["bias"], q["w1q"], q["w3q"],
                                   q["w2q"], q["sf_up"], q["sf_down"], yo, idx, w, ws,
                                   stage_events=events)
        elif events is not None:
            K.kt_moe_forward_profiled(c, T, x, *args[3:8], yo, *args[9:], events)
        else:
            K.kt_moe_forward(c, T, x, *args[3:8], yo, *args[9:])

    def save(rc):
        if dump:
            dump_step(os.path.join(dump, f"{layer.name}_rank{rank}"), layer, inp, idx, w, y,
                      probe, rc, rank)

    for _ in range(warmup):
        fwd(inp["x"])
    rc = K.kt_moe_check(ws)
    if rc != K.KT_OK:
        save(rc)
        raise RuntimeError(f"device error after warm-up: {K.strerror(rc)}")

    # The timed loop: the forwards alone, back to back on the launch stream.
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.mark(layer.name)
    t0.record()
    for s in range(steps):
        fwd(inp["x"])
    t1.record()
    torch.cuda.synchronize()
    if clocks:
        clocks.unmark(layer.name)
    barrier(world)
    ms = t0.elapsed_time(t1)
    rc = K.kt_moe_check(ws)
    save(rc)
    if rc != K.KT_OK:
        raise RuntimeError(f"device error in the timed region: {K.strerror(rc)}")
    ms_max = max_over_ranks(ms, world, dev)

    # Stage times: the same number of steps again, right after, with events
    # recorded on the launch stream at the stage boundaries (created and
    # recorded once beforehand). Its total is reported beside the plain loop's.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(K.KT_STAGE_EVENTS)]
          for _ in range(steps)]
    for row in ev:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark(layer.name + "/stages")
    for s in range(steps):
        fwd(inp["x"], ev[s])
    torch.cuda.synchronize()
    if clocks:
        clocks.unmark(layer.name + "/stages")
    rc = K.kt_moe_check(ws)
    if rc != K.KT_OK:
        raise RuntimeError(f"device error in the stage pass: {K.strerror(rc)}")
    stage_ms = {name: statistics.fmean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps))
                for i, name in enumerate(K.STAGES)}
    staged_ms = statistics.fmean(ev[s][0].elapsed_time(ev[s][-1]) for s in range(steps))

    # fp32-output forward (outside every timed region) for the oracle comparison.
    y32 = y16 = None
    if keep_y32:
        y16 = y.clone()
        y32 = torch.empty(y.shape, dtype=torch.float32, device=dev)
        fwd(inp["x"], y_out=y32, c=K.config_for(layer, y_fp32=True))
        rc = K.kt_moe_check(ws)
        if rc != K.KT_OK:
            raise RuntimeError(f"device error in the fp32-output forward: {K.strerror(rc)}")

    # The same forward replayed as one CUDA graph (kt_moe_graph_*), same buffers.
    graph_ms = None
    if graph:
        gr = (K.KtMoeGraph.mxfp8(cfg, T, inp["x"], inp["w_gate"], inp["bias"], q, y, idx, w, ws)
              if fp8 else K.KtMoeGraph(*args))
        for _ in range(warmup):
            gr.launch()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        t0.record()
        for _ in range(steps):
            gr.launch()
        t1.record()
        torch.cuda.synchronize()
        barrier(world)
        graph_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
        gr.destroy()
        rc = K.kt_moe_check(ws)
        if rc != K.KT_OK:
            raise RuntimeError(f"device error in the graph launches: {K.strerror(rc)}")

    # End to end through the same C ABI call, host buffers: pinned x in, y out.
    x_h = inp["x"].cpu().pin_memory()
    y_h = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    x_d = torch.empty_like(inp["x"])
    for _ in range(3):
        x_d.copy_(x_h, non_blocking=True)
        fwd(x_d)
        y_h.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(e2e_steps):
        x_d.copy_(x_h, non_blocking=True)
        fwd(x_d)
        y_h.copy_(y, non_blocking=True)
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)

    # The same, pipelined as a server would run it: step i+1's x is copied in on
    # one copy stream and step i's y copied out on another while the forwards
    # run back to back on the compute stream (two device and two host buffers
    # of each; every step still copies its own x in and its own y out).
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    xb = [torch.empty_like(inp["x"]) for _ in range(2)]
    yb = [torch.empty_like(y) for _ in range(2)]
    yh = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipe_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])          # x buffer b free again
            xb[b].copy_(x_h, non_blocking=True)
            ev_in[b].record(s_in)
        main.wait_event(ev_in[b])
        if i >= 2:
            main.wait_event(ev_out[b])               # y buffer b copied out
        fwd(xb[b], y_out=yb[b])
        ev_done[b].record(main)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            yh[b].copy_(yb[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(4):
        pipe_step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0.record(main)
    for i in range(e2e_steps):
        pipe_step(i)
    for b in range(2):
        main.wait_event(ev_out[b])
    t1.record(main)
    torch.cuda.synchronize()
    barrier(world)
    e2e_pipe_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    if not torch.equal(yh[(e2e_steps - 1) % 2].to(dev), y):
        raise RuntimeError("pipelined forward differs from the plain one")

    work = algorithmic(layer, idx.cpu().numpy())
    out = dict(inp=inp, idx=idx.cpu().numpy(), ms=ms_max, stage_ms=stage_ms, staged_ms=staged_ms,
               e2e_ms=e2e_ms, e2e_pipe_ms=e2e_pipe_ms, graph_ms=graph_ms,
               work=work, h2d=inp["x"].numel() * inp["x"].element_size(),
               d2h=y.numel() * y.element_size(), y32=y32, y16=y16)
    del ws, y
    return out


# ---------------------------------------------------------------------------
# Dump and replay of one step
# ---------------------------------------------------------------------------
def _np_of(t: torch.Tensor) -> np.ndarray:
    """A tensor as numpy; bf16 as its raw 16-bit patterns (numpy has no bf16)."""
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _tensor_of(a: np.ndarray, dtype: str, dev) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(dev)


def weight_probe(layer, inp) -> np.ndarray:
    """A few rows of the expert weights (first, middle and last slot), as fp32:
    enough to tell whether a redraw from the seed gave the same weights."""
    n = layer.n_experts + layer.n_shared
    rows = [inp["w1"][0, 0], inp["w3"][n // 2, -1], inp["w2"][n - 1, layer.dim // 2]]
    return np.concatenate([r.float().cpu().numpy() for r in rows])


def dump_step(path, layer, inp, idx, w, y, probe, rc, rank):
    from mixture_experts_layer_34_b200 import ktmoe as K
    os.makedirs(path, exist_ok=True)
    torch.cuda.synchronize()
    arrays = {"x": inp["x"], "w_gate": inp["w_gate"], "idx": idx, "w": w, "y": y}
    if inp["bias"] is not None:
        arrays["bias"] = inp["bias"]
    dtypes = {}
    for name, t in arrays.items():
        np.save(os.path.join(path, name + ".npy"), _np_of(t))
        dtypes[name] = "bf16" if t.dtype == torch.bfloat16 else str(t.dtype).replace("torch.", "")
    np.save(os.path.join(path, "w_probe.npy"), probe)
    meta = {"workload": layer.name, "T": layer.T, "rank": rank, "weight_seed": layer.seed,
            "check": K.strerror(rc), "library_version": K.kt_moe_version(),
            "checked_build": K.kt_moe_checked_build(), "dtypes": dtypes,
            "device": torch.cuda.get_device_name(), "torch": torch.__version__}
    with open(os.path.join(path, "meta.json"), "w") as f:
        json.dump(meta, f, indent=1)


def replay_step(path) -> dict:
    """Rerun a dumped step: same weights (redrawn and probed), the dumped x,
    w_gate and bias; the routing and y must come out identical."""
    from mixture_experts_layer_34_b200 import ktmoe as K
    meta = json.load(open(os.path.join(path, "meta.json")))
    layer = W.BY_NAME[meta["workload"]]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    load = lambda n: _tensor_of(np.load(os.path.join(path, n + ".npy")), meta["dtypes"][n], dev)
    inp = W.make_layer(layer, dev)
    probe_ok = bool(np.array_equal(weight_probe(layer, inp),
                                   np.load(os.path.join(path, "w_probe.npy"))))
    inp["x"], inp["w_gate"] = load("x"), load("w_gate")
    inp["bias"] = load("bias") if "bias" in meta["dtypes"] else None
    cfg = K.config_for(layer)
    T = layer.T
    ws = K.alloc_workspace(cfg, T, dev)
    y = torch.empty_like(load("y"))
    idx = torch.empty((T, layer.topk), dtype=torch.int32, device=dev)
    w = torch.empty((T, layer.topk), dtype=torch.float32, device=dev)
    if layer.dtype in ("mxfp8", "mxfp4"):
        q = K.pack_mxfp8(cfg, inp["w1"], inp["w3"], inp["w2"])
        K.kt_moe_forward_mxfp8(cfg, T, inp["x"], inp["w_gate"], inp["bias"], q["w1q"], q["w3q"],
                               q["w2q"], q["sf_up"], q["sf_down"], y, idx, w, ws)
    else:
        K.kt_moe_forward(cfg, T, inp["x"], inp["w_gate"], inp["bias"], inp["w1"], inp["w3"],
                         inp["w2"], y, idx, w, ws)
    rc = K.kt_moe_check(ws)
    y_ref = load("y")
    same = {"idx": torch.equal(idx, load("idx")), "w": torch.equal(w, load("w")),
            "y": torch.equal(y, y_ref)}
    dy = float((y.float() - y_ref.float()).abs().max()) if not same["y"] else 0.0
    return {"replay": meta["workload"], "dumped_check": meta["check"], "check": K.strerror(rc),
            "weights_redrawn_identically": probe_ok, "identical": same, "max_abs_dy": dy,
            "match": probe_ok and rc == K.KT_OK and all(same.values())}


NEAR_TIE = 1e-5   # routing may differ from the oracle's only where its margins are this small


def cpu_baseline_leg(layer, inp, res, target_s: float, full: bool = False) -> dict:
    """The CPU oracle on this host's cores, on the timed workload's own inputs
    (copied to the host outside every GPU timing), and what its results say
    about the timed GPU run.

    Timed: the oracle's gate on all T tokens, then its literal expert loop on
    the first n tokens (n sized for about target_s seconds; all T if `full`).
    value = T / (gate time + loop time x T / n): the whole layer at the two
    measured rates (exactly the measured time when n = T).

    Checked against the GPU run, from those oracle results: the routing of all
    T tokens (how many differ from the oracle's, how many of those are not at
    the oracle's near ties, and the oracle's own near-tie count: k-th and
    (k+1)-th keys, or TG-th and (TG+1)-th group scores, within 1e-5), and the
    outputs of the n tokens routed alike, as max|dy| / RMS(y_oracle) of the fp32
    form and of the bf16 output."""
    import oracle.oracle as O
    kf = layer.kernel_fields()
    threads = O.num_threads()
    T, E, S = layer.T, layer.n_experts, layer.n_shared
    x_h = inp["x"].cpu()
    wg_h = inp["w_gate"].cpu()
    bias = None if inp["bias"] is None else inp["bias"].float().cpu().numpy()
    t = time.perf_counter()
    g = O.gate(kf, x_h, wg_h, bias)
    gate_s = time.perf_counter() - t
    host_w = {}

    def loop(n):
        need = set(range(E, E + S)) | set(int(e) for e in g["idx"][:n].ravel())
        for e in need - set(host_w):
            host_w[e] = (inp["w1"][e].cpu(), inp["w3"][e].cpu(), inp["w2"][e].cpu())
        pick = lambda j: [host_w[e][j] if e in host_w else None for e in range(E + S)]
        t = time.perf_counter()
        y = O.forward(kf, x_h, g["idx"], g["w"], pick(0), pick(1), pick(2), range(n),
                      bias is not None)
        return y, time.perf_counter() - t

    n = T if full else max(1, min(T, threads))
    y_ref, loop_s = loop(n)
    if not full and loop_s < 0.5 * target_s and n < T:
        n = int(min(T, max(n + 1, n * target_s / max(loop_s, 1e-3)), 64 * threads))
        y_ref, loop_s = loop(n)
    total_s = gate_s + loop_s * T / n
    what = (f"all {T} tokens" if n == T else
            f"gate on all {T} tokens ({gate_s:.2f} s) + expert loop on the first {n} "
            f"({loop_s:.2f} s), extrapolated to T")
    cpu = {"value": T / total_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"{layer.name}: {what}; fp64 oracle", "gate_s": round(gate_s, 3),
           "loop_tokens": n, "loop_s": round(loop_s, 3)}

    idx_gpu = res["idx"]
    diff = np.where((g["idx"] != idx_gpu).any(1))[0]
    near = (g["kth_margin"] <= NEAR_TIE) | (g["grp_margin"] <= NEAR_TIE)
    routing = {"tokens": T, "differ_from_oracle": int(len(diff)),
               "differ_away_from_near_ties": int((~near[diff]).sum()),
               "oracle_near_tie_tokens": int(near.sum()), "near_tie_threshold": NEAR_TIE}
    parity = None
    if res.get("y32") is not None:
        keep = np.setdiff1d(np.arange(n), diff)
        rms = float(np.sqrt(np.mean(y_ref[keep] ** 2)))
        sel = torch.as_tensor(keep, device=res["y32"].device)
        d32 = float(np.abs(res["y32"][sel].cpu().numpy() - y_ref[keep]).max())
        d16 = float(np.abs(res["y16"][sel].float().cpu().numpy() - y_ref[keep]).max())
        parity = {"tokens": int(len(keep)), "max_abs_dy_over_rms_fp32": round(d32 / rms, 6),
                  "max_abs_dy_over_rms_bf16_output": round(d16 / rms, 6),
                  "bound": 1e-4 if layer.dtype == "f32" else 2e-2,
                  "note": "first tokens of the timed workload routed alike, against the fp64 "
                          "oracle; fp32 form = the sum before its bf16 rounding"}
    return {"cpu_baseline": cpu, "routing": routing, "parity": parity}


def tensor_mult(layer) -> float:
    """Dense tensor rate of the layer's expert GEMMs relative to bf16: the
    block-scaled forms run tcgen05 kind::mxf8f6f4 at the FP8 rate (nominally 2x;
    E2M1 operands there do not run faster)."""
    return 2.0 if layer.dtype in ("mxfp8", "mxfp4") else 1.0


def layer_fracs(layer, res, steps, peaks, clk_mhz, clk_max) -> dict:
    """A layer's throughput against both roofs: its algorithmic bytes over the
    HBM copy peak and its FLOPs over the clock-matched tensor peak of its dtype."""
    ms = res["ms"] / steps
    tpk, _ = clock_scaled_peak(peaks["bf16_tflops"] * tensor_mult(layer), clk_mhz, clk_max)
    return {"layer_tflops": round(res["work"]["flops_layer"] / (ms / 1e3) / 1e12, 1),
            "layer_hbm_gbs": round(res["work"]["bytes_layer"] / (ms / 1e3) / 1e9, 1),
            "layer_hbm_frac": round(res["work"]["bytes_layer"] / (ms / 1e3) / 1e9
                                    / peaks["hbm_gbs"], 4),
            "layer_tensor_frac": round(res["work"]["flops_layer"] / (ms / 1e3) / 1e12 / tpk, 4)}


def region_clock(clk: dict, name: str):
    """Median SM clock inside a timed region, else of the whole run."""
    reg = (clk.get("regions") or {}).get(name) or {}
    return reg.get("sm_mhz") or clk.get("sm_mhz"), clk.get("sm_max_mhz")


def tensor_roofline(kernel, flops, ms, peaks, clk, region, mult=1.0, traffic_bytes=None,
                    dtype_note="bf16") -> dict:
    """Roofline entry of a tensor-bound kernel: its algorithmic FLOPs over its
    mean event-timed duration, against the measured burst peak (x mult for
    another dtype) matched to the median SM clock of its timed region."""
    f, fmax = region_clock(clk, region)
    peak, rule = clock_scaled_peak(peaks["bf16_tflops"] * mult, f, fmax)
    ach = flops / (ms / 1e3) / 1e12
    return {"kernel": kernel, "bound": "tensor", "achieved": round(ach, 1),
            "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(ach / peak, 4),
            "traffic": traffic_bytes,
            "peak_source": f"{peaks['source']} {dtype_note} burst"
                           + (f" x {mult:g} (nominal dtype ratio)" if mult != 1.0 else "")
                           + f"; {rule}",
            "peak_clock_mhz": f, "sm_max_mhz": fmax,
            "frac_of_sustained": round(ach / (peaks["bf16_tflops_sustained"] * mult), 4)}


def hbm_roofline(kernel, nbytes, ms, peaks, traffic_bytes=None) -> dict:
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"kernel": kernel, "bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic_bytes,
            "peak_source": peaks["source"] + " HBM copy"}


def extra_workloads(a) -> list:
    if a.extra_workloads == "none":
        return []
    if a.extra_workloads == "auto":
        return [W.V2_LITE.name, W.V2.name] if a.workload == W.V3_PREFILL.name else []
    return [n for n in a.extra_workloads.split(",") if n]


def run_ours(a):
    rank, world, local = dist_env()
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    from mixture_experts_layer_34_b200 import ktmoe as K
    K.lib()   # fail loudly if the CUDA library is missing
    peaks = load_peaks()
    layer = W.BY_NAME[a.workload]

    if world > 1 and a.parallel == "ep":
        return run_ep(a, layer, dev, rank, world, local, peaks)
    cpu_leg = rank == 0 and world == 1 and not a.no_cpu_baseline
    clocks = ClockSampler(local)
    clocks.start()
    pre = time_layer(layer, dev, rank, world, a.steps, a.warmup, a.e2e_steps, dump=a.dump,
                     clocks=clocks, keep_y32=cpu_leg)
    epr = None
    if world == 1 and a.ep_ranks > 1:
        epr = time_ep_ranks(layer, pre["inp"], dev, a.ep_ranks, a.steps, a.warmup)
    dec = None
    if a.decode_workload != "none":
        dlayer = W.BY_NAME[a.decode_workload]
        dec = time_layer(dlayer, dev, rank, world, a.steps, a.warmup, a.e2e_steps, graph=True,
                         dump=a.dump, clocks=clocks, keep_y32=cpu_leg)
    # The other named layers (V2-Lite one prefill chunk, V2), timed the same way.
    extra = {}
    for name in extra_workloads(a):
        res = time_layer(W.BY_NAME[name], dev, rank, world, a.steps, a.warmup, a.e2e_steps,
                         dump=a.dump, clocks=clocks)
        res.pop("inp")
        torch.cuda.empty_cache()
        extra[name] = res
    # The same layers with MXFP8 and MXFP4 expert weights (same shapes, seeds and
    # tokens).
    mx = {}
    for fmt, skip in (("mxfp8", a.no_mxfp8), ("mxfp4", a.no_mxfp4)):
        if skip:
            continue
        for key, base in (("prefill", layer.name), ("decode", a.decode_workload)):
            name = base + "_" + fmt
            if name in W.BY_NAME:
                res = time_layer(W.BY_NAME[name], dev, rank, world, a.steps, a.warmup,
                                 a.e2e_steps, graph=key == "decode", dump=a.dump, clocks=clocks)
                res.pop("inp")
                mx.setdefault(fmt, {})[key] = (W.BY_NAME[name], res)
    clk = clocks.stop()

    # CPU baseline leg: the oracle on the host (rank 0, one GPU), after every GPU
    # timing; its results also check the timed runs' routing and outputs.
    leg = dleg = None
    if cpu_leg:
        leg = cpu_baseline_leg(layer, pre["inp"], pre, a.cpu_seconds)
        if dec:
            dleg = cpu_baseline_leg(W.BY_NAME[a.decode_workload], dec["inp"], dec, a.cpu_seconds,
                                    full=True)
    pre.pop("inp")
    if dec:
        dec.pop("inp")
    torch.cuda.empty_cache()

    if rank == 0:
        T, K_ = layer.T, a.steps
        tokens = world * T * K_
        value = tokens / (pre["ms"] / 1e3)
        fl = layer_fracs(layer, pre, K_, peaks, *region_clock(clk, layer.name))
        up_ms = pre["stage_ms"]["up_gemm"]
        routing = load_stats(layer, pre["idx"])
        if leg:
            routing["oracle"] = leg["routing"]
        line = {
            "metric": "MoE layer tokens/s (prefill T=8192, decode T=8) + % of HBM/tensor roofline",
            "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K_,
            "warmup": a.warmup, "ms_per_step": round(pre["ms"] / K_, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if layer.dtype == "bf16" else layer.dtype,
            "data": "synthetic (seeded; random-init weights of the V3 layer shape)",
            "impl": "ours",
            "config": {"workload": layer.name, "T": T, "dim": layer.dim, "experts": layer.n_experts,
                       "groups": f"{layer.n_groups}/{layer.topk_groups}", "topk": layer.topk,
                       "shared": layer.n_shared, "inter": layer.inter,
                       "load": "Zipf(1.1)" if layer.bias == "zipf" else "seeded gate",
                       "parallelism": f"dp{world} (replicas, no collective)",
                       "l2": "inputs larger than L2: ~22 GB of expert weights read per step"},
            # stage_ms: a separate pass of the same steps with stage events;
            # staged_ms_per_step is that pass's step time.
            "stage_ms": {k: round(v, 4) for k, v in pre["stage_ms"].items()},
            "staged_ms_per_step": round(pre["staged_ms"], 4),
            "routing": routing,
            **fl,
            "roofline": tensor_roofline("grouped gate/up GEMM (tcgen05)",
                                        pre["work"]["flops_up"], up_ms, peaks, clk, layer.name,
                                        mult=tensor_mult(layer),
                                        traffic_bytes=traffic("up", layer.name)),
            "e2e": {"value": round(world * T * a.e2e_steps / (pre["e2e_ms"] / 1e3), 1),
                    "unit": "tokens/s", "h2d_bytes_per_step": pre["h2d"],
                    "d2h_bytes_per_step": pre["d2h"]},
            # The same host-buffer steps with the copies of neighbouring steps
            # overlapped with the compute (two copy streams, double buffers).
            "e2e_pipelined": {"value": round(world * T * a.e2e_steps / (pre["e2e_pipe_ms"] / 1e3), 1),
                              "unit": "tokens/s", "h2d_bytes_per_step": pre["h2d"],
                              "d2h_bytes_per_step": pre["d2h"]},
            "gpu_launches": LAUNCHES_PER_FORWARD * K_,
            "cpu_baseline": leg["cpu_baseline"] if leg else None,
            "parity": leg["parity"] if leg else None,
            "clocks": clk,
        }
        line["roofline_down"] = tensor_roofline("grouped down GEMM (tcgen05)",
                                                pre["work"]["flops_down"],
                                                pre["stage_ms"]["down_gemm"], peaks, clk,
                                                layer.name, mult=tensor_mult(layer),
                                                traffic_bytes=traffic("down", layer.name))
        if dec:
            dl = W.BY_NAME[a.decode_workload]
            dms = dec["ms"] / a.steps
            droute = load_stats(dl, dec["idx"])
            if dleg:
                droute["oracle"] = dleg["routing"]
            line["decode"] = {
                "workload": dl.name, "value": round(world * dl.T / (dms / 1e3), 1),
                "unit": "tokens/s", "ms_per_step": round(dms, 4),
                "active_experts": dec["work"]["active_experts"],
                "routing": droute,
                "stage_ms": {k: round(v, 4) for k, v in dec["stage_ms"].items()},
                **layer_fracs(dl, dec, a.steps, peaks, *region_clock(clk, dl.name)),
                "roofline": hbm_roofline("grouped gate/up GEMM (tcgen05)", dec["work"]["bytes_up"],
                                         dec["stage_ms"]["up_gemm"], peaks,
                                         traffic("up", dl.name)),
                "e2e": {"value": round(world * dl.T * a.e2e_steps / (dec["e2e_ms"] / 1e3), 1),
                        "unit": "tokens/s", "h2d_bytes_per_step": dec["h2d"],
                        "d2h_bytes_per_step": dec["d2h"]},
                # the same steps replayed as one CUDA graph per step (kt_moe_graph_launch)
                "graph": {"ms_per_step": round(dec["graph_ms"] / a.steps, 4),
                          "value": round(world * dl.T * a.steps / (dec["graph_ms"] / 1e3), 1),
                          "unit": "tokens/s"},
                "cpu_baseline": dleg["cpu_baseline"] if dleg else None,
                "parity": dleg["parity"] if dleg else None,
            }
        for name, res in extra.items():
            xl = W.BY_NAME[name]
            ms = res["ms"] / K_
            f = layer_fracs(xl, res, K_, peaks, *region_clock(clk, name))
            line[name] = {
                "workload": name, "T": xl.T, "value": round(world * xl.T / (ms / 1e3), 1),
                "unit": "tokens/s", "ms_per_step": round(ms, 4),
                "stage_ms": {k: round(v, 4) for k, v in res["stage_ms"].items()},
                **f,
                "roofline": hbm_roofline("grouped gate/up GEMM (tcgen05)", res["work"]["bytes_up"],
                                         res["stage_ms"]["up_gemm"], peaks, traffic("up", name)),
                "roofline_tensor": tensor_roofline("grouped gate/up GEMM (tcgen05)",
                                                   res["work"]["flops_up"],
                                                   res["stage_ms"]["up_gemm"], peaks, clk, name),
                "e2e": {"value": round(world * xl.T * a.e2e_steps / (res["e2e_ms"] / 1e3), 1),
                        "unit": "tokens/s", "h2d_bytes_per_step": res["h2d"],
                        "d2h_bytes_per_step": res["d2h"]},
            }
        notes = {"mxfp8": "MXFP8 expert weights (E4M3, power-of-two scale per 32 along K); "
                          "bf16 tokens, gate and output",
                 "mxfp4": "MXFP4 expert weights (E2M1 codes two per byte, power-of-two scale "
                          "per 32 along K) against MXFP8 (E4M3) tokens and hidden rows; bf16 "
                          "gate and output"}
        for fmt, runs in mx.items():
            line[fmt] = {"note": notes[fmt]}
            for key, (fl_, res) in runs.items():
                ms = res["ms"] / K_
                ent = {"workload": fl_.name, "value": round(world * fl_.T / (ms / 1e3), 1),
                       "unit": "tokens/s", "ms_per_step": round(ms, 4),
                       "stage_ms": {k: round(v, 4) for k, v in res["stage_ms"].items()},
                       "e2e": {"value": round(world * fl_.T * a.e2e_steps / (res["e2e_ms"] / 1e3), 1),
                               "unit": "tokens/s"}}
                up_ms_ = res["stage_ms"]["up_gemm"]
                kern = ("grouped gate/up GEMM (tcgen05 kind::mxf8f6f4"
                        + (", E2M1 x E4M3)" if fmt == "mxfp4" else ")"))
                if key == "prefill":
                    # Both block-scaled forms run tcgen05 kind::mxf8f6f4, whose
                    # dense rate is the FP8 one (2x bf16; E2M1 operands there do
                    # not run faster).
                    ent["roofline"] = tensor_roofline(kern, res["work"]["flops_up"], up_ms_, peaks,
                                                      clk, fl_.name, mult=2.0,
                                                      traffic_bytes=traffic("up", fl_.name))
                else:
                    lgbs = res["work"]["bytes_layer"] / (ms / 1e3) / 1e9
                    ent["layer_hbm_gbs"] = round(lgbs, 1)
                    ent["layer_hbm_frac"] = round(lgbs / peaks["hbm_gbs"], 4)
                    ent["roofline"] = hbm_roofline(kern, res["work"]["bytes_up"], up_ms_, peaks,
                                                   traffic("up", fl_.name))
                if res.get("graph_ms") is not None:
                    ent["graph"] = {"ms_per_step": round(res["graph_ms"] / K_, 4),
                                    "value": round(world * fl_.T * K_ / (res["graph_ms"] / 1e3), 1),
                                    "unit": "tokens/s"}
                line[fmt][key] = ent
        if epr:
            line["expert_parallel"] = epr
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_ep(a, layer, dev, rank, world, local, peaks):
    """--parallel ep with N > 1: one JSON line for the expert-parallel layer."""
    clocks = ClockSampler(local)
    clocks.start()
    ms = time_ep_layer(layer, dev, rank, world, a.steps, a.warmup, a.ep_placement, a.ep_output)
    clk = clocks.stop()
    if rank == 0:
        T = layer.T
        print(json.dumps({
            "metric": "MoE layer tokens/s (prefill T=8192, decode T=8) + % of HBM/tensor roofline",
            "value": round(T * a.steps / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms / a.steps, 4),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; random-init weights of the V3 layer shape)",
            "impl": "ours",
            "config": {"workload": layer.name, "T": T, "parallelism": f"ep{world} "
                       "(experts split, fp32 partials all-reduced over NCCL)",
                       "placement": a.ep_placement, "output": a.ep_output,
                       "l2": "inputs larger than L2"},
            "gpu_launches": (LAUNCHES_PER_FORWARD + 1) * a.steps,
            "clocks": clk,
        }), flush=True)
    torch.distributed.destroy_process_group()


# ---------------------------------------------------------------------------
# Reference arm: the CPU oracle, rank 0 only
# ---------------------------------------------------------------------------
def run_reference(a):
    rank, world, local = dist_env()
    if rank != 0:
        return
    import oracle.oracle as O
    layer = W.BY_NAME[a.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    threads = O.num_threads()
    n = max(1, min(layer.T, threads))
    gi = W.make_gate_inputs(layer)
    kf = layer.kernel_fields()
    bias = None if gi["bias"] is None else gi["bias"].numpy()
    xs = gi["x"][:n].contiguous()
    g = O.gate(kf, xs, gi["w_gate"], bias)
    need = set(range(layer.n_experts, layer.n_experts + layer.n_shared)) | set(g["idx"].ravel().tolist())
    full = W.make_layer(layer, dev)
    nall = layer.n_experts + layer.n_shared
    w1 = [full["w1"][e].cpu() if e in need else None for e in range(nall)]
    w3 = [full["w3"][e].cpu() if e in need else None for e in range(nall)]
    w2 = [full["w2"][e].cpu() if e in need else None for e in range(nall)]
    del full

    def step():
        gg = O.gate(kf, xs, gi["w_gate"], bias)
        O.forward(kf, xs, gg["idx"], gg["w"], w1, w3, w2, range(n), bias is not None)

    for _ in range(a.warmup):
        step()
    t = time.perf_counter()
    for _ in range(a.steps):
        step()
    dt = time.perf_counter() - t
    value = n * a.steps / dt
    sample = f"first {n} tokens of {layer.name} per step: fp64 gate + literal expert loop"
    print(json.dumps({
        "metric": "MoE layer tokens/s (prefill T=8192, decode T=8) + % of HBM/tensor roofline",
        "value": round(value, 3), "unit": "tokens/s", "n_gpus": a.gpus, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(dt / a.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": layer.name, "T": layer.T, "sample_tokens_per_step": n},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": min(threads, n),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    a = parse_args(argv)
    if a.replay:
        r = replay_step(a.replay)
        print(json.dumps(r))
        sys.exit(0 if r["match"] else 1)
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
