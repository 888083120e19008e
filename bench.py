#!/usr/bin/env python
"""Benchmark the decode weight sweep through libqgemv.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--path launches|persistent]

A step is one full sweep of the decoder's weights (every layer's q|k|v, o,
gate/up + SwiGLU and down, then the LM head + argmax) replayed from a CUDA
graph, one launch per call (chained with programmatic dependent launch).
`--path persistent` times the same S=1 stages as one persistent launch
(qg_sweep_run) instead; on B200 its grid-wide barrier between stages costs
more than the launch chaining it replaces, so it is not the default.  The default workload is the Qwen3-VL-2B-shaped int8 block-32 S=1
sweep (1.83 GB per sweep, far larger than the 126 MB L2, so no flush is
needed between steps).  N > 1 runs one replica per GPU (launch with torchrun):
decode sweeps are independent, so nothing is exchanged and the time is the
max over ranks.

`--impl reference` times the CPU oracle (fp64 dequantize-then-matvec, on the
host's cores) on a bounded sample of the same workload, for the driver's
ratio; it never touches the GPU.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "weight-stream GB/s (% of HBM peak) and decode sweeps/s, S=1 int8 block-32"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic.txt")

# name -> (decoder, body format, head format, S[, decode step[, K/V cache rows]])
WORKLOADS = {
    "qwen3vl-2b": ("QWEN3VL_2B", 0, 0, 1),
    "qwen3vl-2b-f16head": ("QWEN3VL_2B", 0, 2, 1),
    "qwen3vl-2b-decode": ("QWEN3VL_2B", 0, 0, 1, True),
    "qwen3vl-2b-decode-attn4k": ("QWEN3VL_2B", 0, 0, 1, True, 4096),
    "qwen3vl-8b-decode-attn4k": ("QWEN3VL_8B", 0, 0, 1, True, 4096),
    "qwen3vl-4b": ("QWEN3VL_4B", 0, 0, 1),
    "qwen3vl-4b-int4": ("QWEN3VL_4B", 1, 0, 1),
    "qwen3vl-8b": ("QWEN3VL_8B", 0, 0, 1),
    "qwen3vl-8b-int4": ("QWEN3VL_8B", 1, 0, 1),
    "qwen3vl-8b-s16": ("QWEN3VL_8B", 0, 0, 16),
    "dense-27b": ("DENSE_27B", 0, 0, 1),
    "dense-27b-int4": ("DENSE_27B", 1, 1, 1),
}
DEFAULT_WORKLOAD = "qwen3vl-2b"
SINGLE_GEMV = "gemv-2048"  # the single 2048x2048 int8 GEMV (fits in L2: rotated copies)
FMT_NAME = {0: "int8 block-32", 1: "int4 group-64", 2: "fp16"}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(WORKLOADS) + [SINGLE_GEMV])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="launches", choices=["launches", "persistent"],
                    help="S=1 sweep as one launch per call (default) or one persistent launch")
    ap.add_argument("--graph-sweeps", type=int, default=1,
                    help="sweeps captured per CUDA graph (steps are rounded up to a multiple)")
    ap.add_argument("--cpu-budget-s", type=float, default=10.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    return a


# --------------------------------------------------------------- helpers ----

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of `value` over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, elapsed_s_max: float, world: int) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time (weak scaling: each rank runs the same fixed work)."""
    return units_per_rank * world / elapsed_s_max


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# The sources of the S=1, S<=16 and attention kernels whose DRAM traffic profiles/dram_traffic.txt
# records: a committed traffic figure is used only while these are unchanged.
KERNEL_SOURCES = ("qg_device.cuh", "qg_gemv.cu", "qg_gemv_impl.cuh", "qg_internal.h",
                  "qg_gemm_tc.cu", "qg_attention.cu")


def csrc_digest() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "int4_quantized_decode_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None).  Kernel names are stored with
    spaces written as underscores."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            for line in f:
                if line.startswith("#") or "=" not in line:
                    continue
                kv = dict(p.split("=", 1) for p in line.split())
                if (kv.get("kernel") == kernel.replace(" ", "_") and kv.get("workload") == workload
                        and kv.get("csrc") == csrc_digest()):
                    return float(kv["bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons: a sampler every 200 ms while a
    region runs, and one-shot queries right before and after it (a timed
    region shorter than the sampling period still gets a record)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def _cmd(self, loop: bool):
        c = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
             "-i", str(self.gpu)]
        return c + (["-lms", "200"] if loop else [])

    @classmethod
    def _parse(cls, text: str):
        sm, mx, reasons = [], None, set()
        for line in text.splitlines():
            r = line.strip().split(", ")
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(cls.REASONS, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return sm, mx, reasons

    def query_once(self):
        try:
            out = subprocess.run(self._cmd(False), capture_output=True, text=True,
                                 timeout=10).stdout
        except (OSError, subprocess.TimeoutExpired):
            return None
        sm, mx, reasons = self._parse(out)
        if not sm:
            return None
        return {"sm_mhz": sm[0], "sm_max_mhz": mx, "reasons": sorted(reasons)}

    def start(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", delete=False, suffix=".csv")
            self.proc = subprocess.Popen(self._cmd(True), stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self, before=None, after=None, soak_s=0.0):
        """The record: median SM clock and the union of active reasons over
        the sampler's rows and the one-shot queries `before` and `after`."""
        sm, mx, reasons = [], None, set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.flush()
            self.out.seek(0)
            sm, mx, reasons = self._parse(self.out.read())
            self.out.close()
            os.unlink(self.out.name)
        for q in (before, after):
            if q:
                sm.append(q["sm_mhz"])
                mx = q["sm_max_mhz"]
                reasons |= set(q["reasons"])
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons), "before": before, "after": after,
                "soak_s": round(soak_s, 3)}


# ----------------------------------------------------------- CPU oracle ----

# Weights the host quantizes for an oracle sweep: a sweep up to this size is
# run whole (every layer and the head); a larger decoder runs the head and as
# many of its first layers as fit, and says so.
ORACLE_MAX_WEIGHTS = 2.5e9


class OracleSweep:
    """The CPU oracle (test infrastructure) over a decode weight sweep: the
    same matrices, shapes and data flow as the GPU sweep, drawn on the host
    from the same seeded distributions and quantized by the oracle.  One run
    is per layer q|k|v(|gate) -> o (on fp16 q) -> gate/up + SwiGLU -> down (on
    fp16 h), then the head + argmax, each an fp64 dequantize-then-matvec, for
    every one of the S tokens."""

    def __init__(self, dec, body_fmt, head_fmt, S):
        import numpy as np

        import oracle
        from int4_quantized_decode_b200 import workloads as wl
        self.np, self.oracle, self.dec, self.S = np, oracle, dec, S
        self.body_fmt, self.head_fmt = body_fmt, head_fmt
        per_layer = dec.weight_count(include_head=False) // dec.layers
        room = ORACLE_MAX_WEIGHTS - dec.vocab * dec.hidden
        self.layers = max(1, min(dec.layers, int(room // per_layer)))
        self.mats = []
        for l in range(self.layers):
            m = {name: self._quantized(dec.weight_seed(l, name), n, k, body_fmt)
                 for name, n, k in dec.layer_matrices()}
            self.mats.append(m)
        self.head = self._quantized(dec.weight_seed(-1, "head"), dec.vocab, dec.hidden, head_fmt)
        self.bytes = sum(self._nbytes(m) for L in self.mats for m in L.values()) + \
            self._nbytes(self.head)
        self.xs = [[wl.act_fp16(dec.hidden, dec.x_seed(l) + 7919 * t, "cpu").numpy()
                    .view(np.uint16) for t in range(S)] for l in range(self.layers + 1)]

    @staticmethod
    def _nbytes(m):
        return sum(a.nbytes for a in m[:3] if a is not None)

    def _quantized(self, seed, n, k, fmt):
        from int4_quantized_decode_b200 import workloads as wl
        w = wl.weight_fp32(n, k, seed, "cpu").numpy()
        if fmt == 2:
            return (w.astype(self.np.float16).view(self.np.uint16), None, None)
        if fmt == 0:
            c, sc = self.oracle.quantize_block32(w)
            return (c, sc, None)
        return self.oracle.quantize_int4_g64(w)

    def run(self):
        np, orc, dec = self.np, self.oracle, self.dec
        qkv = [name for name, _ in dec.qkv_parts()]
        idx = -1
        for t in range(self.S):
            for l, m in enumerate(self.mats):
                x = self.xs[l][t]
                q, _ = orc.matvec(self.body_fmt, *m[qkv[0]], x)
                for name in qkv[1:]:
                    orc.matvec(self.body_fmt, *m[name], x)
                orc.matvec(self.body_fmt, *m["o"], q.astype(np.float16).view(np.uint16))
                g, mg = orc.matvec(self.body_fmt, *m["gate"], x)
                u, mu = orc.matvec(self.body_fmt, *m["up"], x)
                h, _ = orc.swiglu(g, u, mg, mu, orc.GEMV_TOL)
                orc.matvec(self.body_fmt, *m["down"], h.astype(np.float16).view(np.uint16))
            logits, _ = orc.matvec(self.head_fmt, *self.head, self.xs[self.layers][t])
            idx = orc.argmax(logits)
        return idx

    def describe(self):
        whole = self.layers == self.dec.layers
        what = (f"one whole sweep of the {self.dec.name} workload" if whole else
                f"the head and the first {self.layers} of {self.dec.layers} layers of the "
                f"{self.dec.name} sweep (a whole sweep would quantize more than "
                f"{ORACLE_MAX_WEIGHTS / 1e9:.1f}e9 weights on the host)")
        return (f"{what}: {self.bytes / 1e9:.3f} GB of {FMT_NAME[self.body_fmt]} body + "
                f"{FMT_NAME[self.head_fmt]} head codes+scales, S={self.S}, fp64 "
                f"dequantize-then-matvec + SwiGLU + argmax, host-drawn weights of the same "
                f"seeded distribution quantized by the oracle")


def time_oracle(osw, threads, min_s=0.0, max_runs=1):
    """Seconds per oracle sweep on `threads` host threads: at least one run,
    repeated up to `max_runs` while under `min_s` seconds in total."""
    osw.oracle.set_num_threads(threads)
    runs, t0 = 0, time.perf_counter()
    while True:
        osw.run()
        runs += 1
        el = time.perf_counter() - t0
        if runs >= max_runs or el >= min_s:
            return el / runs, runs


def cpu_baseline(dec, body_fmt, head_fmt, S, sweep_bytes):
    import oracle
    cores = os.cpu_count() or 1
    osw = OracleSweep(dec, body_fmt, head_fmt, S)
    t1, _ = time_oracle(osw, 1)
    tn, runs = time_oracle(osw, cores, min_s=2.0, max_runs=8)
    oracle.set_num_threads(cores)
    gbs = osw.bytes / tn / 1e9
    return {"value": round(gbs, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sweeps_per_s": round(gbs * 1e9 / sweep_bytes, 4),
            "single_thread": {"value": round(osw.bytes / t1 / 1e9, 3), "unit": UNIT,
                              "cores": 1, "s_per_sweep": round(t1, 3)},
            "s_per_sweep": round(tn, 4),
            "sample": osw.describe() + f"; all-core figure the mean of {runs} runs"}


# ------------------------------------------------------------ reference ----

def run_reference(a):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    import oracle
    from int4_quantized_decode_b200 import workloads as wl
    dname, body_fmt, head_fmt, S = WORKLOADS[a.workload][:4]
    dec = getattr(wl, dname)
    sweep_bytes = _sweep_bytes(dec, body_fmt, head_fmt)
    cores = os.cpu_count() or 1
    osw = OracleSweep(dec, body_fmt, head_fmt, S)
    oracle.set_num_threads(cores)
    for _ in range(a.warmup):
        osw.run()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        osw.run()
    el = time.perf_counter() - t0
    gbs = a.steps * osw.bytes / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": UNIT,
        "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(el / a.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(a, dec, body_fmt, head_fmt, S, sweep_bytes),
        "sweeps_per_s": round(gbs * 1e9 / osw.bytes, 5),
        "cpu_baseline": {"value": round(gbs, 4), "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": "each step: " + osw.describe()},
        "e2e": {"value": round(gbs, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def _sweep_bytes(dec, body_fmt, head_fmt):
    bpw = {0: 1.0625, 1: 0.5625, 2: 2.0}
    return int(dec.weight_count(include_head=False) * bpw[body_fmt] +
               dec.vocab * dec.hidden * bpw[head_fmt])


def _context(workload):
    w = WORKLOADS[workload]
    return w[5] if len(w) > 5 else 0


def _config(a, dec, body_fmt, head_fmt, S, sweep_bytes):
    decode = len(WORKLOADS[a.workload]) > 4
    ctx = _context(a.workload)
    if ctx:
        step = (f", whole decode step (embedding gather, RMSNorm and residual fused, "
                f"RoPE + GQA attention over a {ctx}-row fp16 K/V cache per layer at its last "
                f"row; the argmax feeds the next step's gather); value counts weight bytes "
                f"only, the K/V rows read are kv_bytes")
    elif decode:
        step = (", whole decode step minus attention (embedding gather, RMSNorm and residual "
                "fused; the argmax feeds the next step's gather)")
    else:
        step = ""
    return {
        "workload": (f"{dec.name}-shaped decode weight sweep, {FMT_NAME[body_fmt]} body + "
                     f"{FMT_NAME[head_fmt]} head{' (tied)' if dec.tied_head else ''}, "
                     f"S={S}" + step),
        "layers": dec.layers, "hidden": dec.hidden, "inter": dec.inter,
        "vocab": dec.vocab, "S": S, "sweep_bytes": sweep_bytes,
        "parallelism": f"replicas x{a.gpus}",
        "l2": "inputs larger than L2 (no flush needed)",
    }


# ------------------------------------------------------------------- ours --

def run_ours(a):
    import torch

    from int4_quantized_decode_b200 import qgemv as qg
    from int4_quantized_decode_b200 import workloads as wl
    from int4_quantized_decode_b200.sweep import DecodeSweep

    rank, local, world = dist_env()
    if world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    dname, body_fmt, head_fmt, S = WORKLOADS[a.workload][:4]
    decode = len(WORKLOADS[a.workload]) > 4
    dec = getattr(wl, dname)
    sw = DecodeSweep(dec, body_fmt, head_fmt, S=S, device=dev, decode_step=decode,
                     context=_context(a.workload))
    persistent = a.path == "persistent"
    if a.path == "persistent" and S != 1:
        raise SystemExit("--path persistent needs an S=1 workload")
    G = max(1, a.graph_sweeps)
    graph = sw.capture(sweeps_per_graph=G, persistent=persistent)
    steps = ((a.steps + G - 1) // G) * G
    stream = torch.cuda.current_stream(dev)
    sweep_bytes = sw.weight_bytes

    # --- device-timed sweeps (inputs resident in HBM) ----------------------
    w0 = time.perf_counter()
    for _ in range((a.warmup + G - 1) // G):
        graph.replay()
    qg.qg_stream_check()
    per_replay = (time.perf_counter() - w0) / max(1, (a.warmup + G - 1) // G)
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local).start()
    # A timed region shorter than the sampler's period gets a soak of the same
    # replays first (untimed, about a second) so the record sees the clocks
    # this load runs at; one-shot queries bracket the timed region itself.
    soak = 0.0
    if per_replay * (steps // G) < 1.0:
        s0 = time.perf_counter()
        while time.perf_counter() - s0 < 1.0:
            for _ in range(max(1, int(0.05 / max(per_replay, 1e-6)))):
                graph.replay()
            torch.cuda.synchronize(dev)
        soak = time.perf_counter() - s0
    before = clocks.query_once()
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps // G):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    after = clocks.query_once()
    barrier()
    clk = clocks.stop(before, after, soak)
    qg.qg_stream_check()
    el_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    el_s = el_ms / 1e3
    value = aggregate(steps * sweep_bytes / 1e9, el_s, world)
    sweeps_s = aggregate(steps, el_s, world)

    # --- dominant kernel --------------------------------------------------
    if persistent:
        # the persistent sweep kernel is every launch of the timed region; its
        # average duration comes from the same CUDA events on its stream
        dom = {"kernel": "sweep_kernel (persistent sweep)", "us": el_ms * 1e3 / steps,
               "gbs": sweep_bytes / (el_ms * 1e-3 / steps) / 1e9, "bytes": sweep_bytes,
               "launches": steps}
        kinds = None
    else:
        # the dominant kernel is the kind of call with the largest share of
        # the sweep's time
        kinds = _time_kinds(sw, stream, dev, torch)
        names = KERNEL_OF_KIND[(S == 1, decode)]
        kd = max(kinds, key=lambda k: kinds[k]["share"])
        dom = {"kernel": names[kd], "us": kinds[kd]["us"], "gbs": kinds[kd]["gbs"],
               "bytes": kinds[kd]["bytes"], "launches": kinds[kd]["launches_per_sweep"] * steps,
               "share": kinds[kd]["share"], "kind": kd}

    # --- end to end: pinned host inputs -> sweep -> greedy token to host ---
    e2e = _time_e2e(sw, graph, G, steps, a.warmup, stream, dev, world, torch, persistent)

    peak, peak_kind = hbm_peak()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": a.warmup, "ms_per_step": round(el_ms / steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8/i4 x f16 -> f32" if S == 1 else "i8 x f16 -> f32 (mma f16)",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) fp16 activations)",
        "config": dict(_config(a, dec, body_fmt, head_fmt, S, sweep_bytes),
                       path="persistent (one launch per sweep)" if persistent
                       else "one launch per call",
                       **({"kv_bytes": sw.kv_bytes,
                           "gbs_incl_kv": round(value * (sweep_bytes + sw.kv_bytes) /
                                                sweep_bytes, 2)} if sw.kv_bytes else {})),
        "sweeps_per_s": round(sweeps_s, 2),
        "tokens_per_s": round(sweeps_s * S, 2),
        "hbm_frac": round(value / world / peak, 4),
        "roofline": {
            "bound": "hbm", "kernel": dom["kernel"], "achieved": round(dom["gbs"], 1),
            "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs (copy, MEASURED_PEAKS.json)"
            if peak_kind == "measured" else "fallback 6650 GB/s",
            "unit": "GB/s", "frac": round(dom["gbs"] / peak, 4),
            "traffic": profiled_traffic(dom["kernel"], a.workload),
            "algorithmic_bytes_per_launch": dom["bytes"],
            "launch_us": round(dom["us"], 3), "launches": dom["launches"],
            "time_share": round(dom.get("share", 1.0), 4),
            "sweep_frac": round(value / world / peak, 4)},
        **({"kernels": {k: {"kernel": KERNEL_OF_KIND[(S == 1, decode)][k],
                            "us_per_launch": round(v["us"], 3),
                            "launches_per_sweep": v["launches_per_sweep"],
                            "bytes_per_launch": v["bytes"], "gbs": round(v["gbs"], 1),
                            "frac": round(v["gbs"] / peak, 4), "time_share": round(v["share"], 4)}
                        for k, v in kinds.items()},
            "kernels_timing": "each kind alone: graph of its launches over all layers (the "
                              "head: 4 launches), L2 flushed before each replay"} if kinds else {}),
        "e2e": e2e,
        "gpu_launches": steps * sw.launches_per_sweep(persistent),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(dec, body_fmt, head_fmt, S, sweep_bytes)
    if rank == 0:
        print(json.dumps(line))
    del graph, sw
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


KERNEL_OF_KIND = {
    # (S == 1, decode step) -> kind -> the kernel that runs it
    (True, False): {"qkv": "gemv_ring_kernel", "o": "gemv_ring_kernel",
                    "gate_up": "gemv_ring_kernel (fused gate/up + SwiGLU)",
                    "down": "gemv_ring_kernel", "head": "gemv_ring_kernel (head + argmax)"},
    (True, True): {"qkv": "gemv_ring_kernel (RMSNorm in)", "o": "gemv_ring_kernel (residual)",
                   "attention": "decode_attention_kernel",
                   "gate_up": "gemv_ring_kernel (RMSNorm in, fused gate/up + SwiGLU)",
                   "down": "gemv_ring_kernel (residual)",
                   "head": "gemv_ring_kernel (RMSNorm in, head + argmax)"},
    (False, False): {"qkv": "gemm_tc_kernel", "o": "gemm_tc_kernel",
                     "gate_up": "gemm_tc_kernel (fused gate/up + SwiGLU)",
                     "down": "gemm_tc_kernel", "head": "gemv_ring_kernel (head + argmax)"},
}


def _time_kinds(sw, stream, dev, torch, reps=5):
    """Average launch duration of every kind of call in the sweep (qkv, o,
    gate/up, down, head, attention), each timed with CUDA events on its
    stream over a graph of that kind's launches across all layers, with L2
    flushed (a 256 MB write, more than the 126 MB L2) before every timed
    replay.  Returns per kind: us per launch, bytes per launch, launches per
    sweep, GB/s and the share of the summed time."""
    by_kind = {}
    for l in range(sw.dec.layers):
        for kind, nbytes, _ in sw.layer_calls(l):
            by_kind.setdefault(kind, []).append(nbytes)
    by_kind["head"] = [sw.head.nbytes]
    # the head runs once per sweep; its graph holds a few launches back to back
    # (each streams the whole head, far more than L2), as every other kind's
    # graph holds one launch per layer, so no figure carries a lone launch's
    # graph overhead
    head_reps = 4
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(device=dev)
    out = {}
    for kind in by_kind:
        g = torch.cuda.CUDAGraph()
        s.wait_stream(stream)
        with torch.cuda.graph(g, stream=s):
            if kind == "head":
                for _ in range(head_reps):
                    sw.run_head(s)
            else:
                for l in range(sw.dec.layers):
                    for k2, _, enqueue in sw.layer_calls(l, s):
                        if k2 == kind:
                            enqueue()
        stream.wait_stream(s)
        for _ in range(2):
            g.replay()
        total_ms = 0.0
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            total_ms += e0.elapsed_time(e1)
        n = len(by_kind[kind])
        us = total_ms * 1e3 / (reps * n * (head_reps if kind == "head" else 1))
        nbytes = sum(by_kind[kind]) / n
        out[kind] = {"us": us, "bytes": int(nbytes), "launches_per_sweep": n,
                     "gbs": nbytes / (us * 1e-6) / 1e9}
        del g
    del flush
    tot = sum(v["us"] * v["launches_per_sweep"] for v in out.values())
    for v in out.values():
        v["share"] = v["us"] * v["launches_per_sweep"] / tot
    return out


def _time_e2e(sw, graph, G, steps, warmup, stream, dev, world, torch, persistent):
    """Same metric through the public path with host buffers: each step copies
    that step's activations from pinned host memory, replays the sweep, and
    reads the greedy token back."""
    x_host = [x.cpu().pin_memory() for x in sw.inputs()]
    idx_host = torch.empty(1, dtype=torch.int32).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in x_host)
    d2h = idx_host.numel() * idx_host.element_size()
    single = sw.capture(sweeps_per_graph=1, persistent=persistent) if G != 1 else graph
    sw.graph = graph

    def one():
        for xd, xh in zip(sw.inputs(), x_host):
            xd.copy_(xh, non_blocking=True)
        single.replay()
        idx_host.copy_(sw.idx, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize(dev)
    n = max(10, steps // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    el_s = max_over_ranks(e0.elapsed_time(e1), world, dev) / 1e3
    return {"value": round(aggregate(n * sw.weight_bytes / 1e9, el_s, world), 2),
            "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n}


def run_single_gemv(a):
    """The single 2048 x 2048 int8 block-32 GEMV.  Its 4.46 MB fit in L2, so
    the HBM figure rotates through R distinct quantized copies (R x 4.46 MB,
    at least 4x the 126 MB L2), one launch per copy inside a CUDA graph; the
    same graph over one copy gives the labelled L2-hot figure."""
    import torch

    from int4_quantized_decode_b200 import qgemv as qg
    from int4_quantized_decode_b200 import workloads as wl

    rank, local, world = dist_env()
    if world != 1:
        raise SystemExit(f"--workload {SINGLE_GEMV} runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = wl.GEMV_2048
    n, k, R = cfg["n"], cfg["k"], 256
    W0 = qg.quantize(wl.weight_fp32(n, k, cfg["w_seed"], dev), qg.FMT_I8_B32)
    copies = [qg.QWeight(W0.fmt, n, k, W0.codes.clone(), W0.scales.clone(), None)
              for _ in range(R)]
    x = wl.act_fp16(k, cfg["x_seed"], dev)
    y = torch.empty(n, dtype=torch.float32, device=dev)
    nbytes = W0.nbytes
    stream = torch.cuda.Stream(device=dev)

    def graph_over(ws):
        with torch.cuda.stream(stream):
            for w in ws[:4]:
                qg.qg_gemv_s1(w, x, y, None, stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for w in ws:
                qg.qg_gemv_s1(w, x, y, None, stream)
        return g

    def timed(g, reps):
        # a graph replays on the current stream: time it there
        cur = torch.cuda.current_stream(dev)
        for _ in range(max(3, a.warmup)):
            g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for _ in range(reps):
            g.replay()
        e1.record(cur)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / 1e3

    reps = max(1, (a.steps + R - 1) // R)
    g_hbm = graph_over(copies)
    clocks = ClockSampler(local).start()
    before = clocks.query_once()
    el_s = timed(g_hbm, reps)
    clk = clocks.stop(before, clocks.query_once())
    g_hot = graph_over([copies[0]] * R)
    el_hot = timed(g_hot, reps)
    qg.qg_stream_check()
    launches = reps * R
    value = launches * nbytes / el_s / 1e9
    hot = launches * nbytes / el_hot / 1e9

    # end to end through the C ABI with host buffers: x in, y out, every call
    x_host = x.cpu().pin_memory()
    y_host = torch.empty(n, dtype=torch.float32).pin_memory()
    m = max(50, min(2000, a.steps // 4))
    with torch.cuda.stream(stream):
        for i in range(m + 10):
            if i == 10:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            x.copy_(x_host, non_blocking=True)
            qg.qg_gemv_s1(copies[i % R], x, y, None, stream)
            y_host.copy_(y, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e = m * nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9

    peak, peak_kind = hbm_peak()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": 1,
        "steps": launches, "warmup": a.warmup, "ms_per_step": round(el_s * 1e3 / launches, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8 x f16 -> f32", "data": "synthetic (seeded N(0,0.02) weights, N(0,1) x)",
        "config": {"workload": (f"single {n}x{k} int8 block-32 GEMV, S=1; a step is one launch; "
                                f"HBM figure over {R} rotating copies "
                                f"({R * nbytes / 1e9:.2f} GB), one launch per copy in a graph"),
                   "n": n, "k": k, "copies": R, "bytes_per_launch": nbytes,
                   "l2_hot_gbs": round(hot, 2),
                   "l2": "rotating copies totalling >= 4x L2 (no flush needed)"},
        "roofline": {"bound": "hbm", "kernel": "gemv_ring_kernel (single GEMV)",
                     "achieved": round(value, 1), "peak": peak,
                     "peak_kind": f"{peak_kind} hbm_gbs (copy, MEASURED_PEAKS.json)"
                     if peak_kind == "measured" else "fallback 6650 GB/s",
                     "unit": "GB/s", "frac": round(value / peak, 4), "traffic": None,
                     "algorithmic_bytes_per_launch": nbytes,
                     "launch_us": round(el_s * 1e6 / launches, 3), "launches": launches},
        "e2e": {"value": round(e2e, 2), "unit": UNIT, "h2d_bytes_per_step": k * 2,
                "d2h_bytes_per_step": n * 4, "steps": m},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if not a.no_cpu_baseline:
        import numpy as np

        import oracle
        w = wl.weight_fp32(n, k, cfg["w_seed"], "cpu").numpy()
        c, sc = oracle.quantize_block32(w)
        xb = x.cpu().numpy().view(np.uint16)
        passes, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < min(a.cpu_budget_s, 5.0):
            oracle.matvec(0, c, sc, None, xb)
            passes += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": round(passes * nbytes / el / 1e9, 3), "unit": UNIT,
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"the same GEMV x {passes} passes, fp64, {el:.1f} s"}
    print(json.dumps(line))
    return 0


def run_reference_single_gemv(a):
    """The reference arm on the single 2048 x 2048 GEMV: the oracle (fp64
    dequantize-then-matvec on the host cores), each step one call."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    from int4_quantized_decode_b200 import workloads as wl
    cfg = wl.GEMV_2048
    n, k = cfg["n"], cfg["k"]
    w = wl.weight_fp32(n, k, cfg["w_seed"], "cpu").numpy()
    c, sc = oracle.quantize_block32(w)
    xb = wl.act_fp16(k, cfg["x_seed"], "cpu").numpy().view(np.uint16)
    nbytes = c.nbytes + sc.nbytes
    for _ in range(a.warmup):
        oracle.matvec(0, c, sc, None, xb)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        oracle.matvec(0, c, sc, None, xb)
    el = time.perf_counter() - t0
    v = round(a.steps * nbytes / el / 1e9, 4)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(el * 1e3 / a.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"single {n}x{k} int8 block-32 GEMV, S=1; a step is one call",
                   "n": n, "k": k, "bytes_per_launch": nbytes},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": f"{a.steps} calls, fp64, {el:.2f} s"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
    return 0


def main(argv=None):
    a = parse_args(argv)
    if a.workload == SINGLE_GEMV:
        if a.impl == "reference":
            return run_reference_single_gemv(a)
        return run_single_gemv(a)
    if a.impl == "reference":
        return run_reference(a)
    return run_ours(a)


if __name__ == "__main__":
    sys.exit(main())
