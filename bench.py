#!/usr/bin/env python
"""Benchmark of the UltraSketchLLM sketch hot path on B200.

One step = one pass of the whole hot path over one 4096x4096 bf16 layer (the
layer with 0.1 % x20 outliers and calibration importance): usk_build (key, hash,
scatter-select, winner, scale, quantize), usk_gemv at batch 1 (rehash + gather
decode, product) and usk_gemm at batch 16 (decode into tcgen05 tiles).  The
headline value is usk_gemv GB/s (algorithmic bytes of one call / its average
launch duration); usk_build Gweights/s rides along.

Further timed regions, each K steps of its own calls, reported under their own
keys:
  small            256x1024 fp32 weights with lognormal importance: build, GEMV
                   at batch 1 with fp32 and bf16 x
  llama7b_set      the 7B layer set (4096x4096, 11008x4096, 4096x11008): build,
                   GEMV at batch 1 and 4, GEMM at batch 16 per shape, and the
                   layer-set totals
  mlp70b           28672x8192 and 8192x28672: build, GEMV at batch 1, GEMM at
                   batch 16, 32 and 64 (tcgen05)
  stack7b          the 32-layer 7B-shaped stack (224 linears): whole-model build,
                   one token = 224 batch-1 GEMVs back to back, and the same token
                   as dense bf16 torch.mm on the uncompressed weights
  absmaxmin        multi-row AbsMaxMin sketch (format 2, depth 2) of the layer
  colshared        column-shared projection (format 3) and the matrix-vs-hash A/B
                   at 28672x8192
  q4               4-bit codes (format 4)
  rates            format 1 at 2 and 8 hash slots per class
  row_block_rates  one slot count per 64-row block

Timing: every phase (one kind of call) is captured in CUDA graphs covering
exactly K steps.  Warm-up: W eager steps, then one untimed replay of every
graph.  Timed: the K-step region runs REPEATS times; before each repeat L2 is
flushed by reading a buffer twice its size, and a device spin keeps the GPU busy
while the host enqueues the region, so the CUDA events bracket device work
only.  A phase's time per call = median over the repeats of its event time / K
(min and max in the JSON).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl usk|reference]

For N > 1 run under torchrun (one rank per GPU): every rank runs the same work
on its own GPU (weak scaling, no data-path collective); each time is the max
over ranks.  `--impl reference` times the plain CPU oracle (all host cores) on
the headline workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gen  # noqa: E402

M = K = 4096
GEMV_BATCH = 1
GEMM_BATCH = 16
N_WCOPIES = 8      # 8 x 32 MiB of weights per build cycle  (> L2)
N_SKETCHES = 256   # 256 x 1 MiB of codes per decode cycle  (> L2)
AMM_DEPTH = 2      # hash rows of the format-2 (multi-row AbsMaxMin) measurement
AB_M, AB_K = 28672, 8192  # the matrix-vs-hash A/B shape (70B MLP up-projection)
AB_COPIES = 10            # 10 x 14 MiB of codes per format (> L2)
REPEATS = 5               # timed repeats of each K-step region (median reported)
GRAPH_LAUNCHES = 4096     # launches per captured CUDA graph at most
SPIN_CYCLES = 4_000_000   # device spin (~2 ms) that covers the host's enqueue of a region
FLUSH_BYTES = 256 << 20   # read before each timed repeat: twice the 126 MB L2
STACK_LAYERS = 32

METRIC = "usk_gemv GB/s & % roofline (4096x4096, batch 1); usk_build Gweights/s"
WORKLOAD = ("one 4096x4096 bf16 layer, Student-t(4) x 0.02 with 0.1% outliers x20, importance = mean |x| "
            "over 128 N(0,1) rows; usk_build + usk_gemv batch 1 + usk_gemm batch 16")

SMS = 148
SMEM_BYTES_PER_CLK = 128  # shared-memory load bandwidth per SM per clock
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


# ------------------------------------------------------------ algorithmic work

def build_bytes(m, k, wbytes=2, importance=True):
    """HBM bytes a build must move: W in, one code byte per 16 weights out,
    importance in, one binary16 scale per 64 rows out."""
    return wbytes * m * k + m * k // 16 + (4 * k if importance else 0) + 2 * (m // 64)


def gemv_bytes(m, k, batch, xbytes=2, code_bytes=None):
    """HBM bytes of a product: codes and scales in, x in, fp32 y out."""
    cb = m * k // 16 if code_bytes is None else code_bytes
    return cb + 2 * (m // 64) + xbytes * batch * k + 4 * batch * m


N_W = M * K
GEMV_BYTES = gemv_bytes(M, K, GEMV_BATCH)  # 1,073,280
GEMM_BYTES = gemv_bytes(M, K, GEMM_BATCH)
BUILD_BYTES = build_bytes(M, K)
GEMM_FLOPS = 2 * N_W * GEMM_BATCH


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


class Roof:
    """Roofline lines from algorithmic work and the measured peaks.

    Builds are HBM-bound.  Sketch-decode products rebuild every weight from a
    shared-memory gather of its bucket code: at least `gathers` bytes through the
    128 B/clk/SM shared-memory pipe, which binds before HBM (the codes are 1/16
    byte per weight); a tcgen05 product is also held against the dense bf16
    tensor time.  `achieved` is algorithmic HBM bytes / time; `peak` is the same
    bytes over the time at the binding bound."""

    def __init__(self, peaks):
        self.hbm = peaks["hbm_gbs"] * 1e9
        self.clk = peaks.get("sm_max_mhz", 1965.0) * 1e6
        self.smem = SMS * SMEM_BYTES_PER_CLK * self.clk
        self.tensor = peaks["bf16_tflops"] * 1e12
        self.src = peaks["source"]

    def _line(self, bound, achieved, peak, unit, traffic):
        return {"bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 3), "unit": unit,
                "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": self.src}

    def hbm_line(self, nbytes, t, traffic=None):
        return self._line("hbm", nbytes / t / 1e9, self.hbm / 1e9, "GB/s", traffic)

    def gather_line(self, nbytes, gathers, t, traffic=None, flops=None):
        t_bound = max(nbytes / self.hbm, gathers / self.smem, (flops or 0) / self.tensor)
        out = self._line("alu", nbytes / t / 1e9, nbytes / t_bound / 1e9, "GB/s", traffic)
        out["binding"] = "shared-memory gather (1 B/weight per hash row at 128 B/clk/SM)"
        if flops:
            out["tensor_tflops"] = round(flops / t / 1e12, 3)
            if flops / self.tensor >= gathers / self.smem:
                out["binding"] = "dense bf16 tensor time"
        out["bound_us"] = round(t_bound * 1e6, 3)
        return out


def rooflines(peaks, t_build_s, t_gemv_s, t_gemm_s, traffic, depth=1, build_bytes_=None):
    """Rooflines of the headline layer's three calls (depth = hash rows gathered
    per weight)."""
    r = Roof(peaks)
    out = {"usk_build": r.hbm_line(BUILD_BYTES if build_bytes_ is None else build_bytes_, t_build_s,
                                   traffic.get("usk_build")),
           "usk_gemv": r.gather_line(GEMV_BYTES, depth * N_W, t_gemv_s, traffic.get("usk_gemv")),
           "usk_gemm": r.gather_line(GEMM_BYTES, depth * N_W, t_gemm_s, traffic.get("usk_gemm"), GEMM_FLOPS)}
    out["usk_gemv"]["binding"] = "shared-memory gather (%d B/weight at 128 B/clk/SM)" % depth
    return out


def source_sha(name):
    p = os.path.join(ROOT, "sub_bit_weight_usk_b200", "csrc", name)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch from the committed ncu summary, only while the
    kernel source still matches the one the counters were taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    out = {}
    if not os.path.exists(p):
        return out
    with open(p) as f:
        d = json.load(f)
    for kern, rec in d.items():
        try:
            if rec.get("source_sha") == source_sha(rec["source"]):
                out[kern] = rec["dram_bytes_per_launch"]
        except (KeyError, OSError):
            pass
    return out


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed regions."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # samples under load: the GPU draws well above idle power
        loaded = [s for s, p in zip(sm, power) if p > 0.3 * max(power)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len(loaded), "power_w_max": max(power)}


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity for one
    process).  The only collective of the benchmark; NCCL on the GPUs, gloo in
    the CPU tests."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def aggregate(world, per_rank_gemv_s, per_rank_build_s, per_rank_step_s):
    """Whole-job numbers from per-rank timings (each list has one entry per rank):
    every rank did the same work, the time is the slowest rank's."""
    t_gemv = max(per_rank_gemv_s)
    t_build = max(per_rank_build_s)
    t_step = max(per_rank_step_s)
    return {
        "gemv_gbs": world * GEMV_BYTES / t_gemv / 1e9,
        "build_gweights_s": world * N_W / t_build / 1e9,
        "ms_per_step": t_step * 1e3,
    }


def steps_per_graph(steps, launches_per_step):
    """Steps captured per CUDA graph: as many as fit GRAPH_LAUNCHES launches."""
    return max(1, min(steps, GRAPH_LAUNCHES // max(1, launches_per_step)))


def graph_chunks(steps, launches_per_step):
    """(first step, steps) of each graph covering exactly `steps` steps."""
    per = steps_per_graph(steps, launches_per_step)
    return [(s0, min(per, steps - s0)) for s0 in range(0, steps, per)]


def cpu_info():
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except AttributeError:
        avail = os.cpu_count()
    return {"cpu_model": model, "nproc": avail}


# ------------------------------------------------------------------ CPU oracle

def row_block_workload(cfg, usk):
    """The layer with one lognormal gain per 64-row block (rows of unequal
    output energy) and its per-row-block rates: importance of a block = E[a^2]
    of its outputs over the calibration rows, slots from usk_plan_slots at 0.5
    bit/weight.  Returns (W bf16 bits, slot list)."""
    RB = M // 64
    Wv = gen.scale_row_blocks(cfg["W"], gen.row_block_gains(RB, cfg["seed"]))
    a = gen.bf16_bits_to_f32(cfg["x"]) @ gen.bf16_bits_to_f32(Wv).T  # calibration outputs [rows, M]
    imp = (a.astype(np.float64) ** 2).reshape(a.shape[0], RB, 64).mean(axis=(0, 2))
    return Wv, usk.usk_plan_slots([64 * K] * RB, imp.tolist(), 0.5)


def _timed(fn, budget_s, max_reps=50):
    """Mean seconds of fn() over repetitions until about budget_s (at least one)."""
    reps, total = 0, 0.0
    while reps == 0 or (total < budget_s and reps < max_reps):
        t0 = time.perf_counter()
        fn()
        total += time.perf_counter() - t0
        reps += 1
    return total / reps, reps


def cpu_oracle_baseline(extra=None, budget_s=3.0):
    """The oracle as it stands, timed on this host in its two modes: one thread
    (the plain sequential oracle) and all cores (row blocks over OpenMP threads,
    identical results).  The headline layer's GEMV (whole layer, batch 1) and
    build, then the build and GEMV of each (name, W bf16 bits, x) in `extra`
    (sampled rows for the single-thread GEMV of tall matrices, scaled to a full
    call)."""
    import oracle
    cores = oracle.threads(0)
    cfg = gen.layer(1)
    Wl, imp, x, seed = cfg["W"], cfg["importance"], cfg["x"], cfg["seed"]
    o = oracle.build_sketch_mt(Wl, imp, seed)
    res = {"cores_all": cores}
    t_b1, _ = _timed(lambda: oracle.build_sketch(Wl, imp, seed), budget_s / 3, 3)
    t_bn, _ = _timed(lambda: oracle.build_sketch_mt(Wl, imp, seed), budget_s / 3, 10)
    t_g1, r1 = _timed(lambda: oracle.gemv_f64(o["codes"], o["scales"], M, K, x, seed), budget_s, 20)
    t_gn, rn = _timed(lambda: oracle.gemv_f64_mt(o["codes"], o["scales"], M, K, x, seed), budget_s, 50)
    res["layer"] = {"build_s": {"1": t_b1, "all": t_bn}, "gemv_s": {"1": t_g1, "all": t_gn},
                    "gemv_reps": {"1": r1, "all": rn}}
    for name, W, xx, imp_e in (extra or []):
        m, k = W.shape
        ob = oracle.build_sketch_mt(W, imp_e, 7)
        t_b1, _ = _timed(lambda: oracle.build_sketch(W, imp_e, 7), 0.0, 1)
        t_bn, _ = _timed(lambda: oracle.build_sketch_mt(W, imp_e, 7), 0.0, 1)
        nrows = min(m, max(64, int(m * min(1.0, 2.0 / max(1e-9, m * k * 25e-9)))))  # ~2 s of rows
        rows = np.linspace(0, m - 1, nrows).astype(np.int64)
        t_r, _ = _timed(lambda: oracle.gemv_f64(ob["codes"], ob["scales"], m, k, xx, 7, rows=rows), 0.0, 1)
        t_gn, _ = _timed(lambda: oracle.gemv_f64_mt(ob["codes"], ob["scales"], m, k, xx, 7), 0.0, 1)
        res[name] = {"build_s": {"1": t_b1, "all": t_bn}, "gemv_s": {"1": t_r * m / nrows, "all": t_gn},
                     "gemv_rows_sampled_1": int(nrows)}
    return res


def run_reference(args):
    """The base contract's reference arm: the oracle as it stands on the host
    cores (all of them: row blocks over OpenMP threads, the same result as the
    sequential oracle), one whole-layer float64 GEMV per step, same metric and
    workload as the GPU arm."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    cfg = gen.layer(1)
    o = oracle.build_sketch_mt(cfg["W"], cfg["importance"], cfg["seed"])
    cores = oracle.threads(0)
    for _ in range(args.warmup):
        oracle.gemv_f64_mt(o["codes"], o["scales"], M, K, cfg["x"], cfg["seed"])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gemv_f64_mt(o["codes"], o["scales"], M, K, cfg["x"], cfg["seed"])
    t = (time.perf_counter() - t0) / max(args.steps, 1)
    value = GEMV_BYTES / t / 1e9
    info = cpu_info()
    sample = ("one whole-layer float64 oracle GEMV (4096x4096, batch 1) per step, rows over %d host threads "
              "(%s)" % (cores, info["cpu_model"]))
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "batch": GEMV_BATCH},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "nproc": info["nproc"], "cpu_model": info["cpu_model"]},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

class Bench:
    """Captures phases (one kind of call each, K steps) into CUDA graphs and
    times them; see the module docstring for the protocol."""

    def __init__(self, torch, dev, steps, warmup, world, status):
        self.torch = torch
        self.dev = dev
        self.steps = steps
        self.warmup = warmup
        self.world = world
        self.status = status
        self.stream = torch.cuda.Stream(device=dev)
        self.stream.wait_stream(torch.cuda.current_stream())
        self.flush_buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.flush_buf.fill_(1.0)
        self.launches = 0

    def _check(self, where):
        self.torch.cuda.synchronize()
        v = int(self.status.item())
        if v != 0:
            raise SystemExit("device status flags %#x %s" % (v, where))

    def prepare(self, phases):
        """phases: list of (name, fn(step), launches per step[, counted]).  Eager
        warm-up, capture, one untimed replay of every graph.  `counted` False:
        launches that are not this library's (left out of the launch count)."""
        phases = [p if len(p) == 4 else (*p, True) for p in phases]
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for i in range(self.warmup):
                for _, fn, _, _ in phases:
                    fn(i)
        self._check("during warm-up")
        region = []
        for name, fn, lps, counted in phases:
            graphs = []
            for s0, n in graph_chunks(self.steps, lps):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=self.stream):
                    for j in range(n):
                        fn(self.warmup + s0 + j)
                graphs.append(g)
            region.append((name, graphs, lps if counted else 0))
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            for _, graphs, _ in region:
                for g in graphs:
                    g.replay()
        self._check("in the graph warm-up replay")
        return region

    def soak(self, region, seconds):
        """Untimed replays (clock sampling under load before the timed repeats)."""
        torch = self.torch
        t_end = time.perf_counter() + seconds
        with torch.cuda.stream(self.stream):
            while time.perf_counter() < t_end:
                for _, graphs, _ in region:
                    for g in graphs:
                        g.replay()
                self.stream.synchronize()

    def time(self, region):
        """{phase: [seconds per call in each repeat]}."""
        import torch.distributed as dist
        torch = self.torch
        out = {name: [] for name, _, _ in region}
        torch.cuda.nvtx.range_push("timed")  # lets a profiler keep to the timed launches
        for _ in range(REPEATS):
            if self.world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            with torch.cuda.stream(self.stream):
                self.flush_buf.sum()  # evict what the previous repeat left in L2
                torch.cuda._sleep(SPIN_CYCLES)
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(region) + 1)]
                ev[0].record(self.stream)
                for k, (_, graphs, _) in enumerate(region):
                    for g in graphs:
                        g.replay()
                    ev[k + 1].record(self.stream)
            ev[-1].synchronize()
            torch.cuda.synchronize()
            if self.world > 1:
                dist.barrier()
            for k, (name, _, _) in enumerate(region):
                out[name].append(ev[k].elapsed_time(ev[k + 1]) * 1e-3 / max(self.steps, 1))
        torch.cuda.nvtx.range_pop()
        for _, _, lps in region:
            self.launches += REPEATS * self.steps * lps
        self._check("in the timed region")
        return out


def _med(v):
    return statistics.median(v)


def _us(v):
    return round(v * 1e6, 3)


def _spread(times):
    return {k: {"min_us": _us(min(v)), "max_us": _us(max(v))} for k, v in times.items()}


def run_usk(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import sub_bit_weight_usk_b200 as usk

    dev = torch.device("cuda", local)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    B = Bench(torch, dev, args.steps, args.warmup, world, status)

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    def copies(sk, n):
        return [usk.Sketch(sk.M, sk.K, sk.seed, sk.codes.clone(), sk.scales.clone(), sk.version, sk.depth,
                           sk.slots, sk.rates) for _ in range(n)]

    regions = {}   # key -> (region, report fn(times) -> dict)
    order = []

    def add(key, phases, report):
        regions[key] = (B.prepare(phases), report)
        order.append(key)

    # ---------------------------------------------------------- headline layer
    cfg = gen.layer(GEMM_BATCH)
    W = to_dev(cfg["W"])
    imp = to_dev(cfg["importance"])
    x16 = to_dev(cfg["x"])
    x1 = x16[:1].contiguous()
    x4 = x16[:4].contiguous()
    seed = cfg["seed"]
    Ws = [W.clone() for _ in range(N_WCOPIES)]
    sks = copies(usk.usk_build(W, imp, seed), N_SKETCHES)
    y1 = torch.empty((1, M), device=dev)
    y4 = torch.empty((4, M), device=dev)
    y16 = torch.empty((GEMM_BATCH, M), device=dev)
    ws_lay = torch.zeros(usk.usk_gemv_multi_ws_bytes([sks[0]], 1), dtype=torch.uint8, device=dev)

    def lay_build(i):
        b = sks[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status)

    # consecutive decode calls launch as programmatic dependents of the previous
    # one (their code prefetch -- and for usk_gemm the set-up and decoding into
    # tensor memory -- overlaps the previous call's tail)
    add("layer", [("usk_build", lay_build, 1),
                  ("usk_gemv", lambda i: usk.usk_gemv(sks[(i + 128) % N_SKETCHES], x1, y=y1, pdl=True), 1),
                  ("usk_gemv_b4", lambda i: usk.usk_gemv(sks[(i + 160) % N_SKETCHES], x4, y=y4, pdl=True), 1),
                  ("usk_gemm", lambda i: usk.usk_gemm(sks[(i + 64) % N_SKETCHES], x16, y=y16, status=status,
                                                      pdl=True), 1),
                  ("usk_gemv_multi", lambda i: usk.usk_gemv_multi([sks[(i + 192) % N_SKETCHES]], [x1], [y1],
                                                                  ws=ws_lay, pdl=True), 1)],
        None)

    # ---------------------------------------------------------- small (fp32 weights)
    sm = gen.small("f32")
    SM_COPIES = 128
    Wsm = to_dev(sm["W"])
    Wsms = [Wsm.clone() for _ in range(SM_COPIES)]
    impsm = to_dev(sm["importance"])
    xsm32 = to_dev(sm["x"])
    xsm16 = to_dev(gen.small("bf16")["x"])
    sksm = copies(usk.usk_build(Wsm, impsm, sm["seed"]), 256)
    ysm = torch.empty((1, 256), device=dev)

    def sm_build(i):
        b = sksm[i % 256]
        usk.usk_build(Wsms[i % SM_COPIES], impsm, sm["seed"], codes=b.codes, scales=b.scales, status=status)

    add("small", [("usk_build", sm_build, 1),
                  ("usk_gemv_f32x", lambda i: usk.usk_gemv(sksm[i % 256], xsm32, y=ysm, pdl=True), 1),
                  ("usk_gemv_bf16x", lambda i: usk.usk_gemv(sksm[(i + 128) % 256], xsm16, y=ysm, pdl=True), 1)],
        None)

    # ---------------------------------------------------------- the 32-layer stack (configs 3 and 5)
    # device-drawn N(0, 0.02^2) bf16 weights, one seed per linear: the values do
    # not change the work, and 6.48 G weights drawn on the host would take minutes
    stack = []  # (layer, name, W, sketch, x, y)
    for layer in range(STACK_LAYERS):
        for name in gen.LLAMA7B_ORDER:
            m, k = gen.LLAMA7B_SHAPES[name]
            s_ = gen.stack7b_seed(layer, name)
            Wl = gen.device_weights_normal(m, k, s_, 0.02, dev)
            skl = usk.usk_build(Wl, None, s_)
            xl = to_dev(gen.activations(16, k, s_, "bf16"))
            stack.append({"layer": layer, "name": name, "W": Wl, "sk": skl, "x1": xl[:1].contiguous(),
                          "x4": xl[:4].contiguous(), "x16": xl, "y": torch.empty((16, m), device=dev),
                          "ybf": torch.empty((1, m), dtype=torch.bfloat16, device=dev), "seed": s_})
    torch.cuda.synchronize()

    def stack_build(i):
        for e in stack:
            usk.usk_build(e["W"], None, e["seed"], codes=e["sk"].codes, scales=e["sk"].scales, status=status)

    def stack_token(i):
        for e in stack:
            usk.usk_gemv(e["sk"], e["x1"], y=e["y"][:1], pdl=True)

    def stack_dense(i):
        for e in stack:
            torch.mm(e["x1"], e["W"].t(), out=e["ybf"])

    # the same token with usk_gemv_multi: per layer one launch each for the
    # products a transformer's data flow leaves independent -- q, k, v (one
    # input), o, gate and up (one input), down -- 128 launches per token, all
    # sharing one workspace in stream order
    groups = []
    for layer in range(STACK_LAYERS):
        es = [e for e in stack if e["layer"] == layer]
        by = {e["name"]: e for e in es}
        for names in (("q", "k", "v"), ("o",), ("gate", "up"), ("down",)):
            groups.append([by[nm] for nm in names])
    ws_tok = torch.zeros(max(usk.usk_gemv_multi_ws_bytes([e["sk"] for e in g_], 1) for g_ in groups),
                         dtype=torch.uint8, device=dev)
    calls = [(usk.MultiCall([e["sk"] for e in g_], [e["x1"] for e in g_], [e["y"][:1] for e in g_]), g_)
             for g_ in groups]

    def stack_token_multi(i):
        for c, g_ in calls:
            usk.usk_gemv_multi([e["sk"] for e in g_], [e["x1"] for e in g_], [e["y"][:1] for e in g_], ws=ws_tok,
                               pdl=True, call=c)

    # the same token with the products a transformer's data flow leaves
    # independent running concurrently on graph branches (q | k | v, then o,
    # then gate | up, then down): usk_gemv on forked streams, joined by events
    branch = [torch.cuda.Stream(device=dev) for _ in range(2)]

    def stack_token_concurrent(i):
        main = torch.cuda.current_stream()
        for g_ in groups:
            if len(g_) == 1:
                usk.usk_gemv(g_[0]["sk"], g_[0]["x1"], y=g_[0]["y"][:1])
                continue
            ev = torch.cuda.Event()
            ev.record(main)
            for bs, e in zip(branch, g_[1:]):
                bs.wait_event(ev)
                with torch.cuda.stream(bs):
                    usk.usk_gemv(e["sk"], e["x1"], y=e["y"][:1])
            usk.usk_gemv(g_[0]["sk"], g_[0]["x1"], y=g_[0]["y"][:1])
            for bs in branch[:len(g_) - 1]:
                done = torch.cuda.Event()
                done.record(bs)
                main.wait_event(done)

    n_lin = len(stack)
    add("stack7b", [("model_build", stack_build, n_lin), ("token_decode", stack_token, n_lin),
                    ("token_decode_grouped", stack_token_multi, len(groups)),
                    ("token_decode_concurrent", stack_token_concurrent, n_lin),
                    ("token_dense_bf16_torch", stack_dense, n_lin, False)], None)

    # 7B layer set: per shape, cycling over the stack's linears of that shape
    by_shape = {"4096x4096": [e for e in stack if e["name"] in ("q", "k", "v", "o")],
                "11008x4096": [e for e in stack if e["name"] in ("gate", "up")],
                "4096x11008": [e for e in stack if e["name"] == "down"]}
    set_phases = []
    for shp, lst in by_shape.items():
        n = len(lst)

        def b_(i, lst=lst, n=n):
            e = lst[i % n]
            usk.usk_build(e["W"], None, e["seed"], codes=e["sk"].codes, scales=e["sk"].scales, status=status)

        def g1(i, lst=lst, n=n):
            e = lst[(i + n // 2) % n]
            usk.usk_gemv(e["sk"], e["x1"], y=e["y"][:1], pdl=True)

        def g4(i, lst=lst, n=n):
            e = lst[(i + n // 4) % n]
            usk.usk_gemv(e["sk"], e["x4"], y=e["y"][:4], pdl=True)

        def gm(i, lst=lst, n=n):
            e = lst[(i + 3 * n // 4) % n]
            usk.usk_gemm(e["sk"], e["x16"], y=e["y"], status=status, pdl=True)

        ws_s = torch.zeros(max(16, usk.usk_gemv_multi_ws_bytes([lst[0]["sk"]], 4)), dtype=torch.uint8, device=dev)

        def gm1(i, lst=lst, n=n, ws_s=ws_s):
            e = lst[(i + n // 2) % n]
            usk.usk_gemv_multi([e["sk"]], [e["x1"]], [e["y"][:1]], ws=ws_s, pdl=True)

        def gm4(i, lst=lst, n=n, ws_s=ws_s):
            e = lst[(i + n // 4) % n]
            usk.usk_gemv_multi([e["sk"]], [e["x4"]], [e["y"][:4]], ws=ws_s, pdl=True)

        set_phases += [(shp + "/usk_build", b_, 1), (shp + "/usk_gemv_b1", g1, 1), (shp + "/usk_gemv_b4", g4, 1),
                       (shp + "/usk_gemm_b16", gm, 1), (shp + "/usk_gemv_multi_b1", gm1, 1),
                       (shp + "/usk_gemv_multi_b4", gm4, 1)]
    add("llama7b_set", set_phases, None)

    # ---------------------------------------------------------- 70B MLP shapes
    mlp = {}
    for name, (m, k) in gen.MLP70B_SHAPES.items():
        s_ = 3 if name == "up" else 103
        Wm = gen.device_weights_normal(m, k, s_, 0.02, dev)
        skm = usk.usk_build(Wm, None, s_)
        xm = to_dev(gen.activations(64, k, s_, "bf16"))
        mlp[name] = {"W": Wm, "sks": copies(skm, AB_COPIES), "seed": s_, "x": xm,
                     "y": torch.empty((64, m), device=dev), "M": m, "K": k}
    mlp_phases = []
    for name, e in mlp.items():
        shp = "%dx%d" % (e["M"], e["K"])

        def mb(i, e=e):
            b = e["sks"][i % AB_COPIES]
            usk.usk_build(e["W"], None, e["seed"], codes=b.codes, scales=b.scales, status=status)

        mlp_phases.append((shp + "/usk_build", mb, 1))
        xs = {1: e["x"][:1].contiguous(), 16: e["x"][:16].contiguous(), 32: e["x"][:32].contiguous(), 64: e["x"]}

        def mg1(i, e=e, xs=xs):
            usk.usk_gemv(e["sks"][(i + 5) % AB_COPIES], xs[1], y=e["y"][:1], pdl=True)

        mlp_phases.append((shp + "/usk_gemv_b1", mg1, 1))
        ws_m = torch.zeros(max(16, usk.usk_gemv_multi_ws_bytes([e["sks"][0]], 1)), dtype=torch.uint8, device=dev)

        def mgm1(i, e=e, xs=xs, ws_m=ws_m):
            usk.usk_gemv_multi([e["sks"][(i + 7) % AB_COPIES]], [xs[1]], [e["y"][:1]], ws=ws_m, pdl=True)

        mlp_phases.append((shp + "/usk_gemv_multi_b1", mgm1, 1))
        for bb in (16, 32, 64):
            def mgm(i, e=e, xs=xs, bb=bb):
                usk.usk_gemm(e["sks"][(i + bb) % AB_COPIES], xs[bb], y=e["y"][:bb], status=status, pdl=True)
            mlp_phases.append((shp + "/usk_gemm_b%d" % bb, mgm, 1))
    add("mlp70b", mlp_phases, None)

    # ---------------------------------------------------------- format 2 (multi-row AbsMaxMin)
    amm = usk.FORMAT_ABSMAXMIN
    sks2 = copies(usk.usk_build(W, None, seed, version=amm, depth=AMM_DEPTH), N_SKETCHES)

    def amm_build(i):
        b = sks2[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], None, seed, codes=b.codes, scales=b.scales, status=status, version=amm,
                      depth=AMM_DEPTH)

    add("absmaxmin", [("usk_build", amm_build, 1),
                      ("usk_gemv", lambda i: usk.usk_gemv(sks2[(i + 128) % N_SKETCHES], x1, y=y1, pdl=True), 1),
                      ("usk_gemm", lambda i: usk.usk_gemm(sks2[(i + 64) % N_SKETCHES], x16, y=y16, status=status,
                                                                          pdl=True),
                       1)], None)

    # ---------------------------------------------------------- format 3 and the matrix-vs-hash A/B
    cs = usk.FORMAT_COLSHARED
    sks3 = copies(usk.usk_build(W, None, seed, version=cs), N_SKETCHES)

    def cs_build(i):
        b = sks3[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], None, seed, codes=b.codes, scales=b.scales, status=status, version=cs)

    up = mlp["up"]
    abm = copies(usk.usk_build(up["W"], None, up["seed"], version=cs), AB_COPIES)
    xab = up["x"][:1].contiguous()
    add("colshared", [("usk_build", cs_build, 1),
                      ("usk_gemv", lambda i: usk.usk_gemv(sks3[(i + 128) % N_SKETCHES], x1, y=y1, pdl=True), 1),
                      ("ab_hash_gemv", lambda i: usk.usk_gemv(up["sks"][i % AB_COPIES], xab, y=up["y"][:1],
                                                              pdl=True), 1),
                      ("ab_matrix_gemv", lambda i: usk.usk_gemv(abm[i % AB_COPIES], xab, y=up["y"][:1], pdl=True),
                       1)], None)

    # ---------------------------------------------------------- format 4 (4-bit codes)
    q4 = usk.FORMAT_Q4
    sks4 = copies(usk.usk_build(W, imp, seed, version=q4), N_SKETCHES)

    def q4_build(i):
        b = sks4[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status, version=q4)

    add("q4", [("usk_build", q4_build, 1),
               ("usk_gemv", lambda i: usk.usk_gemv(sks4[(i + 128) % N_SKETCHES], x1, y=y1, pdl=True), 1),
               ("usk_gemm", lambda i: usk.usk_gemm(sks4[(i + 64) % N_SKETCHES], x16, y=y16, status=status,
                                                                   pdl=True), 1)],
        None)

    # ---------------------------------------------------------- format 1 at 2 and 8 slots
    rate_sk = {nsl: copies(usk.usk_build(W, imp, seed, slots=nsl), N_SKETCHES) for nsl in (2, 8)}
    rate_phases = []
    for nsl in (2, 8):
        def rb_(i, nsl=nsl):
            b = rate_sk[nsl][i % N_SKETCHES]
            usk.usk_build(Ws[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status, slots=nsl)

        def rg_(i, nsl=nsl):
            usk.usk_gemv(rate_sk[nsl][(i + 128) % N_SKETCHES], x1, y=y1, pdl=True)
        rate_phases += [("slots_%d/usk_build" % nsl, rb_, 1), ("slots_%d/usk_gemv" % nsl, rg_, 1)]
    add("rates", rate_phases, None)

    # ---------------------------------------------------------- per-row-block rates
    Wv_h, vr_slots = row_block_workload(cfg, usk)
    Wv = to_dev(Wv_h)
    Wvs = [Wv.clone() for _ in range(N_WCOPIES)]
    rmap = usk.usk_rate_map(M, K, vr_slots, dev)
    sksv = copies(usk.usk_build(Wv, imp, seed, rates=rmap), N_SKETCHES)

    def vr_build(i):
        b = sksv[i % N_SKETCHES]
        usk.usk_build(Wvs[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status, rates=rmap)

    add("row_block_rates", [("usk_build", vr_build, 1),
                            ("usk_gemv", lambda i: usk.usk_gemv(sksv[(i + 128) % N_SKETCHES], x1, y=y1, pdl=True),
                             1),
                            ("usk_gemm", lambda i: usk.usk_gemm(sksv[(i + 64) % N_SKETCHES], x16, y=y16,
                                                                status=status, pdl=True), 1)], None)

    # ---------------------------------------------------------- timed regions
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    B.soak(regions["layer"][0], 0.5)
    times = {}
    for key in order:
        times[key] = B.time(regions[key][0])
    sampler.stop()

    # ---------------------------------------------------------- end to end
    # (a) the Python binding: x from pinned host memory, y read back, per call
    xh = x1.cpu().pin_memory()
    yh = torch.empty((GEMV_BATCH, M), dtype=torch.float32).pin_memory()
    n_e2e = max(50, min(2000, args.steps))
    for i in range(5):
        usk.usk_gemv(sks[i], xh.to(dev, non_blocking=True), y=y1)
        yh.copy_(y1, non_blocking=True)
        torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(n_e2e):
        xd = xh.to(dev, non_blocking=True)
        usk.usk_gemv(sks[i % N_SKETCHES], xd, y=y1)
        yh.copy_(y1, non_blocking=True)
        torch.cuda.current_stream().synchronize()
    t_e2e_py = (time.perf_counter() - t0) / n_e2e
    # (b) the C ABI alone: the in-tree C driver (usk_gemv with cudaMemcpyAsync of x and y on its stream)
    c_e2e = run_c_driver(local, n_e2e)

    # ---------------------------------------------------------- max over ranks
    flat_keys = [(key, name, r) for key in order for name in times[key] for r in range(REPEATS)]
    flat = [times[key][name][r] for key, name, r in flat_keys] + [t_e2e_py, c_e2e["e2e_s"] if c_e2e else 0.0]
    flat = max_over_ranks(flat, device=dev)
    for (key, name, r), v in zip(flat_keys, flat):
        times[key][name][r] = v
    t_e2e_py, t_e2e_c = flat[-2], flat[-1]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_json(stack, mlp, sm)

    # release the graphs before the process group
    for key in order:
        regions[key] = None
    torch.cuda.synchronize()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = load_peaks()
    R = Roof(peaks)
    tr = load_traffic()
    med = {key: {name: _med(v) for name, v in times[key].items()} for key in order}

    L = med["layer"]
    t_build, t_gemv, t_gemv4, t_gemm = L["usk_build"], L["usk_gemv"], L["usk_gemv_b4"], L["usk_gemm"]
    t_step = t_build + t_gemv + t_gemm
    agg = aggregate(world, [t_gemv], [t_build], [t_step])
    rl = rooflines(peaks, t_build, t_gemv, t_gemm, tr)
    rl["usk_gemv_b4"] = R.gather_line(gemv_bytes(M, K, 4), N_W, t_gemv4)
    rl["usk_gemv_multi"] = R.gather_line(GEMV_BYTES, N_W, L["usk_gemv_multi"], tr.get("multi_usk_gemv"))
    e2e_bytes_c = (c_e2e or {}).get("h2d_bytes", 2 * K) + (c_e2e or {}).get("d2h_bytes", 4 * M)
    clocks = sampler.summary()
    info = cpu_info()

    line = {
        "metric": METRIC,
        "value": round(agg["gemv_gbs"], 3),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_step * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "gemv_batch": GEMV_BATCH, "gemm_batch": GEMM_BATCH,
                   "timing": "each call kind captured in CUDA graphs covering exactly K steps; warm-up = W eager "
                             "steps + one untimed replay of every graph; the K-step region timed %d times with "
                             "CUDA events on the replay stream (a device spin covers the host's enqueue), median "
                             "per call reported, min/max under 'spread'" % REPEATS,
                   "gemv_launch": "programmatic dependent launch (USK_GEMV_PDL, USK_GEMM_PDL) between consecutive "
                                  "GEMV and GEMM calls",
                   "l2": "L2 flushed before each timed repeat (a %d MiB read); within a repeat builds cycle over %d "
                         "weight copies (%d MiB) and the decodes touch %d distinct sketch copies (1 MiB each), so "
                         "every decode reads its codes from HBM"
                         % (FLUSH_BYTES >> 20, N_WCOPIES, N_WCOPIES * 32, min(args.steps, N_SKETCHES)),
                   "parallelism": "replicas" if world > 1 else "single"},
        "usk_build_gweights_per_s": round(agg["build_gweights_s"], 3),
        "kernel_us": {"usk_build": _us(t_build), "usk_gemv": _us(t_gemv), "usk_gemv_b4": _us(t_gemv4),
                      "usk_gemm": _us(t_gemm), "usk_gemv_multi": _us(L["usk_gemv_multi"])},
        "spread": _spread(times["layer"]),
        "roofline": rl["usk_gemv"],
        "rooflines": rl,
        "clocks": clocks,
        "e2e": {"value": round(world * GEMV_BYTES / t_e2e_c / 1e9, 4) if c_e2e else
                round(world * GEMV_BYTES / t_e2e_py / 1e9, 4),
                "unit": "GB/s", "h2d_bytes_per_step": int(2 * K * GEMV_BATCH),
                "d2h_bytes_per_step": int(4 * M * GEMV_BATCH),
                "call": ("usk_gemv through the C ABI (in-tree C driver): cudaMemcpyAsync of x from pinned host "
                         "memory, usk_gemv, cudaMemcpyAsync of y back, stream synchronize, per call"
                         if c_e2e else "usk_gemv via the Python binding (C driver unavailable)"),
                "us_per_call": _us(t_e2e_c if c_e2e else t_e2e_py),
                "c_abi": c_e2e,
                "python_binding": {"value": round(world * GEMV_BYTES / t_e2e_py / 1e9, 4), "unit": "GB/s",
                                   "us_per_call": _us(t_e2e_py),
                                   "call": "usk_gemv via the Python binding, x from pinned host memory, y read "
                                           "back, per call"},
                "bytes_per_call": e2e_bytes_c},
        "gpu_launches": B.launches,
        "gpu_launches_note": "libusk kernel launches in all timed regions (%d repeats each); the stack7b dense "
                             "torch.mm phase is not counted" % REPEATS,
        "cpu_baseline": cpu,
        "host": info,
    }
    line.update(region_reports(med, times, R, tr, world, peaks, rmap))
    print(json.dumps(line), flush=True)
    return 0


def region_reports(med, times, R, tr, world, peaks, rmap):
    """JSON objects of the regions other than the headline."""
    out = {}
    # small: 256x1024 fp32 W with importance
    s = med["small"]
    sm_m, sm_k = 256, 1024
    out["small"] = {
        "workload": "256x1024 fp32 N(0, 0.02^2) weights, lognormal(0, 1) per-column importance, x ~ N(0,1) batch 1",
        "kernel_us": {k: _us(v) for k, v in s.items()},
        "usk_build_gweights_per_s": round(world * sm_m * sm_k / s["usk_build"] / 1e9, 3),
        "rooflines": {"usk_build": R.hbm_line(build_bytes(sm_m, sm_k, 4), s["usk_build"]),
                      "usk_gemv_f32x": R.gather_line(gemv_bytes(sm_m, sm_k, 1, 4), sm_m * sm_k, s["usk_gemv_f32x"]),
                      "usk_gemv_bf16x": R.gather_line(gemv_bytes(sm_m, sm_k, 1, 2), sm_m * sm_k,
                                                      s["usk_gemv_bf16x"])},
        "spread": _spread(times["small"]),
        "note": "262 K weights: every call is launch- and latency-bound",
    }
    # 7B layer set
    st = med["llama7b_set"]
    shapes = {"4096x4096": (4096, 4096, 4), "11008x4096": (11008, 4096, 2), "4096x11008": (4096, 11008, 1)}
    per_shape, totals = {}, {"usk_build": 0.0, "usk_gemv_b1": 0.0, "usk_gemv_b4": 0.0, "usk_gemm_b16": 0.0,
                             "usk_gemv_multi_b1": 0.0, "usk_gemv_multi_b4": 0.0}
    n_set = 0
    for shp, (m, k, cnt) in shapes.items():
        d = {c: st[shp + "/" + c] for c in totals}
        for c in totals:
            totals[c] += cnt * d[c]
        n_set += cnt * m * k
        per_shape[shp] = {
            "count_in_set": cnt, "kernel_us": {c: _us(v) for c, v in d.items()},
            "rooflines": {"usk_build": R.hbm_line(build_bytes(m, k, 2, False), d["usk_build"]),
                          "usk_gemv_b1": R.gather_line(gemv_bytes(m, k, 1), m * k, d["usk_gemv_b1"]),
                          "usk_gemv_b4": R.gather_line(gemv_bytes(m, k, 4), m * k, d["usk_gemv_b4"]),
                          "usk_gemm_b16": R.gather_line(gemv_bytes(m, k, 16), m * k, d["usk_gemm_b16"],
                                                        flops=2 * m * k * 16),
                          "usk_gemv_multi_b1": R.gather_line(gemv_bytes(m, k, 1), m * k, d["usk_gemv_multi_b1"]),
                          "usk_gemv_multi_b4": R.gather_line(gemv_bytes(m, k, 4), m * k, d["usk_gemv_multi_b4"])}}
    out["llama7b_set"] = {
        "workload": "Llama-7B-shaped layer set: q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008, bf16 "
                    "N(0, 0.02^2) (device-drawn), no importance; each shape's calls cycle over the 32 layers' "
                    "linears of that shape (> L2)",
        "per_shape": per_shape,
        "layer_set_us": {c: _us(v) for c, v in totals.items()},
        "layer_set_build_gweights_per_s": round(world * n_set / totals["usk_build"] / 1e9, 3),
        "spread": _spread(times["llama7b_set"]),
    }
    # 70B MLP
    mm = med["mlp70b"]
    per = {}
    for shp in ("28672x8192", "8192x28672"):
        m, k = (int(v) for v in shp.split("x"))
        d = {c.split("/")[1]: v for c, v in mm.items() if c.startswith(shp + "/")}
        # ncu traffic was taken on the 28672 x 8192 shape
        tk = (lambda key: tr.get(key)) if shp == "28672x8192" else (lambda key: None)
        per[shp] = {
            "kernel_us": {c: _us(v) for c, v in d.items()},
            "usk_build_gweights_per_s": round(world * m * k / d["usk_build"] / 1e9, 3),
            "rooflines": {"usk_build": R.hbm_line(build_bytes(m, k, 2, False), d["usk_build"], tk("mlp70b_usk_build")),
                          "usk_gemv_b1": R.gather_line(gemv_bytes(m, k, 1), m * k, d["usk_gemv_b1"],
                                                       tk("mlp70b_usk_gemv_b1")),
                          "usk_gemv_multi_b1": R.gather_line(gemv_bytes(m, k, 1), m * k, d["usk_gemv_multi_b1"],
                                                             tk("mlp70b_usk_gemv_multi_b1"))},
        }
        for bb in (16, 32, 64):
            t = d["usk_gemm_b%d" % bb]
            ln = R.gather_line(gemv_bytes(m, k, bb), m * k, t, tk("mlp70b_usk_gemm_b64") if bb == 64 else None,
                               flops=2 * m * k * bb)
            # issue-bound decode roof: about 5 lane operations per weight at 128 lanes
            # per clock per SM (31.6 us at 28672x8192)
            ln["decode_roof_us"] = round(5 * m * k / (SMS * 128 * R.clk) * 1e6, 3)
            per[shp]["rooflines"]["usk_gemm_b%d" % bb] = ln
    out["mlp70b"] = {"workload": "70B-MLP-shaped 28672x8192 and 8192x28672 bf16 N(0, 0.02^2) (device-drawn), "
                                 "no importance; decodes cycle over %d sketch copies (> L2)" % AB_COPIES,
                     "per_shape": per, "spread": _spread(times["mlp70b"])}
    # stack
    s7 = med["stack7b"]
    n_stack = STACK_LAYERS * sum(m * k for m, k in gen.LLAMA7B_SHAPES.values())
    code_stack = n_stack // 16
    stack_build_bytes = STACK_LAYERS * sum(build_bytes(m, k, 2, False) for m, k in gen.LLAMA7B_SHAPES.values())
    tok_bytes = sum(gemv_bytes(m, k, 1) for m, k in gen.LLAMA7B_SHAPES.values()) * STACK_LAYERS
    dense_bytes = sum(2 * m * k + 2 * k + 2 * m for m, k in gen.LLAMA7B_SHAPES.values()) * STACK_LAYERS
    t_tok, t_dense, t_mb = s7["token_decode"], s7["token_dense_bf16_torch"], s7["model_build"]
    t_tokg = s7["token_decode_grouped"]
    t_tokc = s7["token_decode_concurrent"]
    out["stack7b"] = {
        "workload": "32-layer 7B-shaped stack, 224 linears (q/k/v/o 4096x4096, gate/up 11008x4096, down "
                    "4096x11008 per layer), %.3f G weights, bf16 N(0, 0.02^2) device-drawn, one seed per linear; "
                    "independent N(0,1) bf16 x per linear (no chaining)" % (n_stack / 1e9),
        "model_build_ms": round(t_mb * 1e3, 4),
        "model_build_gweights_per_s": round(world * n_stack / t_mb / 1e9, 3),
        "model_build_roofline": dict(R.hbm_line(stack_build_bytes, t_mb),
                                     roof_ms=round(stack_build_bytes / R.hbm * 1e3, 3)),
        "token_decode_ms": round(t_tok * 1e3, 4),
        "token_decode_us_per_linear": round(t_tok / 224 * 1e6, 3),
        "token_decode_roofline": dict(R.gather_line(tok_bytes, n_stack, t_tok),
                                      issue_roof_ms=round(5 * n_stack / (SMS * 128 * R.clk) * 1e3, 3)),
        "tokens_per_s": round(1.0 / t_tok, 2),
        "token_decode_grouped_ms": round(t_tokg * 1e3, 4),
        "token_decode_grouped_us_per_linear": round(t_tokg / 224 * 1e6, 3),
        "token_decode_grouped_roofline": R.gather_line(tok_bytes, n_stack, t_tokg),
        "token_decode_grouped_vs_dense_speedup": round(t_dense / t_tokg, 3),
        "grouped": "usk_gemv_multi, one launch per group of products a transformer's data flow leaves "
                   "independent: (q, k, v), (o), (gate, up), (down) -- 128 launches per token",
        "token_decode_concurrent_ms": round(t_tokc * 1e3, 4),
        "token_decode_concurrent_us_per_linear": round(t_tokc / 224 * 1e6, 3),
        "token_decode_concurrent_roofline": R.gather_line(tok_bytes, n_stack, t_tokc),
        "token_decode_concurrent_vs_dense_speedup": round(t_dense / t_tokc, 3),
        "concurrent": "224 usk_gemv launches per token in a transformer layer's data-flow order: q, k and v "
                      "concurrently on three graph branches, then o, then gate and up concurrently, then down "
                      "(128 dependency levels per token)",
        "dense_bf16_torch_token_ms": round(t_dense * 1e3, 4),
        "dense_bf16_torch_hbm_frac": round(dense_bytes / t_dense / R.hbm, 4),
        "decode_vs_dense_speedup": round(t_dense / t_tok, 3),
        "code_bytes": code_stack,
        "dense_weight_bytes": 2 * n_stack,
        "timing": "one step = the whole model (224 usk_build calls) / one token (224 usk_gemv calls, batch 1, "
                  "programmatic dependent launches) / the same token as 224 torch.mm on the dense bf16 weights",
        "spread": _spread(times["stack7b"]),
    }
    # format 2
    a2 = med["absmaxmin"]
    tr2 = {k[len("amm_"):]: v for k, v in tr.items() if k.startswith("amm_")}
    out["absmaxmin"] = {
        "format": "multi-row AbsMaxMin sketch (format 2): smallest |w| kept per bucket, largest magnitude over %d "
                  "hash rows decoded; same layer, no importance" % AMM_DEPTH,
        "depth": AMM_DEPTH,
        "usk_gemv_gbs": round(world * GEMV_BYTES / a2["usk_gemv"] / 1e9, 3),
        "usk_build_gweights_per_s": round(world * N_W / a2["usk_build"] / 1e9, 3),
        "kernel_us": {k: _us(v) for k, v in a2.items()},
        "rooflines": rooflines(peaks, a2["usk_build"], a2["usk_gemv"], a2["usk_gemm"], tr2, depth=AMM_DEPTH,
                               build_bytes_=BUILD_BYTES - 4 * K),
    }
    # format 3 + A/B
    c3 = med["colshared"]
    ab_bytes = gemv_bytes(AB_M, AB_K, 1)
    out["colshared"] = {
        "format": "column-shared projection sketch (format 3): W_hat = S . P^T with one seeded one-hot P shared "
                  "by all rows; product y = S (P^T x); same layer, no importance",
        "usk_gemv_gbs": round(world * GEMV_BYTES / c3["usk_gemv"] / 1e9, 3),
        "usk_build_gweights_per_s": round(world * N_W / c3["usk_build"] / 1e9, 3),
        "kernel_us": {k: _us(v) for k, v in c3.items()},
        "rooflines": {"usk_build": R.hbm_line(BUILD_BYTES - 4 * K, c3["usk_build"], tr.get("cs_usk_build")),
                      "usk_gemv": R.hbm_line(GEMV_BYTES, c3["usk_gemv"], tr.get("cs_usk_gemv")),
                      "usk_gemv_%dx%d" % (AB_M, AB_K): R.hbm_line(ab_bytes, c3["ab_matrix_gemv"],
                                                                   tr.get("cs_usk_gemv_ab"))},
        "matrix_vs_hash": {"shape": "%dx%d" % (AB_M, AB_K), "batch": 1,
                           "hash_gemv_us": _us(c3["ab_hash_gemv"]), "matrix_gemv_us": _us(c3["ab_matrix_gemv"]),
                           "speedup": round(c3["ab_hash_gemv"] / c3["ab_matrix_gemv"], 2),
                           "layer_4096_speedup": round(med["layer"]["usk_gemv"] / c3["usk_gemv"], 2)},
    }
    # format 4
    q = med["q4"]
    tr4 = {k[len("q4_"):]: v for k, v in tr.items() if k.startswith("q4_")}
    out["q4"] = {
        "format": "4-bit-code sketch (format 4): the format-1 rule with 8 weights per bucket and a signed 4-bit "
                  "code each (0.5 bit/weight); same layer and importance",
        "usk_gemv_gbs": round(world * GEMV_BYTES / q["usk_gemv"] / 1e9, 3),
        "usk_build_gweights_per_s": round(world * N_W / q["usk_build"] / 1e9, 3),
        "kernel_us": {k: _us(v) for k, v in q.items()},
        "rooflines": rooflines(peaks, q["usk_build"], q["usk_gemv"], q["usk_gemm"], tr4),
    }
    # rates
    r = med["rates"]
    out["rates"] = {
        "format": "format 1 at 2 and 8 hash slots per class (0.25 and 1 bit/weight), the rates the "
                  "importance-aware allocation (usk_plan_slots) assigns; same layer and importance",
        "slots_2": {"kernel_us": {"usk_build": _us(r["slots_2/usk_build"]), "usk_gemv": _us(r["slots_2/usk_gemv"])},
                    "usk_gemv_gbs": round(world * (GEMV_BYTES - N_W // 32) / r["slots_2/usk_gemv"] / 1e9, 3),
                    "usk_build_gweights_per_s": round(world * N_W / r["slots_2/usk_build"] / 1e9, 3)},
        "slots_8": {"kernel_us": {"usk_build": _us(r["slots_8/usk_build"]), "usk_gemv": _us(r["slots_8/usk_gemv"])},
                    "usk_gemv_gbs": round(world * (GEMV_BYTES + N_W // 16) / r["slots_8/usk_gemv"] / 1e9, 3),
                    "usk_build_gweights_per_s": round(world * N_W / r["slots_8/usk_build"] / 1e9, 3)},
    }
    # per-row-block rates
    v = med["row_block_rates"]
    out["row_block_rates"] = {
        "format": "format 1 with one slot count per 64-row block (2, 4 or 8 hash slots per class), codes of the "
                  "blocks back to back; the layer with a lognormal(0, 0.5^2) gain per row block, rates from "
                  "usk_plan_slots at 0.5 bit/weight with importance = E[a^2] of each block's outputs over the %d "
                  "calibration rows; column importance as the headline" % GEMM_BATCH,
        "row_blocks_by_slots": {"2": rmap.count[0], "4": rmap.count[1], "8": rmap.count[2]},
        "bits_per_weight": round(8.0 * rmap.code_bytes / N_W, 4),
        "usk_gemv_gbs": round(world * (GEMV_BYTES - N_W // 16 + rmap.code_bytes) / v["usk_gemv"] / 1e9, 3),
        "usk_build_gweights_per_s": round(world * N_W / v["usk_build"] / 1e9, 3),
        "kernel_us": {k: _us(t) for k, t in v.items()},
    }
    return out


def run_c_driver(local, iters):
    """usk_gemv round trips through the C ABI alone (the in-tree usk_e2e
    program), on this rank's GPU; None if the driver is missing or fails."""
    exe = os.path.join(ROOT, "sub_bit_weight_usk_b200", "usk_e2e")
    if not os.path.exists(exe):
        return None
    env = dict(os.environ)
    vis = env.get("CUDA_VISIBLE_DEVICES")
    devs = vis.split(",") if vis else None
    env["CUDA_VISIBLE_DEVICES"] = devs[local] if devs and local < len(devs) else str(local)
    try:
        p = subprocess.run([exe, str(M), str(K), str(GEMV_BATCH), str(iters), "20"], capture_output=True,
                           text=True, timeout=120, env=env)
    except (OSError, subprocess.TimeoutExpired):
        return None
    if p.returncode != 0:
        sys.stderr.write("usk_e2e failed (%d): %s\n" % (p.returncode, p.stderr.strip()[-500:]))
        return None
    d = json.loads(p.stdout.strip().splitlines()[-1])
    d["e2e_s"] = d["e2e_us"] * 1e-6
    d["value"] = round(GEMV_BYTES / d["e2e_s"] / 1e9, 4)
    d["unit"] = "GB/s"
    return d


def cpu_baseline_json(stack, mlp, sm):
    """cpu_baseline of the JSON line: the oracle on the host cores, one thread
    and all cores, on bounded samples of each workload (host copies of the
    device-drawn weights)."""
    import torch

    def host(t):
        return t.cpu().view(torch.int16).numpy().view(np.uint16)

    pick = {e["name"]: e for e in stack if e["layer"] == 0}
    extra = [("small", sm["W"], sm["x"], sm["importance"])]
    for name in ("q", "gate", "down"):
        e = pick[name]
        extra.append(("7b_" + name, host(e["W"]), host(e["x1"]), None))
    for name, e in mlp.items():
        extra.append(("70b_" + name, host(e["W"]), host(e["x"][:1]), None))
    t0 = time.perf_counter()
    c = cpu_oracle_baseline(extra)
    wall = time.perf_counter() - t0
    info = cpu_info()
    L = c["layer"]
    per = {}
    for name, _, _, _ in extra:
        d = c[name]
        per[name] = {"build_s": {k: round(v, 4) for k, v in d["build_s"].items()},
                     "gemv_s": {k: round(v, 4) for k, v in d["gemv_s"].items()}}
    # the whole stack, from the per-shape times of layer 0 (32 x (4 q + 2 gate + down))
    st_build = {m: 32 * (4 * c["7b_q"]["build_s"][m] + 2 * c["7b_gate"]["build_s"][m] + c["7b_down"]["build_s"][m])
                for m in ("1", "all")}
    st_tok = {m: 32 * (4 * c["7b_q"]["gemv_s"][m] + 2 * c["7b_gate"]["gemv_s"][m] + c["7b_down"]["gemv_s"][m])
              for m in ("1", "all")}
    return {
        "value": round(GEMV_BYTES / L["gemv_s"]["all"] / 1e9, 4), "unit": "GB/s", "cores": c["cores_all"],
        "kind": "oracle",
        "sample": "headline: whole 4096x4096 layer, batch 1, float64 oracle GEMV on all %d host threads (%d "
                  "pass(es)); one-thread mode alongside; other workloads: one build and one GEMV each (tall "
                  "matrices' one-thread GEMV on sampled rows, scaled); %.1f s of host time in all"
                  % (c["cores_all"], L["gemv_reps"]["all"], wall),
        "one_thread": {"value": round(GEMV_BYTES / L["gemv_s"]["1"] / 1e9, 4), "unit": "GB/s", "cores": 1},
        "build_gweights_per_s": {"1": round(N_W / L["build_s"]["1"] / 1e9, 4),
                                 "all": round(N_W / L["build_s"]["all"] / 1e9, 4)},
        "per_workload_s": per,
        "stack7b_estimate_s": {"model_build": {m: round(v, 2) for m, v in st_build.items()},
                               "token_decode": {m: round(v, 2) for m, v in st_tok.items()}},
        "nproc": info["nproc"], "cpu_model": info["cpu_model"],
    }


def run_profile_case(args):
    """A few launches of one kernel on a bench workload, for ncu captures
    (e.g. ncu --set full --clock-control none -k regex:gemv -s 3 -c 1
    python bench.py --profile-case gemv).  Prints nothing but a status line."""
    import torch
    import sub_bit_weight_usk_b200 as usk
    dev = torch.device("cuda", 0)
    cfg = gen.layer(GEMM_BATCH)

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    W = to_dev(cfg["W"])
    imp = torch.from_numpy(cfg["importance"]).to(dev)
    x16 = to_dev(cfg["x"])
    x1 = x16[:GEMV_BATCH].contiguous()
    case = args.profile_case
    fmt = {}
    if case.endswith("_amm"):
        fmt = {"version": usk.FORMAT_ABSMAXMIN, "depth": AMM_DEPTH}
    elif "_cs" in case:
        fmt = {"version": usk.FORMAT_COLSHARED}
    elif case.endswith("_q4"):
        fmt = {"version": usk.FORMAT_Q4}
    if case.endswith("_vr"):  # per-row-block rates on the row-gain layer
        Wv_h, vr_slots = row_block_workload(cfg, usk)
        W = to_dev(Wv_h)
        fmt = {"rates": usk.usk_rate_map(M, K, vr_slots, dev)}
    if case.endswith("_ab") or case.endswith("_70b"):  # the 28672 x 8192 shape, device-drawn weights
        W = gen.device_weights_normal(AB_M, AB_K, 3, 0.02, dev)
        xa = to_dev(gen.activations(64, AB_K, 3, "bf16"))
        x1 = xa[:1].contiguous()
        x16 = xa
    imp_c = imp if (not fmt or case.endswith("_q4") or case.endswith("_vr")) and \
        not (case.endswith("_ab") or case.endswith("_70b")) else None
    sk = usk.usk_build(W, imp_c, cfg["seed"], **fmt)
    torch.cuda.synchronize()
    ws = None
    if case.startswith("gemv_multi"):
        ws = torch.zeros(max(16, usk.usk_gemv_multi_ws_bytes([sk], 1)), dtype=torch.uint8, device=dev)
    for _ in range(3 + 3):  # 3 warm-up launches, then 3 to capture
        if case.startswith("gemv_multi"):
            usk.usk_gemv_multi([sk], [x1], ws=ws)
        elif case.startswith("build"):
            usk.usk_build(W, imp_c, cfg["seed"], codes=sk.codes, scales=sk.scales, **fmt)
        elif case.startswith("gemv"):
            usk.usk_gemv(sk, x1)
        else:
            usk.usk_gemm(sk, x16)
    torch.cuda.synchronize()
    print("profile case %s done" % args.profile_case)
    return 0


PROFILE_CASES = ["build", "gemv", "gemm", "build_amm", "gemv_amm", "gemm_amm", "build_cs", "gemv_cs", "gemv_ab",
                 "gemv_cs_ab", "build_q4", "gemv_q4", "gemm_q4", "build_vr", "gemv_vr", "gemm_vr", "build_70b",
                 "gemm_70b", "gemv_70b", "gemv_multi", "gemv_multi_70b"]


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="usk", choices=["usk", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="run 6 launches of one kernel on a bench workload (for ncu) and exit")
    args = ap.parse_args(argv)
    if args.profile_case:
        return run_profile_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps < 1:
        ap.error("--steps must be at least 1")
    if args.impl == "reference":
        return run_reference(args)
    return run_usk(args)


if __name__ == "__main__":
    sys.exit(main())
