#!/usr/bin/env python
"""Benchmark of the UltraSketchLLM sketch hot path on B200.

One step = one pass of the whole hot path over one 4096x4096 bf16 layer:
usk_build (key, hash, scatter-select, winner, scale, quantize), usk_gemv at
batch 1 (rehash + gather decode, product) and usk_gemm at batch 16 (decode into
tcgen05 tiles).  The headline value is usk_gemv GB/s (algorithmic bytes of one
call / its average launch duration); usk_build Gweights/s rides along.  A second
timed region runs the same three calls K times on the multi-row AbsMaxMin sketch
(format 2, depth 2) of the same layer and reports them under "absmaxmin"; a
third runs K builds and K batch-1 GEMVs of the column-shared projection sketch
(format 3, y = S (P^T x)) and a fourth the "matrix vs hash" A/B: K batch-1 GEMVs
of a 28672x8192 layer in format 1 (per-weight rehash and gather) and in format 3
(bucket sums of x, then dense codes), reported under "colshared"; a fifth runs
the three calls on the 4-bit-code sketch (format 4) of the layer ("q4"), and a
sixth K builds and K batch-1 GEMVs of the layer at 2 and 8 hash slots per class
(0.25 and 1 bit/weight, the rates of the importance-aware allocation, "rates"),
and a seventh the three calls on a sketch whose 64-row blocks carry their own
rates, allocated at 0.5 bit/weight from the E[a^2] of each block's outputs on
the layer with one lognormal gain per row block ("row_block_rates").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl usk|reference]

For N > 1 run under torchrun (one rank per GPU): every rank sketches and
multiplies its own layer (weak scaling, no data-path collective); the timing is
the max over ranks.  `--impl reference` times the plain CPU oracle on the host
cores on a bounded sample of the same workload.
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
GRAPH_STEPS = 256  # steps per captured CUDA graph
AMM_DEPTH = 2      # hash rows of the format-2 (multi-row AbsMaxMin) measurement
AB_M, AB_K = 28672, 8192  # the matrix-vs-hash A/B shape (70B MLP up-projection)
AB_COPIES = 10            # 10 x 14 MiB of codes per format (> L2)

METRIC = "usk_gemv GB/s & % roofline (4096x4096, batch 1); usk_build Gweights/s"
WORKLOAD = ("one 4096x4096 bf16 layer, Student-t(4) x 0.02 with 0.1% outliers x20, importance = mean |x| "
            "over 128 N(0,1) rows; usk_build + usk_gemv batch 1 + usk_gemm batch 16")

# algorithmic bytes / flops per call
N_W = M * K
GEMV_BYTES = N_W // 16 + 2 * (M // 64) + 2 * K * GEMV_BATCH + 4 * M * GEMV_BATCH  # 1,073,280
GEMM_BYTES = N_W // 16 + 2 * (M // 64) + 2 * K * GEMM_BATCH + 4 * M * GEMM_BATCH
BUILD_BYTES = 2 * N_W + N_W // 16 + 4 * K + 2 * (M // 64)
GEMM_FLOPS = 2 * N_W * GEMM_BATCH

SMS = 148
SMEM_BYTES_PER_CLK = 128  # shared-memory load bandwidth per SM per clock
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


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


def rooflines(peaks, t_build_s, t_gemv_s, t_gemm_s, traffic, depth=1, build_bytes=None):
    """Roofline of each kernel from its algorithmic work and the measured peaks.

    usk_build is HBM-bound (2 B of bf16 weight in, 1/16 B of code out per weight).
    usk_gemv / usk_gemm decode every weight by a shared-memory gather of its
    bucket code: at least 1 byte per weight through the 128 B/clk/SM shared
    memory pipe, which binds before HBM (codes are 1/16 B per weight); gemm also
    checks the dense bf16 tensor time.  A depth-D sketch gathers D codes per
    weight."""
    hbm = peaks["hbm_gbs"] * 1e9
    clk = peaks.get("sm_max_mhz", 1965.0) * 1e6
    smem = SMS * SMEM_BYTES_PER_CLK * clk
    src = peaks["source"]

    def line(bound, achieved, peak, unit, tr):
        return {"bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 3), "unit": unit,
                "frac": round(achieved / peak, 4), "traffic": tr, "peak_source": src}

    out = {}
    # build: HBM
    bb = BUILD_BYTES if build_bytes is None else build_bytes
    out["usk_build"] = line("hbm", bb / t_build_s / 1e9, hbm / 1e9, "GB/s", traffic.get("usk_build"))
    # gemv: gather-bound; expressed in algorithmic GB/s against the bytes/time at the binding bound
    t_bound = max(GEMV_BYTES / hbm, depth * N_W / smem)
    out["usk_gemv"] = line("alu", GEMV_BYTES / t_gemv_s / 1e9, GEMV_BYTES / t_bound / 1e9, "GB/s",
                           traffic.get("usk_gemv"))
    out["usk_gemv"]["binding"] = "shared-memory gather (%d B/weight at 128 B/clk/SM)" % depth
    t_bound = max(GEMM_BYTES / hbm, depth * N_W / smem, GEMM_FLOPS / (peaks["bf16_tflops"] * 1e12))
    out["usk_gemm"] = line("alu", GEMM_BYTES / t_gemm_s / 1e9, GEMM_BYTES / t_bound / 1e9, "GB/s",
                           traffic.get("usk_gemm"))
    out["usk_gemm"]["tensor_tflops"] = round(GEMM_FLOPS / t_gemm_s / 1e12, 3)
    return out


def colshared_rooflines(peaks, t_build_s, t_gemv_s, t_gemv_ab_s, traffic):
    """Format 3: the build reads W once (HBM); the product streams 1/16 B of
    code per weight with no gathers, so its bound is HBM too."""
    hbm = peaks["hbm_gbs"] * 1e9
    src = peaks["source"]

    def line(achieved, tr):
        return {"bound": "hbm", "achieved": round(achieved, 3), "peak": round(hbm / 1e9, 3), "unit": "GB/s",
                "frac": round(achieved / (hbm / 1e9), 4), "traffic": tr, "peak_source": src}

    ab_bytes = AB_M * AB_K // 16 + 2 * (AB_M // 64) + 2 * AB_K + 4 * AB_M
    return {"usk_build": line((BUILD_BYTES - 4 * K) / t_build_s / 1e9, traffic.get("cs_usk_build")),
            "usk_gemv": line(GEMV_BYTES / t_gemv_s / 1e9, traffic.get("cs_usk_gemv")),
            "usk_gemv_%dx%d" % (AB_M, AB_K): line(ab_bytes / t_gemv_ab_s / 1e9, traffic.get("cs_usk_gemv_ab"))}


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
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

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
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


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


# ------------------------------------------------------------------ CPU oracle

def cpu_oracle_times(budget_s=20.0):
    """The oracle as it stands, single-threaded on this host: GEMV over the whole
    layer (repeated while within the budget) and the build of the whole layer."""
    import oracle
    cfg = gen.layer(1)
    o = oracle.build_sketch(cfg["W"], cfg["importance"], cfg["seed"])
    t0 = time.perf_counter()
    oracle.build_sketch(cfg["W"], cfg["importance"], cfg["seed"])
    t_build = time.perf_counter() - t0
    reps, t_gemv = 0, 0.0
    while reps == 0 or (t_gemv < budget_s * 0.5 and reps < 20):
        t0 = time.perf_counter()
        oracle.gemv_f64(o["codes"], o["scales"], M, K, cfg["x"], cfg["seed"])
        t_gemv += time.perf_counter() - t0
        reps += 1
    return {"gemv_s": t_gemv / reps, "build_s": t_build, "reps": reps}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    cfg = gen.layer(1)
    o = oracle.build_sketch(cfg["W"], cfg["importance"], cfg["seed"])
    # calibrate: time one 64-row block, size each step to fit the run in about a minute
    t0 = time.perf_counter()
    oracle.gemv_f64(o["codes"], o["scales"], M, K, cfg["x"], cfg["seed"], rows=np.arange(64))
    t_row = (time.perf_counter() - t0) / 64
    total = args.steps + args.warmup
    rows_per_step = int(max(1, min(M, (60.0 / max(total, 1)) / max(t_row, 1e-9))))
    g = np.random.default_rng(7)
    for _ in range(args.warmup):
        oracle.gemv_f64(o["codes"], o["scales"], M, K, cfg["x"], cfg["seed"],
                        rows=g.integers(0, M, rows_per_step))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gemv_f64(o["codes"], o["scales"], M, K, cfg["x"], cfg["seed"],
                        rows=g.integers(0, M, rows_per_step))
    t = (time.perf_counter() - t0) / max(args.steps, 1)
    # scale the sampled rows to one full-layer call
    t_full = t * M / rows_per_step
    value = GEMV_BYTES / t_full / 1e9
    sample = "%d random rows of the 4096x4096 layer per step (of %d), scaled to a full call" % (rows_per_step, M)
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "batch": GEMV_BATCH},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

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
    cfg = gen.layer(GEMM_BATCH)
    W = torch.from_numpy(cfg["W"].view(np.int16)).to(dev).view(torch.bfloat16)
    imp = torch.from_numpy(cfg["importance"]).to(dev)
    x16 = torch.from_numpy(cfg["x"].view(np.int16)).to(dev).view(torch.bfloat16)
    x1 = x16[:GEMV_BATCH].contiguous()
    seed = cfg["seed"]
    Ws = [W.clone() for _ in range(N_WCOPIES)]
    sk0 = usk.usk_build(W, imp, seed)
    sks = [usk.Sketch(M, K, seed, sk0.codes.clone(), sk0.scales.clone()) for _ in range(N_SKETCHES)]
    y1 = torch.empty((GEMV_BATCH, M), device=dev)
    y16 = torch.empty((GEMM_BATCH, M), device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()

    def build(i):
        b = sks[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status)

    def gemv(i):
        # consecutive decode calls: each launches as a programmatic dependent of
        # the previous one (its set-up overlaps the previous call's tail)
        usk.usk_gemv(sks[(i + N_SKETCHES // 2) % N_SKETCHES], x1, y=y1, pdl=True)

    def gemm(i):
        usk.usk_gemm(sks[(i + N_SKETCHES // 4) % N_SKETCHES], x16, y=y16, status=status)

    # the same three calls on the multi-row AbsMaxMin sketch (format 2) of the layer
    amm = usk.FORMAT_ABSMAXMIN
    sk2 = usk.usk_build(W, None, seed, version=amm, depth=AMM_DEPTH)
    sks2 = [usk.Sketch(M, K, seed, sk2.codes.clone(), sk2.scales.clone(), amm, AMM_DEPTH) for _ in range(N_SKETCHES)]

    def build2(i):
        b = sks2[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], None, seed, codes=b.codes, scales=b.scales, status=status, version=amm,
                      depth=AMM_DEPTH)

    def gemv2(i):
        usk.usk_gemv(sks2[(i + N_SKETCHES // 2) % N_SKETCHES], x1, y=y1, pdl=True)

    def gemm2(i):
        usk.usk_gemm(sks2[(i + N_SKETCHES // 4) % N_SKETCHES], x16, y=y16, status=status)

    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())

    def capture(fn, n, offset):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for j in range(n):
                fn(offset + j)
        return g

    full, rem = divmod(args.steps, GRAPH_STEPS)

    def prepare(kernels):
        # warm-up (untimed, eager): W full steps, then one graph per phase
        for i in range(args.warmup):
            for k in kernels:
                k(i)
        torch.cuda.synchronize()
        if int(status.item()) != 0:
            raise SystemExit("device status flags %#x during warm-up" % int(status.item()))
        graphs = []
        for fn in kernels:
            main = capture(fn, GRAPH_STEPS, args.warmup) if full else None
            tail = capture(fn, rem, args.warmup) if rem else None
            graphs.append((main, tail))
        torch.cuda.synchronize()
        return graphs

    def timed(graphs):
        # Timed region: exactly K steps.  The K steps run phase by phase (K
        # builds, then K GEMVs, then K GEMMs; the same work as K build+gemv+gemm
        # passes) so that each kernel's average launch duration is the CUDA-event
        # time of its phase / K, with no timing nodes between kernels.  Each phase
        # replays a CUDA graph of GRAPH_STEPS launches (+ one for the remainder).
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(graphs) + 1)]
        ev[0].record()
        for k, (main, tail) in enumerate(graphs):
            for _ in range(full):
                main.replay()
            if tail is not None:
                tail.replay()
            ev[k + 1].record()
        ev[-1].synchronize()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        if int(status.item()) != 0:
            raise SystemExit("device status flags %#x in the timed region" % int(status.item()))
        n = max(args.steps, 1)
        return [ev[k].elapsed_time(ev[k + 1]) * 1e-3 / n for k in range(len(graphs))] + \
            [ev[0].elapsed_time(ev[-1]) * 1e-3]

    # format 3 (column-shared projection) on the same layer: build and GEMV
    cs = usk.FORMAT_COLSHARED
    sk3 = usk.usk_build(W, None, seed, version=cs)
    sks3 = [usk.Sketch(M, K, seed, sk3.codes.clone(), sk3.scales.clone(), cs, 1) for _ in range(N_SKETCHES)]

    def build3(i):
        b = sks3[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], None, seed, codes=b.codes, scales=b.scales, status=status, version=cs)

    def gemv3(i):
        usk.usk_gemv(sks3[(i + N_SKETCHES // 2) % N_SKETCHES], x1, y=y1, pdl=True)

    # the matrix-vs-hash A/B at 28672 x 8192, batch 1 (device-drawn N(0, 0.02^2)
    # weights: the values do not change the decode work)
    Wab = gen.device_weights_normal(AB_M, AB_K, 3, 0.02, dev)
    skh = usk.usk_build(Wab, None, 3)
    skm = usk.usk_build(Wab, None, 3, version=cs)
    del Wab
    abh = [usk.Sketch(AB_M, AB_K, 3, skh.codes.clone(), skh.scales.clone()) for _ in range(AB_COPIES)]
    abm = [usk.Sketch(AB_M, AB_K, 3, skm.codes.clone(), skm.scales.clone(), cs, 1) for _ in range(AB_COPIES)]
    xab = torch.from_numpy(gen.activations(1, AB_K, 3, "bf16").view(np.int16)).to(dev).view(torch.bfloat16)
    yab = torch.empty((1, AB_M), device=dev)

    def gemv_hash(i):
        usk.usk_gemv(abh[i % AB_COPIES], xab, y=yab, pdl=True)

    def gemv_matrix(i):
        usk.usk_gemv(abm[i % AB_COPIES], xab, y=yab, pdl=True)

    # format 4 (4-bit codes, 8 weights per bucket) on the same layer, with importance
    q4 = usk.FORMAT_Q4
    sk4 = usk.usk_build(W, imp, seed, version=q4)
    sks4 = [usk.Sketch(M, K, seed, sk4.codes.clone(), sk4.scales.clone(), q4, 1) for _ in range(N_SKETCHES)]

    def build4(i):
        b = sks4[i % N_SKETCHES]
        usk.usk_build(Ws[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status, version=q4)

    def gemv4(i):
        usk.usk_gemv(sks4[(i + N_SKETCHES // 2) % N_SKETCHES], x1, y=y1, pdl=True)

    def gemm4(i):
        usk.usk_gemm(sks4[(i + N_SKETCHES // 4) % N_SKETCHES], x16, y=y16, status=status)

    # format 1 at 2 and 8 hash slots per class (0.25 and 1 bit/weight)
    rate_sk = {}
    for nsl in (2, 8):
        skr = usk.usk_build(W, imp, seed, slots=nsl)
        rate_sk[nsl] = [usk.Sketch(M, K, seed, skr.codes.clone(), skr.scales.clone(), usk.FORMAT_MAXKEY, 1, nsl)
                        for _ in range(N_SKETCHES)]

    def build_rate(nsl):
        def f(i):
            b = rate_sk[nsl][i % N_SKETCHES]
            usk.usk_build(Ws[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status, slots=nsl)
        return f

    def gemv_rate(nsl):
        def f(i):
            usk.usk_gemv(rate_sk[nsl][(i + N_SKETCHES // 2) % N_SKETCHES], x1, y=y1, pdl=True)
        return f

    graphs1 = prepare((build, gemv, gemm))
    graphs2 = prepare((build2, gemv2, gemm2))
    graphs3 = prepare((build3, gemv3))
    graphs4 = prepare((gemv_hash, gemv_matrix))
    graphs5 = prepare((build4, gemv4, gemm4))
    graphs6 = prepare((build_rate(2), gemv_rate(2), build_rate(8), gemv_rate(8)))

    # per-row-block rates on the row-gain layer
    Wv_h, vr_slots = row_block_workload(cfg, usk)
    Wv = torch.from_numpy(Wv_h.view(np.int16)).to(dev).view(torch.bfloat16)
    Wvs = [Wv.clone() for _ in range(N_WCOPIES)]
    rmap = usk.usk_rate_map(M, K, vr_slots, dev)
    skv = usk.usk_build(Wv, imp, seed, rates=rmap)
    sksv = [usk.Sketch(M, K, seed, skv.codes.clone(), skv.scales.clone(), usk.FORMAT_MAXKEY, 1, 0, rmap)
            for _ in range(N_SKETCHES)]

    def build_vr(i):
        b = sksv[i % N_SKETCHES]
        usk.usk_build(Wvs[i % N_WCOPIES], imp, seed, codes=b.codes, scales=b.scales, status=status, rates=rmap)

    def gemv_vr(i):
        usk.usk_gemv(sksv[(i + N_SKETCHES // 2) % N_SKETCHES], x1, y=y1, pdl=True)

    def gemm_vr(i):
        usk.usk_gemm(sksv[(i + N_SKETCHES // 4) % N_SKETCHES], x16, y=y16, status=status)

    graphs7 = prepare((build_vr, gemv_vr, gemm_vr))
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    t_build, t_gemv, t_gemm, t_total = timed(graphs1)
    t_build2, t_gemv2, t_gemm2, _ = timed(graphs2)
    t_build3, t_gemv3, _ = timed(graphs3)
    t_hash, t_matrix, _ = timed(graphs4)
    t_build4, t_gemv4, t_gemm4, _ = timed(graphs5)
    t_build_r2, t_gemv_r2, t_build_r8, t_gemv_r8, _ = timed(graphs6)
    t_build_v, t_gemv_v, t_gemm_v, _ = timed(graphs7)
    sampler.stop()
    t_step = t_total / max(args.steps, 1)

    # end to end through the public API with host buffers: x in from pinned host memory, y back out
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
    t_e2e = (time.perf_counter() - t0) / n_e2e

    # max over ranks
    (t_gemv, t_build, t_gemm, t_step, t_total, t_e2e, t_build2, t_gemv2, t_gemm2, t_build3, t_gemv3, t_hash,
     t_matrix, t_build4, t_gemv4, t_gemm4, t_build_r2, t_gemv_r2, t_build_r8, t_gemv_r8, t_build_v, t_gemv_v,
     t_gemm_v) = max_over_ranks(
        [t_gemv, t_build, t_gemm, t_step, t_total, t_e2e, t_build2, t_gemv2, t_gemm2, t_build3, t_gemv3, t_hash,
         t_matrix, t_build4, t_gemv4, t_gemm4, t_build_r2, t_gemv_r2, t_build_r8, t_gemv_r8, t_build_v, t_gemv_v,
         t_gemm_v], device=dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        c = cpu_oracle_times()
        cpu = {"value": round(GEMV_BYTES / c["gemv_s"] / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": "whole 4096x4096 layer, batch 1, float64 oracle GEMV (%d pass(es)); oracle build of the "
                         "layer %.2f s = %.4f Gweights/s" % (c["reps"], c["build_s"], N_W / c["build_s"] / 1e9)}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks = load_peaks()
    agg = aggregate(world, [t_gemv], [t_build], [t_step])
    tr = load_traffic()
    rl = rooflines(peaks, t_build, t_gemv, t_gemm, tr)
    tr2 = {k[len("amm_"):]: v for k, v in tr.items() if k.startswith("amm_")}
    rl2 = rooflines(peaks, t_build2, t_gemv2, t_gemm2, tr2, depth=AMM_DEPTH, build_bytes=BUILD_BYTES - 4 * K)
    tr4 = {k[len("q4_"):]: v for k, v in tr.items() if k.startswith("q4_")}
    rl4 = rooflines(peaks, t_build4, t_gemv4, t_gemm4, tr4)
    clocks = sampler.summary()
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
                   "timing": "K steps run phase by phase (K builds, K GEMVs, K GEMMs) as CUDA graphs; "
                             "kernel time = phase event time / K",
                   "gemv_launch": "programmatic dependent launch (USK_GEMV_PDL) between consecutive GEMV calls",
                   "l2": "inputs larger than L2: builds cycle over %d weight copies (%d MiB), decodes over %d "
                         "sketch copies (%d MiB)" % (N_WCOPIES, N_WCOPIES * 32, N_SKETCHES, N_SKETCHES),
                   "parallelism": "replicas" if world > 1 else "single"},
        "usk_build_gweights_per_s": round(agg["build_gweights_s"], 3),
        "kernel_us": {"usk_build": round(t_build * 1e6, 3), "usk_gemv": round(t_gemv * 1e6, 3),
                      "usk_gemm": round(t_gemm * 1e6, 3)},
        "roofline": rl["usk_gemv"],
        "rooflines": rl,
        "clocks": clocks,
        "e2e": {"value": round(world * GEMV_BYTES / t_e2e / 1e9, 4), "unit": "GB/s",
                "h2d_bytes_per_step": int(xh.numel() * 2), "d2h_bytes_per_step": int(yh.numel() * 4),
                "call": "usk_gemv via the Python binding, x from pinned host memory, y read back, per step"},
        "gpu_launches": 3 * args.steps,
        "cpu_baseline": cpu,
        "absmaxmin": {
            "format": "multi-row AbsMaxMin sketch (format 2): smallest |w| kept per bucket, largest magnitude "
                      "over %d hash rows decoded; same layer, no importance" % AMM_DEPTH,
            "depth": AMM_DEPTH,
            "timing": "a second timed region: K builds, K GEMVs (batch 1), K GEMMs (batch 16) as CUDA graphs",
            "usk_gemv_gbs": round(world * GEMV_BYTES / t_gemv2 / 1e9, 3),
            "usk_build_gweights_per_s": round(world * N_W / t_build2 / 1e9, 3),
            "kernel_us": {"usk_build": round(t_build2 * 1e6, 3), "usk_gemv": round(t_gemv2 * 1e6, 3),
                          "usk_gemm": round(t_gemm2 * 1e6, 3)},
            "rooflines": rl2,
            "gpu_launches": 3 * args.steps,
        },
        "colshared": {
            "format": "column-shared projection sketch (format 3): W_hat = S . P^T with one seeded one-hot P "
                      "shared by all rows; product y = S (P^T x); same layer, no importance",
            "timing": "third timed region: K builds and K GEMVs (batch 1) as CUDA graphs; fourth: K batch-1 "
                      "GEMVs of a %dx%d layer in format 1 and in format 3, %d sketch copies each (> L2)"
                      % (AB_M, AB_K, AB_COPIES),
            "usk_gemv_gbs": round(world * GEMV_BYTES / t_gemv3 / 1e9, 3),
            "usk_build_gweights_per_s": round(world * N_W / t_build3 / 1e9, 3),
            "kernel_us": {"usk_build": round(t_build3 * 1e6, 3), "usk_gemv": round(t_gemv3 * 1e6, 3)},
            "rooflines": colshared_rooflines(peaks, t_build3, t_gemv3, t_matrix, tr),
            "matrix_vs_hash": {
                "shape": "%dx%d" % (AB_M, AB_K), "batch": 1, "data": "device-drawn bf16 N(0, 0.02^2) weights",
                "hash_gemv_us": round(t_hash * 1e6, 3), "matrix_gemv_us": round(t_matrix * 1e6, 3),
                "speedup": round(t_hash / t_matrix, 2),
                "layer_4096_speedup": round(t_gemv / t_gemv3, 2),
            },
            "gpu_launches": 4 * args.steps,
        },
        "q4": {
            "format": "4-bit-code sketch (format 4): the format-1 rule with 8 weights per bucket and a signed "
                      "4-bit code each (0.5 bit/weight); same layer and importance",
            "timing": "fifth timed region: K builds, K GEMVs (batch 1), K GEMMs (batch 16) as CUDA graphs",
            "usk_gemv_gbs": round(world * GEMV_BYTES / t_gemv4 / 1e9, 3),
            "usk_build_gweights_per_s": round(world * N_W / t_build4 / 1e9, 3),
            "kernel_us": {"usk_build": round(t_build4 * 1e6, 3), "usk_gemv": round(t_gemv4 * 1e6, 3),
                          "usk_gemm": round(t_gemm4 * 1e6, 3)},
            "rooflines": rl4,
            "gpu_launches": 3 * args.steps,
        },
        "rates": {
            "format": "format 1 at 2 and 8 hash slots per class (0.25 and 1 bit/weight), the rates the "
                      "importance-aware allocation (usk_plan_slots) assigns; same layer and importance",
            "timing": "sixth timed region: K builds and K GEMVs (batch 1) at each rate as CUDA graphs",
            "slots_2": {"kernel_us": {"usk_build": round(t_build_r2 * 1e6, 3), "usk_gemv": round(t_gemv_r2 * 1e6, 3)},
                        "usk_gemv_gbs": round(world * (GEMV_BYTES - N_W // 32) / t_gemv_r2 / 1e9, 3),
                        "usk_build_gweights_per_s": round(world * N_W / t_build_r2 / 1e9, 3)},
            "slots_8": {"kernel_us": {"usk_build": round(t_build_r8 * 1e6, 3), "usk_gemv": round(t_gemv_r8 * 1e6, 3)},
                        "usk_gemv_gbs": round(world * (GEMV_BYTES + N_W // 16) / t_gemv_r8 / 1e9, 3),
                        "usk_build_gweights_per_s": round(world * N_W / t_build_r8 / 1e9, 3)},
            "gpu_launches": 4 * args.steps,
        },
        "row_block_rates": {
            "format": "format 1 with one slot count per 64-row block (2, 4 or 8 hash slots per class), codes of "
                      "the blocks back to back; the layer with a lognormal(0, 0.5^2) gain per row block, rates "
                      "from usk_plan_slots at 0.5 bit/weight with importance = E[a^2] of each block's outputs "
                      "over the %d calibration rows; column importance as the headline" % GEMM_BATCH,
            "timing": "seventh timed region: K builds, K GEMVs (batch 1), K GEMMs (batch 16) as CUDA graphs; "
                      "each call is one launch over every row block (the block's slot group picks its layout)",
            "row_blocks_by_slots": {"2": rmap.count[0], "4": rmap.count[1], "8": rmap.count[2]},
            "bits_per_weight": round(8.0 * rmap.code_bytes / N_W, 4),
            "usk_gemv_gbs": round(world * (GEMV_BYTES - N_W // 16 + rmap.code_bytes) / t_gemv_v / 1e9, 3),
            "usk_build_gweights_per_s": round(world * N_W / t_build_v / 1e9, 3),
            "kernel_us": {"usk_build": round(t_build_v * 1e6, 3), "usk_gemv": round(t_gemv_v * 1e6, 3),
                          "usk_gemm": round(t_gemm_v * 1e6, 3)},
            "gpu_launches": 3 * args.steps,
        },
    }
    print(json.dumps(line), flush=True)
    return 0


def run_profile_case(args):
    """A few launches of one kernel on the bench workload, for ncu captures
    (e.g. ncu --set full --clock-control none -k regex:gemv -s 3 -c 1
    python bench.py --profile-case gemv).  Prints nothing but a status line."""
    import torch
    import sub_bit_weight_usk_b200 as usk
    dev = torch.device("cuda", 0)
    cfg = gen.layer(GEMM_BATCH)
    W = torch.from_numpy(cfg["W"].view(np.int16)).to(dev).view(torch.bfloat16)
    imp = torch.from_numpy(cfg["importance"]).to(dev)
    x16 = torch.from_numpy(cfg["x"].view(np.int16)).to(dev).view(torch.bfloat16)
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
        W = torch.from_numpy(Wv_h.view(np.int16)).to(dev).view(torch.bfloat16)
        fmt = {"rates": usk.usk_rate_map(M, K, vr_slots, dev)}
    if case.endswith("_ab"):  # the 28672 x 8192 A/B shape, device-drawn weights
        W = gen.device_weights_normal(AB_M, AB_K, 3, 0.02, dev)
        x1 = torch.from_numpy(gen.activations(1, AB_K, 3, "bf16").view(np.int16)).to(dev).view(torch.bfloat16)
    imp_c = imp if (not fmt or case.endswith("_q4") or case.endswith("_vr")) and not case.endswith("_ab") else None
    sk = usk.usk_build(W, imp_c, cfg["seed"], **fmt)
    torch.cuda.synchronize()
    for _ in range(3 + 3):  # 3 warm-up launches, then 3 to capture
        if case.startswith("build"):
            usk.usk_build(W, imp_c, cfg["seed"], codes=sk.codes, scales=sk.scales, **fmt)
        elif case.startswith("gemv"):
            usk.usk_gemv(sk, x1)
        else:
            usk.usk_gemm(sk, x16)
    torch.cuda.synchronize()
    print("profile case %s done" % args.profile_case)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="usk", choices=["usk", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=["build", "gemv", "gemm", "build_amm", "gemv_amm", "gemm_amm",
                                               "build_cs", "gemv_cs", "gemv_ab", "gemv_cs_ab", "build_q4", "gemv_q4",
                                               "gemm_q4", "build_vr", "gemv_vr", "gemm_vr"],
                    default=None,
                    help="run 6 launches of one kernel on the bench workload (for ncu) and exit")
    args = ap.parse_args(argv)
    if args.profile_case:
        return run_profile_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_usk(args)


if __name__ == "__main__":
    sys.exit(main())
