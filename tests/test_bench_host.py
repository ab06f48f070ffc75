"""Host logic of bench.py on the CPU: whole-job aggregation and the
max-over-ranks timing reduction with two gloo ranks."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_aggregate_weak_scaling():
    a = bench.aggregate(1, [2e-6], [10e-6], [20e-6])
    assert a["gemv_gbs"] == pytest.approx(bench.GEMV_BYTES / 2e-6 / 1e9)
    assert a["build_gweights_s"] == pytest.approx(bench.N_W / 10e-6 / 1e9)
    b = bench.aggregate(2, [2e-6, 3e-6], [10e-6, 8e-6], [20e-6, 21e-6])
    assert b["gemv_gbs"] == pytest.approx(2 * bench.GEMV_BYTES / 3e-6 / 1e9)  # slowest rank
    assert b["ms_per_step"] == pytest.approx(21e-3)


def test_algorithmic_bytes():
    assert bench.GEMV_BYTES == 1073280
    assert bench.BUILD_BYTES == 2 * 4096 * 4096 + 4096 * 4096 // 16 + 4 * 4096 + 128


def test_rooflines_shape():
    peaks = {"hbm_gbs": 6540.2, "bf16_tflops": 1645.9, "sm_max_mhz": 1965.0, "source": "measured"}
    r = bench.rooflines(peaks, 5.3e-6, 0.451e-6, 1e-6, {})
    assert r["usk_build"]["bound"] == "hbm" and 0.9 < r["usk_build"]["frac"] < 1.1
    assert r["usk_gemv"]["bound"] == "alu" and 0.95 < r["usk_gemv"]["frac"] < 1.05
    for v in r.values():
        json.dumps(v)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0])
        out[rank] = vals
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == [2.0, 10.0, 5.0] and out[1] == [2.0, 10.0, 5.0]


def test_single_process_identity():
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]


def test_row_block_workload_allocation():
    """The bench's per-row-block-rate workload: the allocation keeps the 0.5
    bit/weight budget, mixes rates, and gives no block fewer slots than a block
    of smaller output energy (the gain per block drives E[a^2])."""
    import numpy as np
    import gen
    import oracle
    import sub_bit_weight_usk_b200 as usk
    cfg = gen.layer(bench.GEMM_BATCH)
    Wv, slots = bench.row_block_workload(cfg, usk)
    RB = bench.M // 64
    assert Wv.shape == (bench.M, bench.K) and Wv.dtype == np.uint16 and len(slots) == RB
    assert set(slots) <= {2, 4, 8} and len(set(slots)) == 3
    assert bench.K * sum(slots) * 8 <= 0.5 * bench.M * bench.K
    xf = gen.bf16_bits_to_f32(cfg["x"])
    a = xf @ gen.bf16_bits_to_f32(Wv).T
    imp = (a.astype(np.float64) ** 2).reshape(a.shape[0], RB, 64).mean(axis=(0, 2))
    assert slots == oracle.plan_slots([64 * bench.K] * RB, imp.tolist(), 0.5)
    order = np.argsort(imp)
    assert all(slots[order[i]] <= slots[order[i + 1]] for i in range(RB - 1))


def test_region_reports_assemble_from_synthetic_timings():
    """Every region report of the bench line assembles from timings alone (no
    GPU): each phase the bench times gets a synthetic per-call time, and the
    report carries the regions, their kernel times and JSON-clean values."""
    from types import SimpleNamespace
    phases = {
        "layer": ["usk_build", "usk_gemv", "usk_gemv_b4", "usk_gemm", "usk_gemv_multi"],
        "small": ["usk_build", "usk_gemv_f32x", "usk_gemv_bf16x"],
        "llama7b_set": ["%s/%s" % (s, c) for s in ("4096x4096", "11008x4096", "4096x11008")
                        for c in ("usk_build", "usk_gemv_b1", "usk_gemv_b4", "usk_gemm_b16", "usk_gemv_multi_b1",
                                  "usk_gemv_multi_b4")],
        "mlp70b": ["%s/%s" % (s, c) for s in ("28672x8192", "8192x28672")
                   for c in ("usk_build", "usk_gemv_b1", "usk_gemv_multi_b1", "usk_gemm_b16", "usk_gemm_b32",
                             "usk_gemm_b64")],
        "stack7b": ["model_build", "token_decode", "token_decode_grouped", "token_decode_concurrent",
                    "token_dense_bf16_torch"],
        "absmaxmin": ["usk_build", "usk_gemv", "usk_gemm"],
        "colshared": ["usk_build", "usk_gemv", "ab_hash_gemv", "ab_matrix_gemv"],
        "q4": ["usk_build", "usk_gemv", "usk_gemm"],
        "rates": ["slots_2/usk_build", "slots_2/usk_gemv", "slots_8/usk_build", "slots_8/usk_gemv"],
        "row_block_rates": ["usk_build", "usk_gemv", "usk_gemm"],
    }
    med = {r: {p: 1e-5 * (1 + i) for i, p in enumerate(ps)} for r, ps in phases.items()}
    times = {r: {p: [v, 1.1 * v] for p, v in d.items()} for r, d in med.items()}
    peaks = {"hbm_gbs": 6540.2, "bf16_tflops": 1645.9, "sm_max_mhz": 1965.0, "source": "measured"}
    rmap = SimpleNamespace(count=[22, 31, 11], code_bytes=bench.N_W // 16)
    out = bench.region_reports(med, times, bench.Roof(peaks), {}, 1, peaks, rmap)
    for region in ("small", "llama7b_set", "mlp70b", "stack7b", "absmaxmin", "colshared", "q4", "rates",
                   "row_block_rates"):
        assert region in out, region
    assert out["small"]["kernel_us"]["usk_build"] == pytest.approx(10.0)
    assert out["mlp70b"]["per_shape"]["28672x8192"]["rooflines"]["usk_gemm_b64"]["decode_roof_us"] > 0
    assert out["stack7b"]["token_decode_roofline"]["issue_roof_ms"] == pytest.approx(0.87, rel=0.01)
    json.dumps(out)
