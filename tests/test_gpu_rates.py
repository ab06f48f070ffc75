"""Importance-aware space allocation on the GPU: format-1 sketches at 2 and 8
hash slots per class (0.25 and 1 bit/weight) against the CPU oracle, and a model
of layers whose rates come from the allocation ("UltraSketchLLM" explainer,
Resumen Tecnico, Metodologia §2).  Builds bit-exact; products on ORACLE-built
sketches within max|y - y_ref| <= 1e-3 max|y_ref|."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, sketch_from_oracle, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3
V1 = usk.FORMAT_MAXKEY


def _gpu_build(W, imp, seed, slots, status=None):
    sk = usk.usk_build(to_dev(W), None if imp is None else to_dev(imp), seed, status=status, version=V1, slots=slots)
    torch.cuda.synchronize()
    return sk


def _compare_build(W, imp, seed, slots):
    o = oracle.build_sketch_rate(W, imp, seed, slots)
    assert o["status"] == oracle.OK
    st = status_tensor()
    sk = _gpu_build(W, imp, seed, slots, st)
    assert int(st.item()) == 0
    assert np.array_equal(scales_np(sk), o["scales"]), "scales differ"
    bad = np.nonzero(codes_np(sk) != o["codes"])[0]
    assert bad.size == 0, "codes differ at %d, first %s" % (bad.size, bad[:8])


def _oracle_sketch(W, imp, seed, slots):
    o = oracle.build_sketch_rate(W, imp, seed, slots)
    assert o["status"] == oracle.OK
    sk = sketch_from_oracle(o, W.shape[0], W.shape[1], seed, V1, 1)
    sk.slots = slots
    return sk, o


def _check_product(sk, o, x, rows=None, gemm=False):
    st = status_tensor()
    xd = to_dev(x)
    y = (usk.usk_gemm(sk, xd, status=st) if gemm else usk.usk_gemv(sk, xd, status=st)).cpu().numpy()
    assert int(st.item()) == 0
    ref = oracle.gemv_rate_f64(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed, sk.slots, rows=rows)
    if rows is not None:
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e


SHAPES = [(64, 256), (128, 1024), (192, 2816), (64, 4352), (256, 512)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("wdtype", ["bf16", "f32"])
@pytest.mark.parametrize("with_imp", [False, True])
@pytest.mark.parametrize("slots", [2, 8])
def test_rate_build_bit_exact(M, K, wdtype, with_imp, slots):
    seed = 99 + slots
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.001, 20.0, wdtype)
    imp = gen.importance_lognormal(K, seed) if with_imp else None
    _compare_build(W, imp, seed, slots)


@pytest.mark.parametrize("slots", [2, 8])
def test_rate_build_ties_geometry_and_layer(slots):
    g = np.random.default_rng(37)
    vals = np.float32([-0.03, -0.01, -0.0, 0.0, 0.01, 0.03])
    _compare_build(gen.f32_to_bf16_bits(vals[g.integers(0, 6, size=(256, 1024))]), None, 4, slots)
    W = gen.weights_student_t(128, 4352, 8, 4.0, 0.02, 0.001, 20.0, "bf16")
    o = oracle.build_sketch_rate(W, None, 9, slots)
    for cluster in (1, 3, 8):
        usk.usk_debug_set_geometry(cluster, 0)
        try:
            sk = _gpu_build(W, None, 9, slots)
        finally:
            usk.usk_debug_set_geometry(0, 0)
        assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])
    cfg = gen.layer(16)
    _compare_build(cfg["W"], cfg["importance"], cfg["seed"], slots)


@pytest.mark.parametrize("slots", [2, 8])
@pytest.mark.parametrize("M,K", [(64, 256), (192, 2816), (128, 4352)])
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
def test_rate_gemv_matches_oracle(slots, M, K, xdtype):
    W = gen.weights_student_t(M, K, 51, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 6, slots)
    for batch in (1, 4, 9, 15):
        _check_product(sk, o, gen.activations(batch, K, 52, xdtype))


@pytest.mark.parametrize("slots", [2, 8])
@pytest.mark.parametrize("path", [1, 2, 3, 4])
def test_rate_gemv_paths(slots, path):
    """The integer paths (2, 3) read 4-slot layouts only; other slot counts fall
    back to a bf16 path."""
    W = gen.weights_student_t(128, 1024, 53, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 8, slots)
    usk.usk_debug_set_gemv_path(path)
    try:
        for batch in (1, 4):
            _check_product(sk, o, gen.activations(batch, 1024, 54, "bf16"))
    finally:
        usk.usk_debug_set_gemv_path(0)


@pytest.mark.parametrize("slots", [2, 8])
@pytest.mark.parametrize("M,K", [(128, 256), (192, 1024), (320, 2048), (128, 4352)])
@pytest.mark.parametrize("batch", [16, 64, 256])
def test_rate_gemm_matches_oracle(slots, M, K, batch):
    W = gen.weights_student_t(M, K, 55, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 12, slots)
    _check_product(sk, o, gen.activations(batch, K, 56, "bf16"), gemm=True)


def test_rate_allocation_over_the_7b_layer_set():
    """Seven linears, importance = mean calibration E[a^2] of each input times a
    per-linear weight (front FFN layers most sensitive, as the page reports);
    the allocation at 0.5 bit/weight gives each layer 2, 4 or 8 slots, the
    sketches fit the budget and every product matches the oracle."""
    names = gen.LLAMA7B_ORDER
    sens = {"q": 1.0, "k": 1.0, "v": 1.0, "o": 1.0, "gate": 3.0, "up": 3.0, "down": 0.5}
    weights, imps = [], []
    for name in names:
        M, K = gen.LLAMA7B_SHAPES[name]
        weights.append(M * K)
        ea2 = float(np.mean(gen.importance_calibration(K, 2 + names.index(name)) ** 2))
        imps.append(ea2 * sens[name])
    slots = usk.usk_plan_slots(weights, imps, 0.5)
    assert slots == oracle.plan_slots(weights, imps, 0.5)
    assert sum(w * s / 8 for w, s in zip(weights, slots)) <= 0.5 * sum(weights)
    total_bytes = 0
    for name, s in zip(names, slots):
        cfg = gen.llama7b_layer(name, 4)
        W = cfg["W"]
        sk = _gpu_build(W, None, cfg["seed"], s)
        total_bytes += sk.codes.numel()
        o = oracle.build_sketch_rate(W, None, cfg["seed"], s)
        assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])
        M = W.shape[0]
        _check_product(sk, o, cfg["x"][:1], rows=np.array([0, 63, 64, M // 2, M - 1]))
    assert total_bytes * 8 <= 0.5 * sum(weights)


def test_rate_flags_and_errors():
    W = gen.weights_normal(64, 256, 1, 0.02, "f32")
    Wn = W.copy()
    Wn[3, 4] = np.nan
    for slots in (2, 8):
        st = status_tensor()
        _gpu_build(Wn, None, 0, slots, st)
        assert int(st.item()) & usk.FLAG_NONFINITE_W
    with pytest.raises(usk.UskError) as ei:
        usk.usk_build(to_dev(W), None, 0, version=V1, slots=3)
    assert ei.value.status == 6
    with pytest.raises(usk.UskError) as ei:
        usk.usk_build(to_dev(W), None, 0, version=usk.FORMAT_ABSMAXMIN, depth=2, slots=8)
    assert ei.value.status == 6
