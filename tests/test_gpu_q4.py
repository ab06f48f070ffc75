"""The 4-bit-code sketch (format 4) on the GPU against the CPU oracle.

"UltraSketchLLM" explainer, Resultados Experimentales: 0.5 bit/weight with 4-bit
quantisation -- here 8 weights per bucket and a signed 4-bit code each, with the
format-1 selection rule.  Builds are compared bit-exact; products run on sketches
the ORACLE built (uploaded) and must be within max|y - y_ref| <= 1e-3 max|y_ref|
of the oracle's float64 product."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, sketch_from_oracle, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3
Q4 = usk.FORMAT_Q4


def _gpu_build(W, imp, seed, status=None):
    sk = usk.usk_build(to_dev(W), None if imp is None else to_dev(imp), seed, status=status, version=Q4)
    torch.cuda.synchronize()
    return sk


def _compare_build(W, imp, seed):
    o = oracle.build_sketch_q4(W, imp, seed)
    assert o["status"] == oracle.OK
    st = status_tensor()
    sk = _gpu_build(W, imp, seed, st)
    assert int(st.item()) == 0
    assert np.array_equal(scales_np(sk), o["scales"]), "scales differ"
    bad = np.nonzero(codes_np(sk) != o["codes"])[0]
    assert bad.size == 0, "code bytes differ at %d, first %s" % (bad.size, bad[:8])


def _oracle_sketch(W, imp, seed):
    o = oracle.build_sketch_q4(W, imp, seed)
    assert o["status"] == oracle.OK
    return sketch_from_oracle(o, W.shape[0], W.shape[1], seed, Q4, 1), o


def _check_product(sk, o, x, rows=None, gemm=False):
    st = status_tensor()
    xd = to_dev(x)
    y = (usk.usk_gemm(sk, xd, status=st) if gemm else usk.usk_gemv(sk, xd, status=st)).cpu().numpy()
    assert int(st.item()) == 0
    ref = oracle.gemv_q4_f64(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed, rows=rows)
    if rows is not None:
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e


SHAPES = [(64, 256), (128, 1024), (192, 2816), (64, 4352), (256, 512)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("wdtype", ["bf16", "f32"])
@pytest.mark.parametrize("with_imp", [False, True])
def test_q4_build_bit_exact(M, K, wdtype, with_imp):
    for seed in (0, 31337):
        W = gen.weights_student_t(M, K, seed + 7, 4.0, 0.02, 0.001, 20.0, wdtype)
        imp = gen.importance_lognormal(K, seed + 7) if with_imp else None
        _compare_build(W, imp, seed)


def test_q4_build_ties_and_special_cases():
    g = np.random.default_rng(29)
    vals = np.float32([-0.03, -0.01, -0.0, 0.0, 0.01, 0.03])
    Wt = gen.f32_to_bf16_bits(vals[g.integers(0, 6, size=(256, 1024))])
    _compare_build(Wt, None, 4)
    _compare_build(Wt, np.ones(1024, np.float32), 4)
    _compare_build(vals[g.integers(0, 6, size=(128, 768))].astype(np.float32), None, 5)
    _compare_build(np.zeros((64, 512), np.float32), None, 1)
    # half-way quotients: one 7 s weight fixes s = 2^-4, the rest 2.5 s -> code 2
    W = np.full((64, 256), np.float32(2.5 / 16), np.float32)
    W[0, 0] = np.float32(7 / 16)
    _compare_build(W, None, 0)


@pytest.mark.parametrize("cluster", [1, 2, 3, 8])
def test_q4_build_geometry_independent(cluster):
    W = gen.weights_student_t(128, 4352, 8, 4.0, 0.02, 0.001, 20.0, "bf16")
    imp = gen.importance_lognormal(4352, 8)
    o = oracle.build_sketch_q4(W, imp, 9)
    usk.usk_debug_set_geometry(cluster, 0)
    try:
        sk = _gpu_build(W, imp, 9)
    finally:
        usk.usk_debug_set_geometry(0, 0)
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])


def test_q4_layer_build_and_products():
    cfg = gen.layer(16)
    _compare_build(cfg["W"], cfg["importance"], cfg["seed"])
    sk, o = _oracle_sketch(cfg["W"], cfg["importance"], cfg["seed"])
    _check_product(sk, o, cfg["x"][:1])
    _check_product(sk, o, cfg["x"][:4])
    _check_product(sk, o, cfg["x"], gemm=True)


def test_q4_mlp70b_build_and_products():
    cfg = gen.mlp70b("up", 64)
    W = cfg["W"]
    gsk = _gpu_build(W, None, cfg["seed"])
    sk, o = _oracle_sketch(W, None, cfg["seed"])
    assert np.array_equal(scales_np(gsk), o["scales"]) and np.array_equal(codes_np(gsk), o["codes"])
    del gsk
    M = W.shape[0]
    rows = np.array([0, 1, 127, 128, M // 2, M - 65, M - 1])
    _check_product(sk, o, cfg["x"][:1], rows=rows)
    _check_product(sk, o, cfg["x"][:16], rows=rows, gemm=True)
    _check_product(sk, o, cfg["x"], rows=rows, gemm=True)


@pytest.mark.parametrize("M,K", [(64, 256), (192, 2816), (128, 4352)])
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
@pytest.mark.parametrize("batch", [1, 3, 8, 9, 15])
def test_q4_gemv_matches_oracle(M, K, xdtype, batch):
    W = gen.weights_student_t(M, K, 41, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 6)
    _check_product(sk, o, gen.activations(batch, K, 42, xdtype))


@pytest.mark.parametrize("path", [1, 2, 3, 4])
def test_q4_gemv_paths(path):
    """Forced paths: the integer paths (2, 3) read 8-bit codes only, so a 4-bit
    sketch falls back to a bf16 path."""
    W = gen.weights_student_t(128, 1024, 43, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 8)
    usk.usk_debug_set_gemv_path(path)
    try:
        for batch in (1, 4):
            _check_product(sk, o, gen.activations(batch, 1024, 44, "bf16"))
    finally:
        usk.usk_debug_set_gemv_path(0)


@pytest.mark.parametrize("tpc", [1, 2, 3, 8])
def test_q4_gemv_geometries(tpc):
    W = gen.weights_student_t(128, 4352, 45, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 10)
    usk.usk_debug_set_geometry(0, tpc)
    try:
        for batch in (1, 5, 12):
            _check_product(sk, o, gen.activations(batch, 4352, 46, "bf16"))
    finally:
        usk.usk_debug_set_geometry(0, 0)


@pytest.mark.parametrize("M,K", [(128, 256), (192, 1024), (320, 2048), (128, 4352)])
@pytest.mark.parametrize("batch", [16, 64, 256])
def test_q4_gemm_matches_oracle(M, K, batch):
    W = gen.weights_student_t(M, K, 47, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 12)
    _check_product(sk, o, gen.activations(batch, K, 48, "bf16"), gemm=True)


def test_q4_flags_errors_and_timeouts():
    W = gen.weights_normal(64, 256, 1, 0.02, "f32")
    Wn = W.copy()
    Wn[5, 9] = np.inf
    st = status_tensor()
    _gpu_build(Wn, None, 0, st)
    assert int(st.item()) & usk.FLAG_NONFINITE_W
    st = status_tensor()
    _gpu_build(np.full((64, 256), 1e6, np.float32), None, 0, st)
    assert int(st.item()) & usk.FLAG_SCALE_OVERFLOW
    with pytest.raises(usk.UskError) as ei:
        usk.usk_build(to_dev(W), None, 0, version=Q4, depth=2)
    assert ei.value.status == 6
    # injected waits that give up, then clean results
    Wb = gen.weights_normal(128, 2048, 2, 0.02, "bf16")
    x1 = gen.activations(1, 2048, 3, "bf16")
    x16 = gen.activations(16, 2048, 3, "bf16")
    sk, o = _oracle_sketch(Wb, None, 0)
    for kind, fn in ((1, lambda s: usk.usk_build(to_dev(Wb), None, 0, status=s, version=Q4)),
                     (2, lambda s: usk.usk_gemm(sk, to_dev(x16), status=s)),
                     (3, lambda s: usk.usk_gemv(sk, to_dev(x1), status=s))):
        st = status_tensor()
        usk.usk_debug_inject_timeout(kind)
        try:
            fn(st)
            torch.cuda.synchronize()
        finally:
            usk.usk_debug_inject_timeout(0)
        assert int(st.item()) & usk.FLAG_TIMEOUT
    _compare_build(Wb, None, 0)
    _check_product(sk, o, x1)
    _check_product(sk, o, x16, gemm=True)
