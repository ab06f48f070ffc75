"""The multi-row AbsMaxMin sketch (format 2) on the GPU against the CPU oracle.

"UltraSketchLLM" explainer, Resumen Tecnico, Metodologia §1: a bucket keeps its
member of smallest magnitude, decompression takes the largest magnitude over
the hash rows.  Builds are compared bit-exact; products run on sketches the
ORACLE built (uploaded), within max|y - y_ref| <= 1e-3 max|y_ref| of the
oracle's float64 product; and the rebuilt weights obey the paper's bound
|w_hat| <= |w| at the full layer size (one-hot x reads columns of W_hat)."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3
AMM = usk.FORMAT_ABSMAXMIN


def _gpu_build(W, seed, depth, status=None):
    sk = usk.usk_build(to_dev(W), None, seed, status=status, version=AMM, depth=depth)
    torch.cuda.synchronize()
    return sk


def _compare_build(W, seed, depth):
    o = oracle.build_sketch_amm(W, seed, depth)
    assert o["status"] == oracle.OK
    st = status_tensor()
    sk = _gpu_build(W, seed, depth, st)
    assert int(st.item()) == 0
    assert np.array_equal(scales_np(sk), o["scales"]), "scales differ"
    bad = np.nonzero(codes_np(sk) != o["codes"])[0]
    assert bad.size == 0, "codes differ at %d buckets, first %s" % (bad.size, bad[:8])


def _oracle_sketch(W, seed, depth):
    """Sketch built by the oracle, uploaded: the products' expected values never
    depend on the CUDA build."""
    o = oracle.build_sketch_amm(W, seed, depth)
    assert o["status"] == oracle.OK
    M, K = W.shape
    codes = torch.from_numpy(o["codes"].copy()).cuda()
    scales = torch.from_numpy(o["scales"].view(np.int16).copy()).cuda()
    return usk.Sketch(M, K, seed, codes, scales, AMM, depth), o


def _check_product(sk, o, x, rows=None, gemm=False):
    st = status_tensor()
    xd = to_dev(x)
    y = (usk.usk_gemm(sk, xd, status=st) if gemm else usk.usk_gemv(sk, xd, status=st)).cpu().numpy()
    assert int(st.item()) == 0
    ref = oracle.gemv_amm_f64(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed, sk.depth, rows=rows)
    if rows is not None:
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e


# several tiles, clusters of 1..8 blocks, uneven tiles per block (11 and 17 tiles)
SHAPES = [(64, 256), (128, 1024), (192, 2816), (64, 4352), (256, 512)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("wdtype", ["bf16", "f32"])
@pytest.mark.parametrize("depth", [1, 2, 4])
def test_amm_build_bit_exact(M, K, wdtype, depth):
    for seed in (0, 777):
        W = gen.weights_student_t(M, K, seed + 3, 4.0, 0.02, 0.001, 20.0, wdtype)
        _compare_build(W, seed, depth)


@pytest.mark.parametrize("depth", [1, 2, 4])
def test_amm_build_ties_heavy(depth):
    g = np.random.default_rng(19)
    vals = np.float32([-0.03, -0.01, -0.0, 0.0, 0.01, 0.03])
    _compare_build(gen.f32_to_bf16_bits(vals[g.integers(0, 6, size=(256, 1024))]), 4, depth)
    _compare_build(vals[g.integers(0, 6, size=(128, 768))].astype(np.float32), 5, depth)


def test_amm_build_special_cases():
    _compare_build(np.zeros((64, 512), np.float32), 1, 2)
    _compare_build(np.ones((128, 256), np.float32), 2, 4)
    # the truncation closed form of the oracle pins: one row-0 bucket all 2.0
    W = np.ones((64, 256), np.float32)
    target = oracle.amm_bucket_index(256, 1, 2, 0, 0, 0)
    for i in range(64):
        for j in range(256):
            if oracle.amm_bucket_index(256, 1, 2, 0, i, j) == target:
                W[i, j] = 2.0
    _compare_build(W, 1, 2)
    _compare_build(gen.f32_to_bf16_bits(W), 1, 2)


@pytest.mark.parametrize("cluster", [1, 2, 3, 8])
def test_amm_build_geometry_independent(cluster):
    W = gen.weights_student_t(128, 4352, 5, 4.0, 0.02, 0.001, 20.0, "bf16")
    o = oracle.build_sketch_amm(W, 9, 2)
    usk.usk_debug_set_geometry(cluster, 0)
    try:
        sk = _gpu_build(W, 9, 2)
    finally:
        usk.usk_debug_set_geometry(0, 0)
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])


@pytest.mark.parametrize("depth", [2, 4])
def test_amm_build_layer_workload_full(depth):
    cfg = gen.layer()
    _compare_build(cfg["W"], cfg["seed"], depth)


def test_amm_build_flags_and_argument_errors():
    W = gen.weights_normal(64, 256, 1, 0.02, "f32")
    Wn = W.copy()
    Wn[5, 9] = np.nan
    st = status_tensor()
    _gpu_build(Wn, 0, 2, st)
    assert int(st.item()) & usk.FLAG_NONFINITE_W
    Wb = gen.f32_to_bf16_bits(Wn)
    st = status_tensor()
    _gpu_build(Wb, 0, 4, st)
    assert int(st.item()) & usk.FLAG_NONFINITE_W
    st = status_tensor()
    _gpu_build(np.full((64, 256), 1e9, np.float32), 0, 2, st)
    assert int(st.item()) & usk.FLAG_SCALE_OVERFLOW
    Wd = to_dev(W)
    imp = torch.ones(256, dtype=torch.float32, device="cuda")
    for kwargs in ({"version": AMM, "depth": 3}, {"version": AMM, "depth": 0}, {"version": 1, "depth": 2},
                   {"version": 9, "depth": 1}):
        with pytest.raises(usk.UskError) as ei:
            usk.usk_build(Wd, None, 0, **kwargs)
        assert ei.value.status == 6
    with pytest.raises(usk.UskError) as ei:
        usk.usk_build(Wd, imp, 0, version=AMM, depth=2)
    assert ei.value.status == 6
    sk = _gpu_build(W, 0, 2)
    bad = usk.Sketch(sk.M, sk.K, sk.seed, sk.codes, sk.scales, AMM, 3)
    with pytest.raises(usk.UskError):
        usk.usk_gemv(bad, to_dev(gen.activations(1, 256, 1, "bf16")))


GEMV_SHAPES = [(64, 256), (192, 2816), (128, 4352)]


@pytest.mark.parametrize("M,K", GEMV_SHAPES)
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
@pytest.mark.parametrize("batch", [1, 3, 8, 9, 15])
@pytest.mark.parametrize("depth", [1, 2, 4])
def test_amm_gemv_matches_oracle(M, K, xdtype, batch, depth):
    W = gen.weights_student_t(M, K, 21, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, 6, depth)
    _check_product(sk, o, gen.activations(batch, K, 22, xdtype))


@pytest.mark.parametrize("path", [1, 2, 3, 4])
@pytest.mark.parametrize("depth", [1, 2, 4])
def test_amm_gemv_paths(path, depth):
    """Forced paths: the integer paths (2, 3) serve single-row sketches; for
    depth > 1 the library falls back to a bf16 path."""
    W = gen.weights_student_t(128, 1024, 23, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, 8, depth)
    usk.usk_debug_set_gemv_path(path)
    try:
        for batch in (1, 4):
            _check_product(sk, o, gen.activations(batch, 1024, 24, "bf16"))
    finally:
        usk.usk_debug_set_gemv_path(0)


@pytest.mark.parametrize("tpc", [1, 2, 3, 8])
@pytest.mark.parametrize("depth", [2, 4])
def test_amm_gemv_geometries(tpc, depth):
    W = gen.weights_student_t(128, 4352, 25, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, 10, depth)
    usk.usk_debug_set_geometry(0, tpc)
    try:
        for batch in (1, 5):
            _check_product(sk, o, gen.activations(batch, 4352, 26, "bf16"))
    finally:
        usk.usk_debug_set_geometry(0, 0)


@pytest.mark.parametrize("M,K", [(128, 256), (192, 1024), (320, 2048), (128, 4352)])
@pytest.mark.parametrize("batch", [16, 64, 256])
@pytest.mark.parametrize("depth", [1, 2, 4])
def test_amm_gemm_matches_oracle(M, K, batch, depth):
    W = gen.weights_student_t(M, K, 27, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, 12, depth)
    _check_product(sk, o, gen.activations(batch, K, 28, "bf16"), gemm=True)


@pytest.mark.parametrize("depth", [2, 4])
def test_amm_layer_workload_products(depth):
    """The 4096 x 4096 layer: GEMV at batch 1 and 4 on every output, GEMM at 16."""
    cfg = gen.layer(16)
    sk, o = _oracle_sketch(cfg["W"], cfg["seed"], depth)
    _check_product(sk, o, cfg["x"][:1])
    _check_product(sk, o, cfg["x"][:4])
    _check_product(sk, o, cfg["x"], gemm=True)


def test_amm_mlp70b_build_and_products():
    """28672 x 8192 at depth 2: the whole build bit-exact; GEMV at 1 and GEMM at
    16 and 64 on sampled rows of the oracle's sketch."""
    cfg = gen.mlp70b("up", 64)
    W = cfg["W"]
    gsk = _gpu_build(W, cfg["seed"], 2)
    sk, o = _oracle_sketch(W, cfg["seed"], 2)
    assert np.array_equal(scales_np(gsk), o["scales"]) and np.array_equal(codes_np(gsk), o["codes"])
    del gsk
    M = W.shape[0]
    rows = np.array([0, 1, 127, 128, M // 2, M - 65, M - 1])
    _check_product(sk, o, cfg["x"][:1], rows=rows)
    _check_product(sk, o, cfg["x"][:16], rows=rows, gemm=True)
    _check_product(sk, o, cfg["x"], rows=rows, gemm=True)


@pytest.mark.parametrize("depth", [1, 2, 4])
def test_amm_magnitude_bound_through_gpu_products(depth):
    """|w_hat| <= |w| for every weight (Metodologia §1), read back through the
    GPU path: one-hot rows of x select columns of W_hat (GEMV and GEMM)."""
    cfg = gen.layer()
    W = cfg["W"]
    Wf = gen.bf16_bits_to_f32(W)
    sk = _gpu_build(W, cfg["seed"], depth)
    K = W.shape[1]
    cols = np.array([0, 1, 255, 256, 1000, 2047, 3000, K - 1])
    x = np.zeros((16, K), np.float32)
    x[np.arange(8), cols] = 1.0
    x[8 + np.arange(8), cols[::-1]] = 1.0
    xb = gen.f32_to_bf16_bits(x)
    y8 = usk.usk_gemv(sk, to_dev(xb[:8])).cpu().numpy()
    y16 = usk.usk_gemm(sk, to_dev(xb)).cpu().numpy()
    for t, j in enumerate(cols):
        assert np.all(np.abs(y8[t]) <= np.abs(Wf[:, j]))
        assert np.array_equal(y16[t], y8[t])
        assert np.array_equal(y16[15 - t], y8[t])


def test_amm_build_wait_timeout_reported_then_recovers():
    W = gen.weights_normal(64, 256, 1, 0.02, "bf16")
    st = status_tensor()
    usk.usk_debug_inject_timeout(1)
    try:
        usk.usk_build(to_dev(W), None, 0, status=st, version=AMM, depth=2)
        torch.cuda.synchronize()
    finally:
        usk.usk_debug_inject_timeout(0)
    assert int(st.item()) & usk.FLAG_TIMEOUT
    _compare_build(W, 0, 2)
