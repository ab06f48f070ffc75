"""The column-shared projection sketch (format 3) on the GPU against the CPU oracle.

"UltraSketchLLM" explainer, Resumen Tecnico, Metodologia §4: W_hat = S . P^T with
a one-hot projection P shared by every row; the library multiplies it as
y = S (P^T x).  Builds are compared bit-exact; products run on sketches the
ORACLE built (uploaded) and must be within max|y - y_ref| <= 1e-3 max|y_ref| of
the oracle's float64 product, which sums w_hat[i][j] x[j] over the columns (the
definition, not the factorised form)."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, sketch_from_oracle, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3
CS = usk.FORMAT_COLSHARED


def _gpu_build(W, seed, status=None):
    sk = usk.usk_build(to_dev(W), None, seed, status=status, version=CS)
    torch.cuda.synchronize()
    return sk


def _compare_build(W, seed):
    o = oracle.build_sketch_cs(W, seed)
    assert o["status"] == oracle.OK
    st = status_tensor()
    sk = _gpu_build(W, seed, st)
    assert int(st.item()) == 0
    assert np.array_equal(scales_np(sk), o["scales"]), "scales differ"
    bad = np.nonzero(codes_np(sk) != o["codes"])[0]
    assert bad.size == 0, "codes differ at %d entries, first %s" % (bad.size, bad[:8])
    return o


def _oracle_sketch(W, seed):
    o = oracle.build_sketch_cs(W, seed)
    assert o["status"] == oracle.OK
    return sketch_from_oracle(o, W.shape[0], W.shape[1], seed, CS, 1), o


def _check_product(sk, o, x, rows=None, pdl=False):
    st = status_tensor()
    y = usk.usk_gemv(sk, to_dev(x), status=st, pdl=pdl).cpu().numpy()
    assert int(st.item()) == 0
    ref = oracle.gemv_cs_f64(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed, rows=rows)
    if rows is not None:
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e
    return y


SHAPES = [(64, 256), (128, 1024), (192, 2816), (64, 4352), (256, 512)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("wdtype", ["bf16", "f32"])
def test_cs_build_bit_exact(M, K, wdtype):
    for seed in (0, 4242):
        _compare_build(gen.weights_student_t(M, K, seed + 5, 4.0, 0.02, 0.001, 20.0, wdtype), seed)


def test_cs_build_ties_and_special_cases():
    g = np.random.default_rng(23)
    vals = np.float32([-0.03, -0.01, -0.0, 0.0, 0.01, 0.03])
    _compare_build(gen.f32_to_bf16_bits(vals[g.integers(0, 6, size=(256, 1024))]), 4)
    _compare_build(vals[g.integers(0, 6, size=(128, 768))].astype(np.float32), 5)
    _compare_build(np.zeros((64, 512), np.float32), 1)
    # truncation closed form of the oracle pins: row 0's bucket 0 all 2.0, rest 1.0
    W = np.ones((64, 256), np.float32)
    W[0, [oracle.cs_sigma(4, 0, k) for k in range(16)]] = 2.0
    o = _compare_build(W, 4)
    assert o["codes"][0] == 127 and np.all(o["codes"][1:] == 63)
    _compare_build(gen.f32_to_bf16_bits(W), 4)


@pytest.mark.parametrize("cluster", [1, 2, 3, 8])
def test_cs_build_geometry_independent(cluster):
    W = gen.weights_student_t(128, 4352, 6, 4.0, 0.02, 0.001, 20.0, "bf16")
    o = oracle.build_sketch_cs(W, 9)
    usk.usk_debug_set_geometry(cluster, 0)
    try:
        sk = _gpu_build(W, 9)
    finally:
        usk.usk_debug_set_geometry(0, 0)
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])


def test_cs_build_max_k():
    _compare_build(gen.weights_normal(64, 65536, 7, 0.02, "bf16"), 3)


def test_cs_layer_build_and_products():
    cfg = gen.layer(15)
    _compare_build(cfg["W"], cfg["seed"])
    sk, o = _oracle_sketch(cfg["W"], cfg["seed"])
    for b in (1, 4, 15):
        _check_product(sk, o, cfg["x"][:b])


def test_cs_mlp70b_build_and_products():
    cfg = gen.mlp70b("up", 16)
    W = cfg["W"]
    gsk = _gpu_build(W, cfg["seed"])
    sk, o = _oracle_sketch(W, cfg["seed"])
    assert np.array_equal(scales_np(gsk), o["scales"]) and np.array_equal(codes_np(gsk), o["codes"])
    del gsk
    M = W.shape[0]
    rows = np.array([0, 1, 63, 64, M // 2, M - 65, M - 1])
    _check_product(sk, o, cfg["x"][:1], rows=rows)
    _check_product(sk, o, cfg["x"][:8], rows=rows)


@pytest.mark.parametrize("M,K", [(64, 256), (192, 2816), (128, 4352), (64, 65536)])
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
@pytest.mark.parametrize("batch", [1, 2, 5, 8, 15])
def test_cs_gemv_matches_oracle(M, K, xdtype, batch):
    W = gen.weights_student_t(M, K, 31, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, 13)
    _check_product(sk, o, gen.activations(batch, K, 32, xdtype))


@pytest.mark.parametrize("tpb", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("rows", [64, 256])
def test_cs_gemv_geometries(tpb, rows):
    """Tiles per block (rounded down to a power of two, capped at 8 for
    256-row blocks) and rows per block; M = 320 is not a multiple of 256
    (partial last row group)."""
    W = gen.weights_student_t(320, 4352, 33, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, 14)
    usk.usk_debug_set_geometry(0, tpb)
    usk.usk_debug_set_gemv_rows(rows)
    try:
        for batch in (1, 7, 15):
            _check_product(sk, o, gen.activations(batch, 4352, 34, "bf16"))
    finally:
        usk.usk_debug_set_geometry(0, 0)
        usk.usk_debug_set_gemv_rows(0)


@pytest.mark.parametrize("M,K", [(320, 2816), (256, 11008), (8192, 4096), (64, 65536)])
def test_cs_gemv_more_shapes(M, K):
    """Ragged tile counts (11, 43), a tall matrix (automatic 256-row blocks) and
    the largest K (16 tiles per block)."""
    W = gen.weights_student_t(M, K, 37, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, 16)
    rows = None if M <= 320 else np.array([0, 1, 31, 32, 255, 256, M // 2 + 3, M - 1])
    for batch in (1, 2, 3, 9, 15):
        _check_product(sk, o, gen.activations(batch, K, 38, "bf16"), rows=rows)
    _check_product(sk, o, gen.activations(2, K, 39, "f32"), rows=rows)


def test_cs_gemv_repeatable_and_pdl():
    W = gen.weights_normal(512, 4096, 35, 0.02, "bf16")
    sk, o = _oracle_sketch(W, 15)
    x = to_dev(gen.activations(4, 4096, 36, "bf16"))
    a = usk.usk_gemv(sk, x)
    for _ in range(3):
        assert torch.equal(a, usk.usk_gemv(sk, x))
        assert torch.equal(a, usk.usk_gemv(sk, x, pdl=True))


def test_cs_magnitude_bound_through_gpu_product():
    """|w_hat| <= |w| (the MIN reduction) read back through the GPU product:
    one-hot x selects columns of W_hat."""
    cfg = gen.layer()
    W = cfg["W"]
    Wf = gen.bf16_bits_to_f32(W)
    sk = _gpu_build(W, cfg["seed"])
    K = W.shape[1]
    cols = np.array([0, 1, 255, 256, 1000, 2047, 3000, K - 1])
    x = np.zeros((8, K), np.float32)
    x[np.arange(8), cols] = 1.0
    y = usk.usk_gemv(sk, to_dev(gen.f32_to_bf16_bits(x))).cpu().numpy()
    for t, j in enumerate(cols):
        assert np.all(np.abs(y[t]) <= np.abs(Wf[:, j]))


def test_cs_flags_and_argument_errors():
    W = gen.weights_normal(64, 256, 1, 0.02, "f32")
    Wn = W.copy()
    Wn[5, 9] = np.nan
    st = status_tensor()
    _gpu_build(Wn, 0, st)
    assert int(st.item()) & usk.FLAG_NONFINITE_W
    st = status_tensor()
    _gpu_build(gen.f32_to_bf16_bits(Wn), 0, st)
    assert int(st.item()) & usk.FLAG_NONFINITE_W
    st = status_tensor()
    _gpu_build(np.full((64, 256), 1e9, np.float32), 0, st)
    assert int(st.item()) & usk.FLAG_SCALE_OVERFLOW
    Wd = to_dev(W)
    with pytest.raises(usk.UskError) as ei:
        usk.usk_build(Wd, torch.ones(256, dtype=torch.float32, device="cuda"), 0, version=CS)
    assert ei.value.status == 6
    with pytest.raises(usk.UskError) as ei:
        usk.usk_build(Wd, None, 0, version=CS, depth=2)
    assert ei.value.status == 6
    sk = _gpu_build(W, 0)
    with pytest.raises(usk.UskError) as ei:
        usk.usk_gemm(sk, to_dev(gen.activations(16, 256, 1, "bf16")))
    assert ei.value.status == 6
    with pytest.raises(usk.UskError) as ei:
        usk.usk_gemv(sk, to_dev(gen.activations(16, 256, 1, "bf16")))
    assert ei.value.status == 4


def test_cs_wait_timeouts_reported_then_recover():
    """Build: block (0, 0) skips a weight-tile copy; product: block 1 of the
    first row group skips its partial sums.  Each bounded wait gives up and
    sets the flag."""
    W = gen.weights_normal(64, 2048, 2, 0.02, "bf16")  # two blocks per row block in the product
    x = gen.activations(1, 2048, 3, "bf16")
    for kind in (1, 3):
        st = status_tensor()
        usk.usk_debug_inject_timeout(kind)
        try:
            if kind == 1:
                usk.usk_build(to_dev(W), None, 0, status=st, version=CS)
            else:
                sk, _ = _oracle_sketch(W, 0)
                usk.usk_gemv(sk, to_dev(x), status=st)
            torch.cuda.synchronize()
        finally:
            usk.usk_debug_inject_timeout(0)
        assert int(st.item()) & usk.FLAG_TIMEOUT
    o = _compare_build(W, 0)
    sk, o = _oracle_sketch(W, 0)
    _check_product(sk, o, x)
