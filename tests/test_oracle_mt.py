"""The oracle's all-core mode (row blocks spread over host threads) returns
exactly what the single-thread oracle returns: same codes, scales, status and
float64 products, for any thread count.  Row blocks are independent in the
method (every bucket's members lie in one 64-row block and the scale is per
block: "UltraSketchLLM" explainer, Metodologia §1), so any difference is a bug
in the threading wrapper."""
import numpy as np
import pytest

import gen
import oracle


@pytest.mark.parametrize("threads", [1, 3, 8])
@pytest.mark.parametrize("shape,dtype,with_imp", [
    ((64, 256), "bf16", False),
    ((320, 768), "bf16", True),
    ((256, 1024), "f32", True),
    ((1024, 512), "bf16", False),
])
def test_build_mt_identical(shape, dtype, with_imp, threads):
    M, K = shape
    W = gen.weights_student_t(M, K, 11, 4.0, 0.02, 0.01, 20.0, dtype)
    imp = gen.importance_lognormal(K, 11) if with_imp else None
    a = oracle.build_sketch(W, imp, 99)
    b = oracle.build_sketch_mt(W, imp, 99, threads=threads)
    assert a["status"] == b["status"] == 0
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scales"], b["scales"])


def test_build_mt_status_matches_sequential():
    """A non-finite weight in a late row block and a scale overflow in an early
    one: the sequential scan reports the non-finite weight; so must the
    all-core mode.  Each alone is reported as such."""
    M, K = 256, 256
    W = gen.weights_normal(M, K, 5, 0.02, "f32")
    W[10, 3] = 3e38  # row block 0: max|v|/127 overflows binary16
    W2 = W.copy()
    W2[200, 7] = np.nan  # row block 3
    for Wt in (W, W2):
        a = oracle.build_sketch(Wt, None, 1)
        b = oracle.build_sketch_mt(Wt, None, 1, threads=4)
        assert a["status"] == b["status"]
        assert np.array_equal(a["scales"], b["scales"])
    assert oracle.build_sketch_mt(W, None, 1)["status"] == oracle.ERR_SCALE_OVERFLOW
    assert oracle.build_sketch_mt(W2, None, 1)["status"] == oracle.ERR_NONFINITE
    bad = np.ones(K, dtype=np.float32)
    bad[5] = -1.0
    assert oracle.build_sketch_mt(W, bad, 1)["status"] == oracle.ERR_IMPORTANCE


@pytest.mark.parametrize("batch", [1, 4, 17])
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
def test_gemv_mt_identical(batch, xdtype):
    M, K = 384, 512
    W = gen.weights_normal(M, K, 6, 0.02, "bf16")
    o = oracle.build_sketch(W, None, 3)
    x = gen.activations(batch, K, 6, xdtype)
    y1 = oracle.gemv_f64(o["codes"], o["scales"], M, K, x, 3)
    y2 = oracle.gemv_f64_mt(o["codes"], o["scales"], M, K, x, 3, threads=5)
    assert y1.shape == y2.shape == (batch, M)
    assert np.array_equal(y1, y2)


def test_threads_reported():
    assert oracle.threads(3) == 3
    assert oracle.threads(0) >= 1
