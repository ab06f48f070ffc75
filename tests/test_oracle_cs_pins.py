"""Pins of the format-3 oracle (the column-shared projection, W_hat = S . P^T)
against things other than itself (CPU only).

"UltraSketchLLM" explainer, Resumen Tecnico, Metodologia §4: compression is a
matrix product with a projection P whose reduction is a MIN over absolute
values; decompression is the plain product W_hat = S . P^T.  Each test names what
fixes its expected value: the bijection property of the column lists, the
independent brute force of tests/brute_force.py (member lists, exact rational
quantisation), the matrix identity W_hat = S . P^T with an explicit one-hot P
built in numpy, the magnitude bound, or a closed form.
"""
import numpy as np
import pytest

import gen
import oracle
from tests import brute_force


def test_sigma_is_a_bijection():
    for seed in (0, 1, 2**63 + 11, 12345):
        for tc in (0, 1, 7, 255, 4095):
            assert sorted(oracle.cs_sigma(seed, tc, u) for u in range(256)) == list(range(256))


def test_buckets_hold_exactly_sixteen_columns_of_their_tile():
    K, seed = 1024, 9
    b = np.array([oracle.cs_bucket(K, seed, j) for j in range(K)])
    for tc in range(K // 256):
        tile = b[256 * tc:256 * (tc + 1)]
        assert np.all((tile >= 16 * tc) & (tile < 16 * tc + 16))
        assert np.all(np.bincount(tile - 16 * tc, minlength=16) == 16)
    # column j of bucket b sits at position u of sigma's list with u // 16 == b'
    for j in range(0, K, 37):
        tc, c = divmod(j, 256)
        u = [oracle.cs_sigma(seed, tc, v) for v in range(256)].index(c)
        assert b[j] == 16 * tc + u // 16


@pytest.mark.parametrize("M,K", [(64, 256), (128, 512), (64, 1024)])
@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
def test_build_matches_brute_force(M, K, wdtype):
    seed = 3 + M + K
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, wdtype)
    o = oracle.build_sketch_cs(W, seed, want_winners=True)
    assert o["status"] == oracle.OK
    codes, scales, winner = brute_force.build_cs(W, seed)
    assert np.array_equal(o["winner"], winner)
    assert np.array_equal(o["scales"], scales)
    assert np.array_equal(o["codes"], codes)


def test_ties_heavy_matches_brute_force():
    g = np.random.default_rng(31)
    vals = np.float32([-0.03, -0.01, 0.0, 0.01, 0.03])
    W = gen.f32_to_bf16_bits(vals[g.integers(0, 5, size=(128, 512))])
    o = oracle.build_sketch_cs(W, 2, want_winners=True)
    codes, scales, winner = brute_force.build_cs(W, 2)
    assert np.array_equal(o["winner"], winner)
    assert np.array_equal(o["codes"], codes) and np.array_equal(o["scales"], scales)


def _projection(K, seed):
    """Explicit one-hot P [K, K/16] (numpy), from the bucket of every column."""
    P = np.zeros((K, K // 16), np.float64)
    for j in range(K):
        P[j, oracle.cs_bucket(K, seed, j)] = 1.0
    return P


def test_decode_is_s_times_p_transpose():
    # W_hat = S . P^T with S = codes * block scale (Metodologia §4)
    M, K, seed = 128, 768, 5
    W = gen.weights_normal(M, K, seed, 0.02, "bf16")
    o = oracle.build_sketch_cs(W, seed)
    s = o["scales"].view(np.float16).astype(np.float64)
    S = o["codes"].reshape(M, K // 16).astype(np.float64) * np.repeat(s, 64)[:, None]
    ref = S @ _projection(K, seed).T
    assert np.array_equal(oracle.decode_cs(o["codes"], o["scales"], M, K, seed).astype(np.float64), ref)


@pytest.mark.parametrize("xdtype", ["f32", "bf16"])
def test_gemv_equals_s_times_pt_x(xdtype):
    # y = W_hat x = S (P^T x): the bucket sums of x times the dense code matrix
    M, K, seed = 128, 1024, 6
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, "bf16")
    o = oracle.build_sketch_cs(W, seed)
    x = gen.activations(3, K, seed, xdtype)
    xf = (gen.bf16_bits_to_f32(x) if xdtype == "bf16" else x).astype(np.float64)
    s = o["scales"].view(np.float16).astype(np.float64)
    S = o["codes"].reshape(M, K // 16).astype(np.float64) * np.repeat(s, 64)[:, None]
    z = xf @ _projection(K, seed)           # [batch, K/16] bucket sums
    ref = z @ S.T
    y = oracle.gemv_cs_f64(o["codes"], o["scales"], M, K, x, seed)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    rows = np.array([0, 63, 64, 127])
    assert np.array_equal(oracle.gemv_cs_f64(o["codes"], o["scales"], M, K, x, seed, rows=rows), y[:, rows])


@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
def test_magnitude_bound_every_weight(wdtype):
    M, K, seed = 128, 1024, 7
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, wdtype)
    Wf = gen.bf16_bits_to_f32(W) if wdtype == "bf16" else W
    o = oracle.build_sketch_cs(W, seed)
    Wh = oracle.decode_cs(o["codes"], o["scales"], M, K, seed)
    assert np.all(np.abs(Wh.astype(np.float64)) <= np.abs(Wf.astype(np.float64)))


def test_truncation_not_rounding_closed_form():
    # |w| = 1 everywhere except the 16 columns of row 0's bucket 0 (all 2.0):
    # S[0][0] = 2, every other entry 1; s16 = f16(2/127) = 1032 * 2^-16, so the
    # toward-zero codes are 127 and 63 (rounding would give 64)
    M, K, seed = 64, 256, 4
    W = np.ones((M, K), np.float32)
    cols = [oracle.cs_sigma(seed, 0, k) for k in range(16)]
    W[0, cols] = 2.0
    o = oracle.build_sketch_cs(W, seed)
    assert float(np.uint16(o["scales"][0]).view(np.float16)) == 1032 * 2.0**-16
    c = o["codes"].reshape(M, K // 16)
    assert c[0, 0] == 127
    assert np.all(c.reshape(-1)[1:] == 63)


def test_equal_magnitudes_keep_smallest_column():
    M, K, seed = 64, 512, 8
    g = np.random.default_rng(2)
    W = np.where(g.random((M, K)) < 0.5, -0.5, 0.5).astype(np.float32)
    o = oracle.build_sketch_cs(W, seed, want_winners=True)
    nb = K // 16
    for i in range(0, M, 7):
        for b in range(nb):
            cols = [j for j in range(K) if oracle.cs_bucket(K, seed, j) == b]
            assert o["winner"][i * nb + b] == i * K + min(cols)


def test_zero_matrix_and_errors():
    o = oracle.build_sketch_cs(np.zeros((64, 256), np.float32), 0)
    assert o["status"] == oracle.OK and np.all(o["codes"] == 0) and np.all(o["scales"] == 0)
    assert oracle.build_sketch_cs(np.zeros((64, 100), np.float32), 0)["status"] == oracle.ERR_SHAPE
    W = np.zeros((64, 256), np.float32)
    W[1, 2] = np.inf
    assert oracle.build_sketch_cs(W, 0)["status"] == oracle.ERR_NONFINITE
    assert oracle.build_sketch_cs(np.full((64, 256), 1e9, np.float32), 0)["status"] == oracle.ERR_SCALE_OVERFLOW
