"""Pins of the format-2 oracle (the multi-row AbsMaxMin sketch) against things
other than itself (CPU only).

"UltraSketchLLM" explainer, Resumen Tecnico, Metodologia §1: a bucket stores
its member of smallest absolute value, decompression takes the maximum over
several independently hashed sketch rows, and every rebuilt weight is the
original one or one of smaller magnitude.  Each test names what fixes its
expected value: the independent brute force of tests/brute_force.py (member
lists, exact rational quantisation), the format-1 hash it reduces to at depth 1,
the magnitude bound, or a closed form.
"""
from fractions import Fraction

import numpy as np
import pytest

import gen
import oracle
from tests import brute_force

DEPTHS = (1, 2, 4)
CASES = [(64, 256), (128, 256), (64, 768), (128, 512)]


@pytest.mark.parametrize("M,K", CASES)
@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
@pytest.mark.parametrize("depth", DEPTHS)
def test_build_matches_brute_force(M, K, wdtype, depth):
    seed = 7 + M + K
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, wdtype)
    o = oracle.build_sketch_amm(W, seed, depth, want_winners=True)
    assert o["status"] == oracle.OK
    codes, scales, winner = brute_force.build_amm(W, seed, depth)
    assert np.array_equal(o["winner"], winner)
    assert np.array_equal(o["scales"], scales)
    assert np.array_equal(o["codes"], codes)


@pytest.mark.parametrize("depth", DEPTHS)
def test_ties_heavy_matches_brute_force(depth):
    # five magnitudes, random signs: many equal |w| in every bucket
    g = np.random.default_rng(21)
    vals = np.float32([-0.03, -0.01, 0.0, 0.01, 0.03, 0.05])
    W = gen.f32_to_bf16_bits(vals[g.integers(0, 6, size=(128, 512))])
    o = oracle.build_sketch_amm(W, 4, depth, want_winners=True)
    codes, scales, winner = brute_force.build_amm(W, 4, depth)
    assert np.array_equal(o["winner"], winner)
    assert np.array_equal(o["codes"], codes) and np.array_equal(o["scales"], scales)


@pytest.mark.parametrize("depth", DEPTHS)
def test_decode_matches_brute_force(depth):
    M, K, seed = 64, 512, 11
    W = gen.weights_normal(M, K, seed, 0.02, "f32")
    o = oracle.build_sketch_amm(W, seed, depth)
    ours = oracle.decode_amm(o["codes"], o["scales"], M, K, seed, depth)
    ref = brute_force.decode_amm(o["codes"], o["scales"], M, K, seed, depth)
    assert np.array_equal(ours.astype(np.float64), ref)


def test_depth_one_hash_is_the_format_one_hash():
    M, K = 128, 512
    for seed in (0, 5):
        for i in range(0, M, 7):
            for j in range(0, K, 3):
                assert oracle.amm_bucket_index(K, seed, 1, 0, i, j) == oracle.bucket_index(K, seed, i, j)


@pytest.mark.parametrize("depth", (2, 4))
def test_rows_partition_the_tile(depth):
    # row rho only ever lands in its own 1024/depth buckets of the weight's tile
    M, K, seed = 128, 512, 3
    per = 1024 // depth
    for rho in range(depth):
        for i in range(0, M, 5):
            for j in range(0, K, 11):
                b = oracle.amm_bucket_index(K, seed, depth, rho, i, j)
                base = (i // 64) * 4 * K + 1024 * (j // 256)
                assert base + rho * per <= b < base + (rho + 1) * per


@pytest.mark.parametrize("depth", DEPTHS)
@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
def test_magnitude_bound_every_weight(depth, wdtype):
    # the paper's bound: the rebuilt weight never exceeds the original in magnitude
    M, K, seed = 256, 1024, 2
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, wdtype)
    Wf = gen.bf16_bits_to_f32(W) if wdtype == "bf16" else W
    o = oracle.build_sketch_amm(W, seed, depth)
    Wh = oracle.decode_amm(o["codes"], o["scales"], M, K, seed, depth)
    assert np.all(np.abs(Wh.astype(np.float64)) <= np.abs(Wf.astype(np.float64)))


@pytest.mark.parametrize("depth", DEPTHS)
def test_codes_are_toward_zero_quotients(depth):
    M, K, seed = 128, 512, 8
    W = gen.weights_normal(M, K, seed, 0.02, "f32")
    o = oracle.build_sketch_amm(W, seed, depth, want_winners=True)
    per = 4 * K
    for q in range(0, M * K // 16, 37):
        s = Fraction(float(np.uint16(o["scales"][q // per]).view(np.float16)))
        v = Fraction(float(o["value"][q]))
        n = abs(int(o["codes"][q]))
        assert n * s <= abs(v)
        assert n == 127 or abs(v) < (n + 1) * s
        assert n == 0 or (o["codes"][q] < 0) == (v < 0)


def test_truncation_not_rounding_closed_form():
    # all |w| = 1 except every member of one row-0 bucket = 2: that bucket keeps
    # 2, every other bucket keeps a 1.  s16 = f16(2/127) = 1032 * 2^-16, so
    # 1/s = 63.50..: a toward-zero code is 63 (rounding would give 64), and
    # 2/s = 127.0..: 127.
    M, K, seed, depth = 64, 256, 1, 2
    W = np.ones((M, K), np.float32)
    target = oracle.amm_bucket_index(K, seed, depth, 0, 0, 0)
    for i in range(M):
        for j in range(K):
            if oracle.amm_bucket_index(K, seed, depth, 0, i, j) == target:
                W[i, j] = 2.0
    o = oracle.build_sketch_amm(W, seed, depth, want_winners=True)
    assert int(o["scales"][0]) == int(np.float16(2.0 / 127.0).view(np.uint16))
    assert float(np.uint16(o["scales"][0]).view(np.float16)) == 1032 * 2.0**-16
    assert o["codes"][target] == 127
    others = np.array([b for b in range(1024) if b != target and o["winner"][b] >= 0])
    assert np.all(o["value"][others] == 1.0)
    assert np.all(o["codes"][others] == 63)


def test_all_equal_magnitudes_tie_to_lowest_index_and_row_zero():
    # |w| = 1 everywhere, random signs: each bucket keeps its lowest-index
    # member; every weight sees |code| = 127 in both rows, so decode takes row 0
    M, K, seed, depth = 64, 512, 6, 2
    g = np.random.default_rng(1)
    W = np.where(g.random((M, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    o = oracle.build_sketch_amm(W, seed, depth, want_winners=True)
    s = float(np.uint16(o["scales"][0]).view(np.float16))
    Wh = oracle.decode_amm(o["codes"], o["scales"], M, K, seed, depth)
    first = {}
    for i in range(M):
        for j in range(K):
            first.setdefault(oracle.amm_bucket_index(K, seed, depth, 0, i, j), i * K + j)
    for i in range(0, M, 3):
        for j in range(0, K, 5):
            b0 = oracle.amm_bucket_index(K, seed, depth, 0, i, j)
            sign = W.reshape(-1)[first[b0]]
            assert Wh[i, j] == np.float32(sign * 127 * s)


def test_winner_has_minimum_magnitude_among_members():
    M, K, seed, depth = 128, 512, 9, 4
    W = gen.weights_normal(M, K, seed, 0.02, "bf16")
    Wf = gen.bf16_bits_to_f32(W).reshape(-1)
    o = oracle.build_sketch_amm(W, seed, depth, want_winners=True)
    mem = {}
    for i in range(M):
        for j in range(K):
            for rho in range(depth):
                mem.setdefault(oracle.amm_bucket_index(K, seed, depth, rho, i, j), []).append(i * K + j)
    for b, ms in mem.items():
        w = o["winner"][b]
        assert w in ms
        assert abs(Wf[w]) == min(abs(Wf[q]) for q in ms)
        assert w == min(q for q in ms if abs(Wf[q]) == abs(Wf[w]))


def test_zero_matrix():
    o = oracle.build_sketch_amm(np.zeros((64, 256), np.float32), 0, 2)
    assert o["status"] == oracle.OK
    assert np.all(o["codes"] == 0) and np.all(o["scales"] == 0)


@pytest.mark.parametrize("xdtype", ["f32", "bf16"])
@pytest.mark.parametrize("depth", DEPTHS)
def test_gemv_matches_numpy_matmul_of_decode(xdtype, depth):
    M, K, seed = 128, 768, 4
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, "bf16")
    o = oracle.build_sketch_amm(W, seed, depth)
    x = gen.activations(3, K, seed, xdtype)
    xf = gen.bf16_bits_to_f32(x) if xdtype == "bf16" else x
    Wh = oracle.decode_amm(o["codes"], o["scales"], M, K, seed, depth).astype(np.float64)
    ref = xf.astype(np.float64) @ Wh.T
    y = oracle.gemv_amm_f64(o["codes"], o["scales"], M, K, x, seed, depth)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    rows = np.array([0, 5, 64, 127])
    ys = oracle.gemv_amm_f64(o["codes"], o["scales"], M, K, x, seed, depth, rows=rows)
    assert np.array_equal(ys, y[:, rows])


def test_error_statuses():
    W = np.zeros((64, 256), np.float32)
    assert oracle.build_sketch_amm(W, 0, 3)["status"] == oracle.ERR_SHAPE
    assert oracle.build_sketch_amm(np.zeros((64, 100), np.float32), 0, 2)["status"] == oracle.ERR_SHAPE
    W[3, 7] = np.nan
    assert oracle.build_sketch_amm(W, 0, 2)["status"] == oracle.ERR_NONFINITE
    W[3, 7] = 1e9  # max |v| / 127 above the binary16 range only if it is kept: all others are 0
    big = np.full((64, 256), 1e9, np.float32)
    assert oracle.build_sketch_amm(big, 0, 2)["status"] == oracle.ERR_SCALE_OVERFLOW


def test_rows_slice_equals_full_build():
    M, K, seed = 256, 512, 12
    W = gen.weights_normal(M, K, seed, 0.02, "bf16")
    full = oracle.build_sketch_amm(W, seed, 2)
    per = 4 * K
    part = oracle.build_sketch_amm(W[128:192], seed, 2, row_block0=2)
    assert np.array_equal(part["codes"], full["codes"][2 * per:3 * per])
    assert np.array_equal(part["scales"], full["scales"][2:3])
