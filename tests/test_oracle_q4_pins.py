"""Pins of the format-4 oracle (the format-1 sketch with 4-bit codes and 8
weights per bucket; "UltraSketchLLM" explainer, Resultados Experimentales:
0.5 bit/weight with 4-bit quantisation) against things other than itself.

Each test names what fixes its expected value: the independent brute force of
tests/brute_force.py (its own hash with 8 slots, member lists, numpy float16 and
rint, its own nibble packing), closed forms, invariants, numpy matmul.
"""
import numpy as np
import pytest

import gen
import oracle
from tests import brute_force


@pytest.mark.parametrize("M,K", [(64, 256), (128, 512), (64, 768)])
@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
@pytest.mark.parametrize("with_imp", [False, True])
def test_build_matches_brute_force(M, K, wdtype, with_imp):
    seed = 5 + M + K
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, wdtype)
    imp = gen.importance_lognormal(K, seed) if with_imp else None
    o = oracle.build_sketch_q4(W, imp, seed, want_winners=True)
    assert o["status"] == oracle.OK
    codes, scales, winner = brute_force.build_q4(W, imp, seed)
    assert np.array_equal(o["winner"], winner)
    assert np.array_equal(o["scales"], scales)
    assert np.array_equal(o["codes"], codes)


def test_ties_heavy_matches_brute_force():
    g = np.random.default_rng(41)
    vals = np.float32([-0.03, -0.01, 0.0, 0.01, 0.03])
    W = gen.f32_to_bf16_bits(vals[g.integers(0, 5, size=(128, 512))])
    o = oracle.build_sketch_q4(W, None, 3, want_winners=True)
    codes, scales, winner = brute_force.build_q4(W, None, 3)
    assert np.array_equal(o["winner"], winner)
    assert np.array_equal(o["codes"], codes) and np.array_equal(o["scales"], scales)


def test_bucket_structure_eight_members_per_bucket_on_average():
    # 2048 buckets per 64 x 256 tile; each (class, sub) owns one octet column per
    # row: 64 members over 8 slots
    K, seed = 512, 7
    counts = np.zeros(8 * K, np.int64)
    for i in range(64):
        for j in range(K):
            counts[oracle.q4_bucket(K, seed, i, j)] += 1
    assert counts.sum() == 64 * K and counts.mean() == 8.0
    for tc in range(K // 256):
        t = counts[2048 * tc:2048 * (tc + 1)].reshape(8, 32, 8)  # slot, class, sub
        assert np.all(t.sum(axis=0) == 64)


def test_storage_identity_half_bit_per_weight():
    W = gen.weights_normal(128, 1024, 1, 0.02, "bf16")
    o = oracle.build_sketch_q4(W, None, 1)
    assert o["codes"].nbytes * 8 == 128 * 1024 // 2
    assert o["scales"].nbytes * 8 == 16 * (128 // 64)


def test_all_equal_magnitudes_full_codes():
    # every kept |v| = 0.5: s16 = f16(0.5/7); 0.5/s rounds to 7 -> codes +-7
    M, K = 64, 256
    g = np.random.default_rng(3)
    W = np.where(g.random((M, K)) < 0.5, -0.5, 0.5).astype(np.float32)
    o = oracle.build_sketch_q4(W, None, 2, want_winners=True)
    Wh = oracle.decode_q4(o["codes"], o["scales"], M, K, 2)
    s = float(np.uint16(o["scales"][0]).view(np.float16))
    assert np.all(np.abs(Wh) == np.float32(7 * s))


def test_outlier_takes_the_scale():
    M, K = 64, 256
    W = np.full((M, K), 0.01, np.float32)
    W[10, 20] = 10.0
    o = oracle.build_sketch_q4(W, None, 0)
    assert int(o["scales"][0]) == int(np.float16(np.float32(10.0) / np.float32(7.0)).view(np.uint16))
    Wh = oracle.decode_q4(o["codes"], o["scales"], M, K, 0)
    assert Wh[10, 20] == np.float32(7 * float(np.uint16(o["scales"][0]).view(np.float16)))


def test_half_way_quotients_round_to_even():
    # one weight 7 s fixes s16 = f16(7 s / 7) = s = 2^-4 exactly; every other
    # bucket keeps v s (all its members equal), so it decodes to rint(v) s with
    # ties to even: 2.5 -> 2, 3.5 -> 4, -2.5 -> -2, 0.5 -> 0, 1.5 -> 2
    M, K = 64, 256
    s = 2.0 ** -4
    b0 = oracle.q4_bucket(K, 0, 0, 0)
    probe = next((i, j) for i in range(M) for j in range(K) if oracle.q4_bucket(K, 0, i, j) != b0)
    for v, want in ((2.5, 2), (3.5, 4), (-2.5, -2), (0.5, 0), (1.5, 2)):
        W = np.full((M, K), np.float32(v * s), np.float32)
        W[0, 0] = np.float32(7 * s)
        o = oracle.build_sketch_q4(W, None, 0)
        assert float(np.uint16(o["scales"][0]).view(np.float16)) == s
        Wh = oracle.decode_q4(o["codes"], o["scales"], M, K, 0)
        assert Wh[probe] == np.float32(want * s)


def test_decode_reads_the_right_nibble():
    M, K, seed = 64, 512, 9
    W = gen.weights_normal(M, K, seed, 0.02, "f32")
    o = oracle.build_sketch_q4(W, None, seed)
    Wh = oracle.decode_q4(o["codes"], o["scales"], M, K, seed)
    s = float(np.uint16(o["scales"][0]).view(np.float16))
    raw = o["codes"].view(np.uint8)
    for i in range(0, M, 5):
        for j in range(0, K, 7):
            b = oracle.q4_bucket(K, seed, i, j)
            nib = (int(raw[b // 2]) >> (4 * (b % 2))) & 15
            code = nib - 16 if nib >= 8 else nib
            assert Wh[i, j] == np.float32(code * s)


@pytest.mark.parametrize("xdtype", ["f32", "bf16"])
def test_gemv_matches_numpy_matmul(xdtype):
    M, K, seed = 128, 768, 4
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, "bf16")
    o = oracle.build_sketch_q4(W, None, seed)
    x = gen.activations(3, K, seed, xdtype)
    xf = gen.bf16_bits_to_f32(x) if xdtype == "bf16" else x
    ref = xf.astype(np.float64) @ oracle.decode_q4(o["codes"], o["scales"], M, K, seed).astype(np.float64).T
    y = oracle.gemv_q4_f64(o["codes"], o["scales"], M, K, x, seed)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_errors_and_rows_slice():
    assert oracle.build_sketch_q4(np.zeros((64, 100), np.float32))["status"] == oracle.ERR_SHAPE
    W = np.zeros((64, 256), np.float32)
    W[0, 1] = np.nan
    assert oracle.build_sketch_q4(W)["status"] == oracle.ERR_NONFINITE
    assert oracle.build_sketch_q4(np.zeros((64, 256), np.float32),
                                  -np.ones(256, np.float32))["status"] == oracle.ERR_IMPORTANCE
    W = gen.weights_normal(192, 512, 5, 0.02, "bf16")
    full = oracle.build_sketch_q4(W, None, 6)
    part = oracle.build_sketch_q4(W[128:192], None, 6, row_block0=2)
    assert np.array_equal(part["codes"], full["codes"][2 * 4 * 512:3 * 4 * 512])
    assert np.array_equal(part["scales"], full["scales"][2:3])
