"""Pins of the per-row-block rate oracle: each 64-row block of a format-1
sketch carries its own slot count (2, 4 or 8 hash slots per class), the blocks'
codes back to back in matrix order ("UltraSketchLLM" explainer, Resumen
Tecnico, Metodologia §2: rows of higher importance E[a^2] receive larger
sketch spaces).  Expected values come from the independent brute force, the
per-sketch rate oracle (a uniform table reduces to it), closed forms of the
offsets and storage, and the float64 product of the brute-force decode."""
import numpy as np
import pytest

import gen
import oracle
from tests import brute_force


def test_offsets_closed_form():
    off, total = oracle.vr_offsets(256, 512, [2, 8, 4, 2])
    assert off.tolist() == [0, 2 * 512, 10 * 512, 14 * 512] and total == 16 * 512
    off, total = oracle.vr_offsets(64, 256, [8])
    assert off.tolist() == [0] and total == 2048
    with pytest.raises(ValueError):
        oracle.vr_offsets(128, 256, [2, 3])


@pytest.mark.parametrize("S", [2, 4, 8])
def test_uniform_table_is_the_rate_sketch(S):
    W = gen.weights_student_t(192, 1024, 4, 4.0, 0.02, 0.01, 20.0, "bf16")
    imp = gen.importance_lognormal(1024, 4)
    a = oracle.build_sketch_vr(W, imp, 7, [S] * 3)
    b = oracle.build_sketch_rate(W, imp, 7, S)
    assert a["status"] == oracle.OK
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


def test_each_block_is_its_rate_sketchs_block():
    """Block rb's segment equals row block rb of the uniform slots[rb] sketch
    (same hash tiles, same selection): the layout only moves segments."""
    slots = [8, 2, 4, 2, 8]
    M, K = 64 * len(slots), 768
    W = gen.weights_student_t(M, K, 6, 4.0, 0.02, 0.01, 20.0, "f32")
    o = oracle.build_sketch_vr(W, None, 11, slots)
    off, total = oracle.vr_offsets(M, K, slots)
    assert o["codes"].size == total
    for rb, S in enumerate(slots):
        u = oracle.build_sketch_rate(W, None, 11, S)
        seg = u["codes"][rb * S * K:(rb + 1) * S * K]
        assert np.array_equal(o["codes"][off[rb]:off[rb] + S * K], seg)
        assert o["scales"][rb] == u["scales"][rb]


@pytest.mark.parametrize("with_imp", [False, True])
def test_brute_force_mixed_table(with_imp):
    slots = [2, 8, 4]
    W = gen.weights_student_t(192, 512, 8, 4.0, 0.02, 0.01, 20.0, "bf16")
    imp = gen.importance_lognormal(512, 8) if with_imp else None
    o = oracle.build_sketch_vr(W, imp, 13, slots)
    codes, scales = brute_force.build_vr(W, imp, 13, slots)
    assert o["status"] == oracle.OK
    assert np.array_equal(o["codes"], codes) and np.array_equal(o["scales"], scales)


def test_bucket_index_matches_brute_force():
    slots = [4, 2, 8, 8]
    K = 512
    g = np.random.default_rng(3)
    for _ in range(300):
        i, j = int(g.integers(0, 256)), int(g.integers(0, K))
        assert oracle.vr_bucket(K, 21, slots, i, j) == brute_force.bucket_of_vr(K, 21, slots, i, j)


def test_storage_and_bits_per_weight():
    """K * sum(slots) code bytes: 2, 4, 8 slots give 0.25, 0.5, 1 bit/weight;
    a table averaging 4 slots averages 0.5 bit/weight."""
    slots = [2, 8, 2, 4, 4]
    M, K = 320, 256
    o = oracle.build_sketch_vr(np.zeros((M, K), np.float32), None, 0, slots)
    assert o["codes"].size == K * sum(slots)
    assert o["codes"].size * 8 / (M * K) == np.mean(slots) / 8 == 0.5
    assert not o["codes"].any() and not o["scales"].any()


def test_product_is_the_brute_force_decode():
    slots = [2, 8, 4]
    M, K = 192, 512
    W = gen.weights_student_t(M, K, 9, 4.0, 0.02, 0.01, 20.0, "bf16")
    codes, scales = brute_force.build_vr(W, None, 17, slots)
    What = np.zeros((M, K), np.float64)
    for i in range(M):
        s = np.float32(np.frombuffer(np.uint16(scales[i // 64]).tobytes(), np.float16)[0])
        for j in range(K):
            What[i, j] = np.float64(np.float32(codes[brute_force.bucket_of_vr(K, 17, slots, i, j)]) * s)
    x = gen.activations(3, K, 10, "f32")
    y = oracle.gemv_vr_f64(codes, scales, M, K, x, 17, slots)
    ref = x.astype(np.float64) @ What.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)
    rows = np.array([0, 63, 64, 130, 191])
    assert np.array_equal(oracle.gemv_vr_f64(codes, scales, M, K, x, 17, slots, rows=rows), y[:, rows])


def test_one_hot_reads_back_the_bucket():
    slots = [8, 2]
    M, K = 128, 256
    W = gen.weights_normal(M, K, 2, 0.02, "f32")
    o = oracle.build_sketch_vr(W, None, 5, slots)
    for j in (0, 7, 100, 255):
        x = np.zeros((1, K), np.float32)
        x[0, j] = 1.0
        y = oracle.gemv_vr_f64(o["codes"], o["scales"], M, K, x, 5, slots)[0]
        for i in (0, 63, 64, 127):
            s = float(np.frombuffer(np.uint16(o["scales"][i // 64]).tobytes(), np.float16)[0])
            assert y[i] == float(o["codes"][brute_force.bucket_of_vr(K, 5, slots, i, j)]) * s


def test_errors():
    W = np.zeros((128, 256), np.float32)
    assert oracle.build_sketch_vr(W, None, 0, [2, 3])["status"] == oracle.ERR_SHAPE
    with pytest.raises(ValueError):
        oracle.build_sketch_vr(W, None, 0, [2])
    Wn = gen.weights_normal(128, 256, 1, 0.02, "f32")
    Wn[70, 3] = np.inf
    assert oracle.build_sketch_vr(Wn, None, 0, [2, 8])["status"] == oracle.ERR_NONFINITE
