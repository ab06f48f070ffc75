"""Pins of the CPU oracle against things other than itself (CPU only).

Each test names what fixes the expected value: a published generator output,
numpy's IEEE conversions, an independent brute-force enumeration, a closed
form or an invariant of the format.
"""
import os

import numpy as np
import pytest

import gen
import oracle
from tests import brute_force

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------- SplitMix64

def test_splitmix64_published_outputs():
    with open(os.path.join(GOLDEN, "splitmix64.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert rows
    for seed, n, hexv in rows:
        assert oracle.splitmix64(int(seed), int(n)) == int(hexv, 16)


def test_tile_hash_params_odd_and_from_splitmix():
    for seed in (0, 1, 2**63 + 5):
        for t in (0, 1, 17, 1000):
            A, C = oracle.tile_hash_params(seed, t)
            z = brute_force.splitmix64_output(seed, t + 1)
            assert A & 1 == 1
            assert A == (z & 0xFFFFFFFF) | 1 and C == z >> 32


# ------------------------------------------------------------- binary16

def test_f16_round_trip_all_halves():
    h = np.arange(65536, dtype=np.uint16)
    f = oracle.f16_to_f32_array(h)
    ref = h.view(np.float16).astype(np.float32)
    finite = np.isfinite(ref)
    assert np.array_equal(f[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.all(np.isnan(f[np.isnan(ref)]))
    back = oracle.f32_to_f16_array(f[finite])
    assert np.array_equal(back, h[finite])


def test_f16_ties_and_neighbours_match_numpy():
    # every exact midpoint between consecutive finite halves, and 1 ulp (fp32) either side
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)  # exact in fp32
    cand = np.concatenate([mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(np.inf))])
    cand = np.concatenate([cand, -cand, np.float32([65504, 65519.99, 65520, 65536, 1e-8, 2.0**-25, 2.0**-24 * 1.5])])
    ours = oracle.f32_to_f16_array(cand)
    with np.errstate(over="ignore"):
        ref = cand.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f16_random_bit_patterns_match_numpy():
    g = np.random.default_rng(123)
    u = g.integers(0, 2**32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.f32_to_f16_array(f), ref)


# ------------------------------------------------------------- hash / bucket

def test_bucket_index_matches_independent_python():
    g = np.random.default_rng(5)
    for K in (256, 512, 1280):
        M = 128
        for seed in (0, 7, 2**40 + 3):
            for _ in range(300):
                i = int(g.integers(0, M))
                j = int(g.integers(0, K))
                assert oracle.bucket_index(K, seed, i, j) == brute_force.bucket_of(K, seed, i, j)


def test_bucket_structure_one_octet_per_row_per_class():
    """Every (class, sub) of a tile owns exactly one octet column per row: 64
    members spread over 4 slots (16 per bucket on average)."""
    K, seed = 512, 11
    counts = np.zeros(64 * K // 16, dtype=np.int64)
    for i in range(64):
        for j in range(K):
            b = oracle.bucket_index(K, seed, i, j)
            assert b // 1024 == j // 256  # bucket stays in its tile
            assert b % 8 == j % 8  # sub = column mod 8
            counts[b] += 1
    assert counts.sum() == 64 * K
    per_class_sub = counts.reshape(K // 256, 4, 32, 8).sum(axis=1)
    assert np.all(per_class_sub == 64)
    assert counts.mean() == 16


def test_hash_load_distribution():
    """Bucket loads over many tiles: mean 16, near-binomial(64, 1/4) spread, no
    pathological buckets (hash quality, not parity)."""
    loads = []
    for seed in range(6):
        K = 1024
        cnt = np.zeros(64 * K // 16, dtype=np.int64)
        for i in range(64):
            for j in range(0, K, 8):  # one column per octet; the 8 subs share the slot
                cnt[oracle.bucket_index(K, seed, i, j)] += 1
        loads.append(cnt.reshape(K // 256, 4, 32, 8)[..., 0].reshape(-1))
    loads = np.concatenate(loads)
    assert abs(loads.mean() - 16) < 1e-9
    var = loads.var()
    assert 2.0 < var < 20.0  # binomial(64, 1/4) has variance 12
    assert loads.max() <= 40 and loads.min() >= 0


# ------------------------------------------------------------- build vs brute force

CASES = [(64, 256), (64, 512), (128, 256), (64, 768), (128, 1024)]


@pytest.mark.parametrize("M,K", CASES)
@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
@pytest.mark.parametrize("with_imp", [False, True])
def test_build_matches_brute_force(M, K, wdtype, with_imp):
    for seed in (0, 3):
        W = gen.weights_student_t(M, K, seed + 10, 4.0, 0.02, 0.01, 20.0, wdtype)
        imp = gen.importance_lognormal(K, seed + 10) if with_imp else None
        o = oracle.build_sketch(W, imp, seed, want_winners=True)
        assert o["status"] == oracle.OK
        codes, scales, winner = brute_force.build(W, imp, seed)
        assert np.array_equal(o["winner"], winner)
        assert np.array_equal(o["scales"], scales)
        assert np.array_equal(o["codes"], codes)


def test_build_ties_heavy_bf16_matches_brute_force():
    # bf16 weights drawn from 5 values: many equal keys in every bucket
    g = np.random.default_rng(9)
    vals = np.float32([-0.03, -0.01, 0.0, 0.01, 0.03])
    W = gen.f32_to_bf16_bits(vals[g.integers(0, 5, size=(128, 512))])
    o = oracle.build_sketch(W, None, 4, want_winners=True)
    codes, scales, winner = brute_force.build(W, None, 4)
    assert np.array_equal(o["winner"], winner)
    assert np.array_equal(o["codes"], codes) and np.array_equal(o["scales"], scales)


# ------------------------------------------------------------- invariants

def _members(M, K, seed):
    mem = {}
    for i in range(M):
        for j in range(K):
            mem.setdefault(oracle.bucket_index(K, seed, i, j), []).append(i * K + j)
    return mem


def test_invariants_small_workload():
    cfg = gen.small()
    W, imp, seed = cfg["W"], cfg["importance"], cfg["seed"]
    M, K = W.shape
    o = oracle.build_sketch(W, imp, seed, want_winners=True)
    assert o["status"] == oracle.OK
    flat = W.reshape(-1)
    mem = _members(M, K, seed)
    scales = o["scales"].view(np.float16).astype(np.float32)
    for b in range(M * K // 16):
        ms = mem.get(b, [])
        w = o["winner"][b]
        if not ms:
            assert w == -1 and o["codes"][b] == 0
            continue
        assert w in ms  # the kept value is one of the bucket's members
        assert o["value"][b] == flat[w]
        kw = np.float32(abs(flat[w])) * imp[w % K]
        for q in ms:
            kq = np.float32(abs(flat[q])) * imp[q % K]
            assert kw > kq or (kw == kq and w <= q)  # key(winner) >= key(loser), ties to smaller index
        s = scales[b // (4 * K)]
        q = np.clip(np.rint(np.float32(flat[w]) / s), -127, 127)
        assert o["codes"][b] == q  # code is the quantized member value


def test_unit_importance_literal_magnitude_invariant():
    W = gen.weights_normal(64, 512, 21, 0.02, "bf16")
    o = oracle.build_sketch(W, None, 21, want_winners=True)
    Wf = gen.bf16_bits_to_f32(W).reshape(-1)
    mem = _members(64, 512, 21)
    for b, ms in mem.items():
        v = abs(Wf[o["winner"][b]])
        assert all(v >= abs(Wf[q]) for q in ms)


def test_null_importance_equals_all_ones():
    W = gen.weights_normal(128, 768, 2, 0.02, "bf16")
    a = oracle.build_sketch(W, None, 2, want_winners=True)
    b = oracle.build_sketch(W, np.ones(768, np.float32), 2, want_winners=True)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    assert np.array_equal(a["winner"], b["winner"])


# ------------------------------------------------------------- closed forms

def test_all_equal_magnitude_mixed_signs_lowest_index_wins():
    g = np.random.default_rng(1)
    W = (np.where(g.random((64, 256)) < 0.5, -1.0, 1.0) * 0.5).astype(np.float32)
    o = oracle.build_sketch(W, None, 3, want_winners=True)
    mem = _members(64, 256, 3)
    for b, ms in mem.items():
        assert o["winner"][b] == min(ms)
        # s16 = f16(0.5/127); code = rint(+-0.5 / s16) = +-127 exactly at this scale
        assert abs(int(o["codes"][b])) == 127
        assert np.sign(o["codes"][b]) == np.sign(W.reshape(-1)[min(ms)])


def test_zero_matrix_scale_zero_codes_zero():
    W = np.zeros((128, 512), np.float32)
    o = oracle.build_sketch(W, None, 0)
    assert o["status"] == oracle.OK
    assert not o["codes"].any() and not o["scales"].any()
    y = oracle.gemv_f64(o["codes"], o["scales"], 128, 512, np.ones((2, 512), np.float32), 0)
    assert np.all(y == 0.0)


def test_single_outlier_gets_full_code():
    W = gen.weights_normal(64, 512, 4, 0.02, "f32")
    W[17, 300] = 40.0
    o = oracle.build_sketch(W, None, 5)
    b = oracle.bucket_index(512, 5, 17, 300)
    assert o["codes"][b] == 127
    s = np.float16(np.float32(40.0) / np.float32(127.0))
    assert o["scales"][0] == s.view(np.uint16)
    # every other code is tiny compared with the outlier's
    others = np.delete(o["codes"], b)
    assert np.abs(others).max() <= 2


def test_quantization_half_even_closed_form():
    # v / s lands exactly on k + 0.5 for a power-of-two scale: ties go to even
    # max |v| = 127 * 2^-6 gives s16 = 2^-6 exactly
    W = np.zeros((64, 256), np.float32)
    s = 2.0 ** -6
    W[0, 0] = 127 * s
    W[1, 8] = 2.5 * s  # -> 2
    W[2, 16] = 3.5 * s  # -> 4
    W[3, 24] = -2.5 * s  # -> -2
    o = oracle.build_sketch(W, None, 6)
    assert o["scales"][0] == np.float16(s).view(np.uint16)
    want = {(0, 0): 127, (1, 8): 2, (2, 16): 4, (3, 24): -2}
    for (i, j), c in want.items():
        b = oracle.bucket_index(256, 6, i, j)
        # the weight must be its bucket's winner for the check to mean anything
        assert o["codes"][b] == c


def test_storage_identity_half_bit_per_weight():
    for M, K in [(64, 256), (4096, 4096), (28672, 8192), (4096, 11008)]:
        cb, sb = oracle.storage_bytes(M, K)
        assert cb * 8 * 2 == M * K  # 0.5 bit per weight for the codes
        assert sb == 2 * (M // 64)
        # total bits per weight = 0.5 + 16 / (64 K) = 0.5 + 0.25 / K
        assert (cb * 8 + sb * 8) / (M * K) == pytest.approx(0.5 + 0.25 / K, rel=1e-12)


# ------------------------------------------------------------- errors

def test_error_statuses():
    W = np.zeros((64, 256), np.float32)
    assert oracle.build_sketch(np.zeros((63, 256), np.float32))["status"] == oracle.ERR_SHAPE
    assert oracle.build_sketch(np.zeros((64, 200), np.float32))["status"] == oracle.ERR_SHAPE
    bad = W.copy()
    bad[3, 3] = np.nan
    assert oracle.build_sketch(bad)["status"] == oracle.ERR_NONFINITE
    bad[3, 3] = np.inf
    assert oracle.build_sketch(bad)["status"] == oracle.ERR_NONFINITE
    imp = np.ones(256, np.float32)
    imp[5] = -1.0
    assert oracle.build_sketch(W, imp)["status"] == oracle.ERR_IMPORTANCE
    imp[5] = -0.0
    assert oracle.build_sketch(W, imp)["status"] == oracle.ERR_IMPORTANCE
    imp[5] = np.inf
    assert oracle.build_sketch(W, imp)["status"] == oracle.ERR_IMPORTANCE
    big = W.copy()
    big[0, 0] = 1e7  # 1e7 / 127 > 65504: the binary16 scale overflows
    assert oracle.build_sketch(big)["status"] == oracle.ERR_SCALE_OVERFLOW


def test_empty_shapes():
    o = oracle.build_sketch(np.zeros((0, 256), np.float32))
    assert o["status"] == oracle.OK and o["codes"].size == 0
    o = oracle.build_sketch(np.zeros((128, 0), np.float32))
    assert o["status"] == oracle.OK and o["codes"].size == 0 and np.all(o["scales"] == 0)


# ------------------------------------------------------------- decode / products

def test_decode_reads_back_bucket_code_times_scale():
    W = gen.weights_normal(128, 512, 8, 0.02, "bf16")
    o = oracle.build_sketch(W, None, 8)
    What = oracle.decode(o["codes"], o["scales"], 128, 512, 8)
    s = o["scales"].view(np.float16).astype(np.float32)
    g = np.random.default_rng(0)
    for _ in range(500):
        i, j = int(g.integers(0, 128)), int(g.integers(0, 512))
        b = brute_force.bucket_of(512, 8, i, j)
        assert What[i, j] == np.float32(o["codes"][b]) * s[i // 64]


@pytest.mark.parametrize("xdtype", ["f32", "bf16"])
def test_gemv_f64_matches_numpy_matmul(xdtype):
    M, K = 192, 768
    W = gen.weights_normal(M, K, 12, 0.02, "f32")
    imp = gen.importance_lognormal(K, 12)
    o = oracle.build_sketch(W, imp, 12)
    What = oracle.decode(o["codes"], o["scales"], M, K, 12).astype(np.float64)
    x = gen.activations(5, K, 12, xdtype)
    xf = x.astype(np.float64) if xdtype == "f32" else gen.bf16_bits_to_f32(x).astype(np.float64)
    y = oracle.gemv_f64(o["codes"], o["scales"], M, K, x, 12)
    ref = xf @ What.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([0, 63, 64, 191])
    ys = oracle.gemv_f64(o["codes"], o["scales"], M, K, x, 12, rows=rows)
    assert np.allclose(ys, ref[:, rows], rtol=1e-12, atol=1e-12)


def test_build_rows_slice_equals_full_build():
    W = gen.weights_normal(256, 512, 31, 0.02, "bf16")
    full = oracle.build_sketch(W, None, 31)
    per = 64 * 512 // 16
    for rb0 in (1, 2):
        part = oracle.build_sketch(W[64 * rb0:64 * rb0 + 128], None, 31, row_block0=rb0)
        assert np.array_equal(part["codes"], full["codes"][rb0 * per:(rb0 + 2) * per])
        assert np.array_equal(part["scales"], full["scales"][rb0:rb0 + 2])
