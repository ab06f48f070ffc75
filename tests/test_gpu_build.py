"""usk_build on the GPU against the CPU oracle: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, scales_np, status_tensor, to_dev

pytestmark = pytest.mark.gpu


def _gpu_build(W, imp, seed, status=None):
    return usk.usk_build(to_dev(W), None if imp is None else to_dev(imp), seed, status=status)


def _compare(W, imp, seed):
    o = oracle.build_sketch(W, imp, seed)
    assert o["status"] == oracle.OK
    sk = _gpu_build(W, imp, seed)
    torch.cuda.synchronize()
    c, s = codes_np(sk), scales_np(sk)
    assert np.array_equal(s, o["scales"]), "scales differ"
    bad = np.nonzero(c != o["codes"])[0]
    assert bad.size == 0, "codes differ at %d buckets, first %s" % (bad.size, bad[:8])


# several tiles, clusters of 1..8 blocks, uneven tiles per block (11 and 17 tiles)
SHAPES = [(64, 256), (128, 1024), (192, 2816), (64, 4352), (256, 512)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("wdtype", ["bf16", "f32"])
@pytest.mark.parametrize("with_imp", [False, True])
def test_build_bit_exact(M, K, wdtype, with_imp):
    for seed in (0, 12345):
        W = gen.weights_student_t(M, K, seed + 1, 4.0, 0.02, 0.001, 20.0, wdtype)
        imp = gen.importance_lognormal(K, seed + 1) if with_imp else None
        _compare(W, imp, seed)


def test_build_small_workload():
    cfg = gen.small()
    _compare(cfg["W"], cfg["importance"], cfg["seed"])


def test_build_layer_workload_full():
    cfg = gen.layer()
    _compare(cfg["W"], cfg["importance"], cfg["seed"])


def test_build_ties_heavy():
    g = np.random.default_rng(9)
    vals = np.float32([-0.03, -0.01, -0.0, 0.0, 0.01, 0.03])
    W = gen.f32_to_bf16_bits(vals[g.integers(0, 6, size=(256, 1024))])
    _compare(W, None, 4)
    _compare(W, np.ones(1024, np.float32), 4)
    Wf = vals[g.integers(0, 6, size=(128, 768))].astype(np.float32)
    _compare(Wf, None, 5)


def test_build_special_cases():
    _compare(np.zeros((128, 512), np.float32), None, 1)  # all zero -> scale 0, codes 0
    W = gen.weights_normal(64, 512, 4, 0.02, "f32")
    W[17, 300] = 40.0  # single outlier -> its code is 127
    _compare(W, None, 5)
    g = np.random.default_rng(1)
    W = (np.where(g.random((64, 256)) < 0.5, -1.0, 1.0) * 0.5).astype(np.float32)
    _compare(W, None, 3)  # all-equal magnitudes: lowest index wins
    Wb = gen.weights_normal(128, 768, 2, 0.02, "bf16")
    a = _gpu_build(Wb, None, 2)
    b = _gpu_build(Wb, np.ones(768, np.float32), 2)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)


@pytest.mark.parametrize("scale_exp", [-6, -14, 3])
def test_build_half_way_quotients_round_to_even(scale_exp):
    """Winners at exact half-integer multiples of the scale: the quantizer must
    round those ties to even, as rint of the IEEE quotient does.  Scales 2^-6,
    2^-14 (the smallest normal binary16) and 2^3."""
    g = np.random.default_rng(77 + scale_exp)
    s = 2.0 ** scale_exp
    M, K = 128, 1024
    n = g.integers(0, 127, size=(M, K))
    w = ((2 * n + 1) / 2.0) * s * np.where(g.random((M, K)) < 0.5, -1.0, 1.0)
    w[::64, 0] = 127.0 * s  # each row block's maximum: s16 = s exactly
    W = gen.f32_to_bf16_bits(w.astype(np.float32))
    assert np.array_equal(gen.bf16_bits_to_f32(W), w.astype(np.float32))  # every value exact in bf16
    o = oracle.build_sketch(W, None, 5, want_winners=True)
    assert np.all(o["scales"] == np.float16(s).view(np.uint16))
    ties = np.abs(o["value"]) / np.float32(s)
    assert np.count_nonzero(ties != np.round(ties)) > 1000  # plenty of half-way quotients
    _compare(W, None, 5)


def test_build_row_stride():
    W = gen.weights_normal(128, 768, 7, 0.02, "bf16")
    big = np.zeros((128, 1024), np.uint16)
    big[:, :768] = W
    d = to_dev(big)[:, :768]
    assert d.stride(0) == 1024
    sk = usk.usk_build(d, None, 7)
    o = oracle.build_sketch(W, None, 7)
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])


@pytest.mark.parametrize("cluster", [1, 2, 3, 5, 8])
def test_build_geometry_independent(cluster):
    W = gen.weights_student_t(128, 4352, 3, 4.0, 0.02, 0.001, 20.0, "bf16")
    imp = gen.importance_lognormal(4352, 3)
    ref = _gpu_build(W, imp, 9)
    try:
        usk.usk_debug_set_geometry(cluster, 0)
        got = _gpu_build(W, imp, 9)
    finally:
        usk.usk_debug_set_geometry(0, 0)
    assert torch.equal(ref.codes, got.codes) and torch.equal(ref.scales, got.scales)


def test_build_repeatable():
    cfg = gen.layer(M=1024, K=4096)
    a = _gpu_build(cfg["W"], cfg["importance"], 1)
    for _ in range(3):
        b = _gpu_build(cfg["W"], cfg["importance"], 1)
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)


def test_build_device_flags():
    W = gen.weights_normal(64, 512, 4, 0.02, "f32")
    st = status_tensor()
    _gpu_build(W, None, 0, st)
    assert int(st.item()) == 0
    bad = W.copy()
    bad[5, 7] = np.nan
    st = status_tensor()
    _gpu_build(bad, None, 0, st)
    assert int(st.item()) & usk.FLAG_NONFINITE_W
    bad[5, 7] = np.inf
    st = status_tensor()
    _gpu_build(bad, None, 0, st)
    assert int(st.item()) & usk.FLAG_NONFINITE_W
    # huge importance overflows the key to +Inf without any non-finite weight
    imp = np.full(512, 3e38, np.float32)
    st = status_tensor()
    _gpu_build(W, imp, 0, st)
    assert not (int(st.item()) & usk.FLAG_NONFINITE_W)
    imp = np.ones(512, np.float32)
    imp[3] = -0.0
    st = status_tensor()
    _gpu_build(W, imp, 0, st)
    assert int(st.item()) & usk.FLAG_BAD_IMPORTANCE
    big = W.copy()
    big[0, 0] = 1e7
    st = status_tensor()
    _gpu_build(big, None, 0, st)
    assert int(st.item()) & usk.FLAG_SCALE_OVERFLOW


def test_build_argument_errors():
    W = to_dev(gen.weights_normal(64, 512, 4, 0.02, "bf16"))
    with pytest.raises(usk.UskError) as e:
        usk.usk_build(W[:, :500].contiguous(), None, 0)
    assert e.value.status == 2
    with pytest.raises(usk.UskError) as e:
        usk.usk_build(to_dev(gen.weights_normal(63, 512, 4, 0.02, "bf16")), None, 0)
    assert e.value.status == 2
    # misaligned row start (odd element offset)
    flat = torch.zeros(64 * 512 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(usk.UskError) as e:
        usk.usk_build(flat[1:1 + 64 * 512].view(64, 512), None, 0)
    assert e.value.status == 10


def test_build_empty():
    sk = usk.usk_build(torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda"), None, 0)
    assert sk.codes.numel() == 0
    sc = torch.full((2,), 7, dtype=torch.int16, device="cuda")
    usk.usk_build(torch.zeros((128, 0), dtype=torch.bfloat16, device="cuda"), None, 0, scales=sc)
    torch.cuda.synchronize()
    assert int(sc.abs().sum().item()) == 0


def test_build_max_k():
    # the library's largest K (2^16) on one row block
    W = gen.weights_normal(64, 65536, 8, 0.02, "bf16")
    _compare(W, None, 8)


def test_build_mlp70b_sampled_row_blocks():
    """Full 28672x8192 build in the bench's launch configuration; the oracle
    checks a sample of row blocks (the sketch of a row block depends only on its
    rows)."""
    cfg = gen.mlp70b("up")
    W = cfg["W"]
    sk = _gpu_build(W, None, cfg["seed"])
    c, s = codes_np(sk), scales_np(sk)
    K = W.shape[1]
    per = 4 * K
    for rb in (0, 1, 223, 447):
        o = oracle.build_sketch(W[64 * rb:64 * rb + 64], None, cfg["seed"], row_block0=rb)
        assert np.array_equal(s[rb:rb + 1], o["scales"])
        assert np.array_equal(c[rb * per:(rb + 1) * per], o["codes"])
