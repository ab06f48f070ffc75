"""usk_gemv on the GPU against the float64 oracle product on the same sketch.

Tolerance (stated by the method's target): max|y - y_ref| <= 1e-3 * max|y_ref|
over the whole [batch, M] output.  bf16 x gives exact products in the tensor
core with fp32 accumulation; fp32 x is split into two bf16 terms."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import sketch_from_oracle, codes_np, rel_err, scales_np, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _sketch(W, imp, seed):
    sk = usk.usk_build(to_dev(W), None if imp is None else to_dev(imp), seed)
    o = oracle.build_sketch(W, imp, seed)
    torch.cuda.synchronize()
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])
    return sk, o


def _check(sk, o, x, rows=None):
    M, K = sk.M, sk.K
    y = usk.usk_gemv(sk, to_dev(x)).cpu().numpy()
    ref = oracle.gemv_f64(o["codes"], o["scales"], M, K, x, sk.seed, rows=rows)
    if rows is not None:
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e
    return e


@pytest.mark.parametrize("M,K", [(64, 256), (128, 1024), (192, 2816), (128, 4352), (64, 11008)])
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
@pytest.mark.parametrize("batch", [1, 4, 8, 9, 15])
def test_gemv_matches_oracle(M, K, xdtype, batch):
    W = gen.weights_student_t(M, K, 5, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _sketch(W, None, 77)
    x = gen.activations(batch, K, 6, xdtype)
    _check(sk, o, x)


def test_gemv_small_workload_fp32_and_bf16():
    cfg = gen.small("f32")
    sk, o = _sketch(cfg["W"], cfg["importance"], cfg["seed"])
    _check(sk, o, cfg["x"])
    _check(sk, o, gen.small("bf16")["x"])


@pytest.mark.parametrize("batch", [1, 4])
def test_gemv_layer_workload_full(batch):
    """4096x4096 at the bench's launch configuration, every output checked."""
    cfg = gen.layer(batch)
    sk, o = _sketch(cfg["W"], cfg["importance"], cfg["seed"])
    _check(sk, o, cfg["x"])


def test_gemv_llama7b_down_sampled_rows():
    cfg = gen.llama7b_layer("down", 4)
    W = cfg["W"]
    o = oracle.build_sketch(W, None, cfg["seed"])
    sk = sketch_from_oracle(o, W.shape[0], W.shape[1], cfg["seed"])
    rows = np.array([0, 1, 63, 64, 2047, 4095])
    _check(sk, o, cfg["x"], rows=rows)


def test_gemv_zero_sketch_gives_zero():
    W = np.zeros((128, 512), np.float32)
    sk, o = _sketch(W, None, 3)
    y = usk.usk_gemv(sk, to_dev(gen.activations(3, 512, 1, "bf16")))
    assert torch.count_nonzero(y).item() == 0


def test_gemv_repeatable_bitwise():
    cfg = gen.layer(4, M=1024, K=4096)
    sk, _ = _sketch(cfg["W"], cfg["importance"], cfg["seed"])
    x = to_dev(cfg["x"])
    a = usk.usk_gemv(sk, x)
    for _ in range(3):
        assert torch.equal(a, usk.usk_gemv(sk, x))


@pytest.mark.parametrize("tpc", [1, 2, 3, 5])
def test_gemv_geometry_within_tolerance(tpc):
    W = gen.weights_normal(128, 4352, 4, 0.02, "bf16")
    sk, o = _sketch(W, None, 8)
    x = gen.activations(4, 4352, 2, "bf16")
    try:
        usk.usk_debug_set_geometry(0, tpc)
        _check(sk, o, x)
    finally:
        usk.usk_debug_set_geometry(0, 0)


def test_gemv_edges_and_errors():
    W = gen.weights_normal(64, 512, 4, 0.02, "bf16")
    sk, _ = _sketch(W, None, 1)
    x = to_dev(gen.activations(16, 512, 1, "bf16"))
    with pytest.raises(usk.UskError) as e:
        usk.usk_gemv(sk, x)  # batch 16 belongs to usk_gemm
    assert e.value.status == 4
    y = usk.usk_gemv(sk, x[:0])
    assert y.shape == (0, 64)
    # K == 0 writes zeros
    empty = usk.usk_build(torch.zeros((64, 0), dtype=torch.bfloat16, device="cuda"), None, 0)
    y = torch.full((2, 64), 5.0, device="cuda")
    usk.usk_gemv(empty, torch.zeros((2, 0), dtype=torch.bfloat16, device="cuda"), y=y)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0
    # misaligned x
    buf = torch.zeros(2 * 512 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(usk.UskError) as e:
        usk.usk_gemv(sk, buf[1:1 + 2 * 512].view(2, 512))
    assert e.value.status == 10


# ------------------------------------------------------------- integer path (bf16 x, batch <= 4)

@pytest.mark.parametrize("batch", [1, 2, 3, 4])
@pytest.mark.parametrize("path", [1, 2, 3, 4])
def test_gemv_paths_match_oracle(batch, path):
    W = gen.weights_student_t(192, 2816, 7, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _sketch(W, gen.importance_lognormal(2816, 7), 19)
    x = gen.activations(batch, 2816, 8, "bf16")
    try:
        usk.usk_debug_set_gemv_path(path)
        y = usk.usk_gemv(sk, to_dev(x)).cpu().numpy()
    finally:
        usk.usk_debug_set_gemv_path(0)
    ref = oracle.gemv_f64(o["codes"], o["scales"], 192, 2816, x, 19)
    e = rel_err(y, ref)
    # the integer paths sum code * x exactly: only the final fp32 rounding remains
    assert e <= (1e-6 if path in (2, 3) else TOL), "relative error %.3e" % e


def _int_path(sk, x, pdl=False, path=2):
    usk.usk_debug_set_gemv_path(path)
    try:
        return usk.usk_gemv(sk, to_dev(x), pdl=pdl).cpu().numpy()
    finally:
        usk.usk_debug_set_gemv_path(0)


# ------------------------------------------------------------- bf16 path with x fragments from global memory

@pytest.mark.parametrize("tpc", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("M,K,batch", [(64, 256, 1), (192, 2816, 5), (128, 4352, 8), (320, 11008, 2)])
def test_gemv_direct_x_path_geometries(tpc, M, K, batch):
    """Tiles per block 1..8 (clusters of 1 to 16 blocks, ragged last block),
    every batch width of the path."""
    W = gen.weights_student_t(M, K, 31, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _sketch(W, None, 32)
    x = gen.activations(batch, K, 33, "bf16")
    usk.usk_debug_set_geometry(0, tpc)
    try:
        y = _int_path(sk, x, path=4)
    finally:
        usk.usk_debug_set_geometry(0, 0)
    assert rel_err(y, oracle.gemv_f64(o["codes"], o["scales"], M, K, x, 32)) <= TOL


def test_gemv_direct_x_path_nonfinite_x_propagates():
    W = gen.weights_normal(64, 512, 10, 0.02, "bf16")
    sk, o = _sketch(W, None, 2)
    x = gen.activations(1, 512, 5, "bf16")
    x[0, 100] = 0x7FC0  # NaN
    y = _int_path(sk, x, path=4)
    assert np.all(np.isnan(y))


# ------------------------------------------------------------- row-slab path (batch * K <= 16384)

@pytest.mark.parametrize("rows", [16, 32, 64])
@pytest.mark.parametrize("M,K,batch", [(64, 256, 1), (192, 2816, 3), (128, 4352, 2), (320, 1024, 4)])
def test_gemv_slab_rows_match_oracle(rows, M, K, batch):
    """Every slab height, ragged tile counts (11 and 17 tiles: partial copy
    groups), row blocks that are not a multiple of the slab count."""
    W = gen.weights_student_t(M, K, 21, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _sketch(W, gen.importance_lognormal(K, 21), 23)
    x = gen.activations(batch, K, 24, "bf16")
    usk.usk_debug_set_gemv_rows(rows)
    try:
        y = _int_path(sk, x, path=3)
    finally:
        usk.usk_debug_set_gemv_rows(0)
    assert rel_err(y, oracle.gemv_f64(o["codes"], o["scales"], M, K, x, 23)) <= 1e-6


@pytest.mark.parametrize("K,batch", [(16384, 1), (8192, 2), (4096, 4)])
def test_gemv_slab_largest_x(K, batch):
    """batch * K at the slab path's limit (x of the whole row in registers)."""
    W = gen.weights_normal(128, K, 25, 0.02, "bf16")
    sk, o = _sketch(W, None, 26)
    x = gen.activations(batch, K, 27, "bf16")
    y = _int_path(sk, x, path=3)
    assert rel_err(y, oracle.gemv_f64(o["codes"], o["scales"], 128, K, x, 26)) <= 1e-6


def test_gemv_slab_rows_do_not_change_result():
    W = gen.weights_normal(256, 4096, 28, 0.02, "bf16")
    sk, _ = _sketch(W, None, 29)
    x = to_dev(gen.activations(2, 4096, 30, "bf16"))
    ys = []
    usk.usk_debug_set_gemv_path(3)
    try:
        for rows in (16, 32, 64):
            usk.usk_debug_set_gemv_rows(rows)
            ys.append(usk.usk_gemv(sk, x))
    finally:
        usk.usk_debug_set_gemv_rows(0)
        usk.usk_debug_set_gemv_path(0)
    # each output is one exact integer sum rounded once: identical bits
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


@pytest.mark.parametrize("path", [2, 3])
def test_gemv_int_path_extreme_dynamic_range_is_exact(path):
    """Elements far below the block's largest leave the digit planes and are
    added by the exact correction."""
    W = gen.weights_normal(128, 2048, 9, 0.02, "bf16")
    sk, o = _sketch(W, None, 4)
    g = np.random.default_rng(3)
    xf = g.standard_normal((2, 2048)).astype(np.float32)
    xf[0, 5] = 3.0e30          # 100 binades above the rest: every other element is residual
    xf[0, 700] = 1.0e-30
    xf[1, ::7] *= np.float32(1e-12)  # a spread of 40 binades in row 1
    xf[1, 1] = 1.0e-38         # bf16 subnormal
    x = gen.f32_to_bf16_bits(xf)
    y = _int_path(sk, x, path=path)
    ref = oracle.gemv_f64(o["codes"], o["scales"], 128, 2048, x, 4)
    assert rel_err(y[0:1], ref[0:1]) <= 1e-6
    assert rel_err(y[1:2], ref[1:2]) <= 1e-6
    # the residual-only contribution of row 1 is still exact relative to itself
    small = x.copy()
    small[1, 0::7] = 0
    assert np.all(np.isfinite(y))


@pytest.mark.parametrize("path", [2, 3])
def test_gemv_int_path_nonfinite_x_propagates(path):
    W = gen.weights_normal(64, 512, 10, 0.02, "bf16")
    sk, o = _sketch(W, None, 2)
    x = gen.activations(1, 512, 5, "bf16")
    x[0, 100] = 0x7FC0  # NaN
    y = _int_path(sk, x, path=path)
    assert np.all(np.isnan(y))
    x[0, 100] = 0x7F80  # +Inf
    y = _int_path(sk, x, path=path)
    ref = oracle.gemv_f64(o["codes"], o["scales"], 64, 512, x, 2)
    assert np.array_equal(np.isnan(y), np.isnan(ref)) and np.array_equal(np.isinf(y), np.isinf(ref))
    fin = np.isfinite(ref)
    assert np.array_equal(np.sign(y[np.isinf(y)]), np.sign(ref[np.isinf(ref)]))
    assert not fin.any() or rel_err(y[fin], ref[fin]) <= 1e-6


def test_gemv_pdl_launch_matches_plain():
    W = gen.weights_normal(256, 4096, 11, 0.02, "bf16")
    sk, o = _sketch(W, None, 6)
    other = usk.usk_build(to_dev(gen.weights_normal(256, 4096, 12, 0.02, "bf16")), None, 6)
    x = to_dev(gen.activations(1, 4096, 13, "bf16"))
    plain = usk.usk_gemv(sk, x)
    ys = []
    for _ in range(3):
        usk.usk_build(to_dev(gen.weights_normal(256, 4096, 12, 0.02, "bf16")), None, 6,
                      codes=other.codes, scales=other.scales)  # a neighbour kernel that writes another sketch
        ys.append(usk.usk_gemv(sk, x, pdl=True))
    torch.cuda.synchronize()
    for yp in ys:
        assert torch.equal(yp, plain)
    ref = oracle.gemv_f64(o["codes"], o["scales"], 256, 4096, gen.activations(1, 4096, 13, "bf16"), 6)
    assert rel_err(plain.cpu().numpy(), ref) <= 1e-6
