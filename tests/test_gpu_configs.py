"""The five workload configurations end to end on the GPU against the oracle.

Builds are compared bit-exact (whole matrices, up to 28672 x 8192; the whole
32-layer stack is tests/test_gpu_stack7b.py); products run on the ORACLE's
sketch, uploaded, within max|y - y_ref| <= 1e-3 max|y_ref| on every output (the
oracle's all-core mode computes the float64 products of the largest shapes in
seconds).  The kernels run in the launch configurations the library picks for
these shapes."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, sketch_from_oracle, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _build_checked(W, imp, seed):
    """GPU build compared bit-exact with the oracle's; returns the oracle's
    sketch uploaded (for the products) and the oracle's arrays."""
    sk = usk.usk_build(to_dev(W), None if imp is None else to_dev(imp), seed)
    torch.cuda.synchronize()
    o = oracle.build_sketch_mt(W, imp, seed)
    assert o["status"] == 0
    assert np.array_equal(scales_np(sk), o["scales"]), "scales differ"
    assert np.array_equal(codes_np(sk), o["codes"]), "codes differ"
    return sketch_from_oracle(o, W.shape[0], W.shape[1], seed), o


def _build(W, imp, seed):
    sk = usk.usk_build(to_dev(W), None if imp is None else to_dev(imp), seed)
    torch.cuda.synchronize()
    return sk, codes_np(sk), scales_np(sk)


def _check_rows_built(W, seed, c, s, row_blocks):
    per = 4 * W.shape[1]
    for rb in row_blocks:
        o = oracle.build_sketch(W[64 * rb:64 * rb + 64], None, seed, row_block0=rb)
        assert np.array_equal(s[rb:rb + 1], o["scales"]), "scale of row block %d" % rb
        assert np.array_equal(c[rb * per:(rb + 1) * per], o["codes"]), "codes of row block %d" % rb


def _check_product(sk, o, x, rows=None, gemm=False):
    xd = to_dev(x)
    y = (usk.usk_gemm(sk, xd) if gemm else usk.usk_gemv(sk, xd)).cpu().numpy()
    if rows is None:
        ref = oracle.gemv_f64_mt(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed)
    else:
        ref = oracle.gemv_f64(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed, rows=rows)
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e


def test_config_small_fp32():
    """256x1024 fp32 weights, lognormal importance, GEMV at batch 1 (fp32 and bf16 x)."""
    cfg = gen.small("f32")
    sk, o = _build_checked(cfg["W"], cfg["importance"], cfg["seed"])
    _check_product(sk, o, cfg["x"])
    _check_product(sk, o, gen.small("bf16")["x"])


def test_config_layer_4096():
    """One 4096x4096 layer with outliers and calibration importance; GEMV at 1 and 4."""
    cfg = gen.layer(4)
    sk, o = _build_checked(cfg["W"], cfg["importance"], cfg["seed"])
    _check_product(sk, o, cfg["x"][:1])
    _check_product(sk, o, cfg["x"])


@pytest.mark.parametrize("name", gen.LLAMA7B_ORDER)
def test_config_llama7b_layer_set(name):
    """Every linear of the 7B layer set: whole build bit-exact, GEMV at batch 1
    and 4, GEMM at batch 16, every output."""
    cfg = gen.llama7b_layer(name, 16)
    W = cfg["W"]
    sk, o = _build_checked(W, None, cfg["seed"])
    _check_product(sk, o, cfg["x"][:1])
    _check_product(sk, o, cfg["x"][:4])
    _check_product(sk, o, cfg["x"], gemm=True)


@pytest.mark.parametrize("name", ["up", "down"])
def test_config_mlp70b(name):
    """28672x8192 and 8192x28672: the whole build bit-exact, GEMM at 16, 32 and
    64 and GEMV at 1, every output (every row tile and K split)."""
    cfg = gen.mlp70b(name, 64)
    W = cfg["W"]
    sk, o = _build_checked(W, None, cfg["seed"])
    _check_product(sk, o, cfg["x"][:16], gemm=True)
    _check_product(sk, o, cfg["x"][:32], gemm=True)
    _check_product(sk, o, cfg["x"], gemm=True)
    _check_product(sk, o, cfg["x"][:1])


@pytest.mark.parametrize("layer,linear", [(0, "q"), (0, "down"), (17, "gate"), (31, "o"), (31, "up")])
def test_config_stack7b_sampled(layer, linear):
    """Linears of the 32-layer stack (their own seeds): sampled row blocks of the
    build and a batch-1 GEMV on sampled rows."""
    seed = gen.stack7b_seed(layer, linear)
    M, K = gen.LLAMA7B_SHAPES[linear]
    W = gen.weights_normal(M, K, seed, 0.02, "bf16")
    sk, c, s = _build(W, None, seed)
    RB = M // 64
    _check_rows_built(W, seed, c, s, (0, RB // 3, RB - 1))
    o = oracle.build_sketch(W, None, seed)
    x = gen.activations(1, K, seed, "bf16")
    _check_product(sketch_from_oracle(o, M, K, seed), o, x, rows=np.array([0, 64 * (RB // 3) + 7, M - 1]))
