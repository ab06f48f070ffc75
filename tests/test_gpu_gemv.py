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
from tests.gpu_util import codes_np, rel_err, scales_np, to_dev

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
    sk = usk.usk_build(to_dev(W), None, cfg["seed"])
    torch.cuda.synchronize()
    o = {"codes": codes_np(sk), "scales": scales_np(sk)}
    # the sketch itself is pinned by the build tests; here the product is
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
