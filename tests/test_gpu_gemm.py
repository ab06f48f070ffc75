"""usk_gemm (tcgen05 tensor cores) on the GPU against the float64 oracle product.

Tolerance: max|y - y_ref| <= 1e-3 * max|y_ref| (bf16 x, exact bf16 products,
fp32 accumulation in tensor memory)."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, sketch_from_oracle, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _sketch(W, seed, imp=None):
    """The oracle's sketch of W, uploaded (the build kernel is pinned elsewhere)."""
    o = oracle.build_sketch(W, imp, seed)
    assert o["status"] == oracle.OK
    return sketch_from_oracle(o, W.shape[0], W.shape[1], seed), o


def _check(sk, o, x, rows=None):
    st = status_tensor()
    y = usk.usk_gemm(sk, to_dev(x), status=st).cpu().numpy()
    assert int(st.item()) == 0
    ref = oracle.gemv_f64(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed, rows=rows)
    if rows is not None:
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e


@pytest.mark.parametrize("M,K", [(128, 256), (192, 1024), (128, 4352), (320, 2048)])
@pytest.mark.parametrize("batch", [16, 32, 48, 64, 128, 256])
def test_gemm_matches_oracle(M, K, batch):
    W = gen.weights_student_t(M, K, 11, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _sketch(W, 5)
    x = gen.activations(batch, K, 12, "bf16")
    _check(sk, o, x)


def test_gemm_on_gpu_built_sketch():
    """The whole product path: GPU build (checked bit-exact) then GPU GEMM."""
    W = gen.weights_normal(256, 1024, 13, 0.02, "bf16")
    o = oracle.build_sketch(W, None, 6)
    sk = usk.usk_build(to_dev(W), None, 6)
    torch.cuda.synchronize()
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])
    _check(sk, o, gen.activations(16, 1024, 14, "bf16"))


@pytest.mark.parametrize("batch", [16, 64])
def test_gemm_layer_workload_full(batch):
    cfg = gen.layer(batch)
    sk, o = _sketch(cfg["W"], cfg["seed"], cfg["importance"])
    _check(sk, o, cfg["x"])


@pytest.mark.parametrize("name", ["up", "down"])
def test_gemm_mlp70b_sampled_rows(name):
    cfg = gen.mlp70b(name, 64)
    sk, o = _sketch(cfg["W"], cfg["seed"])
    M = sk.M
    rows = np.array([0, 1, 127, 128, M // 2, M - 65, M - 1])
    _check(sk, o, cfg["x"], rows=rows)


def test_gemm_matches_gemv_on_same_sketch():
    W = gen.weights_normal(256, 2048, 15, 0.02, "bf16")
    sk, _ = _sketch(W, 7)
    x = to_dev(gen.activations(16, 2048, 16, "bf16"))
    yg = usk.usk_gemm(sk, x)
    yv = torch.cat([usk.usk_gemv(sk, x[i:i + 8]) for i in range(0, 16, 8)])
    d = (yg - yv).abs().max().item() / yv.abs().max().item()
    assert d <= 1e-5


def test_gemm_repeatable_bitwise():
    W = gen.weights_normal(512, 4096, 17, 0.02, "bf16")
    sk, _ = _sketch(W, 8)
    x = to_dev(gen.activations(32, 4096, 18, "bf16"))
    a = usk.usk_gemm(sk, x)
    for _ in range(3):
        assert torch.equal(a, usk.usk_gemm(sk, x))


def test_gemm_zero_sketch_and_errors():
    sk, _ = _sketch(np.zeros((128, 512), np.float32), 3)
    y = usk.usk_gemm(sk, to_dev(gen.activations(16, 512, 1, "bf16")))
    assert torch.count_nonzero(y).item() == 0
    x = to_dev(gen.activations(24, 512, 1, "bf16"))
    with pytest.raises(usk.UskError) as e:
        usk.usk_gemm(sk, x)  # not a multiple of 16
    assert e.value.status == 4
    with pytest.raises(usk.UskError) as e:
        usk.usk_gemm(sk, x[:8])  # below 16: usk_gemv's range
    assert e.value.status == 4


@pytest.mark.parametrize("issuers", [1, 2, 4])
@pytest.mark.parametrize("batch", [16, 48, 64, 128])
def test_gemm_issuer_counts(issuers, batch):
    """Every MMA issuer count the planner may pick (forced through the test
    hook where it does not exceed the batch's default), with and without a K
    split: same products within the tolerance."""
    W = gen.weights_student_t(512, 2048, 13, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _sketch(W, 21)
    x = gen.activations(batch, 2048, 22, "bf16")
    try:
        usk.usk_debug_set_gemm_issuers(issuers)
        for splits in (0, 1, 2):
            usk.usk_debug_set_gemm_splits(splits)
            _check(sk, o, x)
    finally:
        usk.usk_debug_set_gemm_issuers(0)
        usk.usk_debug_set_gemm_splits(0)


@pytest.mark.parametrize("M,K,batch", [(256, 1024, 16), (128, 4352, 64), (4096, 4096, 16)])
def test_gemm_pdl_after_producer(M, K, batch):
    """Launched as a programmatic dependent: x is written by the kernel just
    before (after a long spin, so an early read would see the zeros), y is
    filled with NaN by another kernel before that; the dependent GEMM gives the
    bits of the plain launch."""
    W = gen.weights_student_t(M, K, 17, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _sketch(W, 8)
    xh = gen.activations(batch, K, 18, "bf16")
    x_src = to_dev(xh)
    ref = usk.usk_gemm(sk, x_src).clone()
    st = status_tensor()
    x = torch.zeros_like(x_src)
    y = torch.empty((batch, M), dtype=torch.float32, device="cuda")
    for _ in range(3):
        x.zero_()
        y.fill_(float("nan"))
        torch.cuda._sleep(2_000_000)
        torch.mul(x_src, 1, out=x)
        usk.usk_gemm(sk, x, y=y, status=st, pdl=True)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert torch.equal(y, ref), "dependent launch differs from the plain one"
    e = rel_err(y.cpu().numpy(), oracle.gemv_f64(o["codes"], o["scales"], M, K, xh, sk.seed))
    assert e <= TOL


def test_gemm_pdl_chain_in_graph():
    """A CUDA graph of back-to-back dependent GEMMs, each reading the x that the
    elementwise kernel before it wrote and writing its own y: every output has
    the bits of the plain launch."""
    shapes = [(256, 1024), (4096, 4096), (128, 4352), (4096, 4096)]
    sks, xs_src, refs = [], [], []
    for i, (M, K) in enumerate(shapes):
        W = gen.weights_normal(M, K, 30 + i, 0.02, "bf16")
        sk, _ = _sketch(W, 40 + i)
        sks.append(sk)
        xs_src.append(to_dev(gen.activations(16 * (1 + i % 2), K, 50 + i, "bf16")))
        refs.append(usk.usk_gemm(sk, xs_src[-1]).clone())
    xs = [torch.zeros_like(x) for x in xs_src]
    ys = [torch.full_like(r, float("nan")) for r in refs]
    st = status_tensor()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for sk, xsrc, x, y in zip(sks, xs_src, xs, ys):
            torch.mul(xsrc, 1, out=x)
            usk.usk_gemm(sk, x, y=y, status=st, pdl=True)
    for _ in range(2):
        for x, y in zip(xs, ys):
            x.zero_()
            y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for y, r in zip(ys, refs):
            assert torch.equal(y, r)
    del g


def test_gemm_pdl_back_to_back_same_output():
    """Dependent GEMMs one after another on one y: each launch starts while the
    one before runs (that one triggers its dependents early), and y ends with
    the last product's bits (no write of an earlier launch lands after it)."""
    M, K = 4096, 4096
    a, _ = _sketch(gen.weights_normal(M, K, 61, 0.02, "bf16"), 62)
    b, _ = _sketch(gen.weights_normal(M, K, 63, 0.02, "bf16"), 64)
    x = to_dev(gen.activations(16, K, 65, "bf16"))
    ref_b = usk.usk_gemm(b, x).clone()
    ref_a = usk.usk_gemm(a, x).clone()
    y = torch.empty_like(ref_b)
    for n in (2, 5, 8):
        y.fill_(float("nan"))
        for i in range(n):
            usk.usk_gemm(a if (n - 1 - i) % 2 else b, x, y=y, pdl=True)
        torch.cuda.synchronize()
        assert torch.equal(y, ref_b)
    usk.usk_gemm(a, x, y=y, pdl=True)
    torch.cuda.synchronize()
    assert torch.equal(y, ref_a)


@pytest.mark.parametrize("fmt", ["amm2", "amm4", "q4"])
def test_gemm_pdl_formats(fmt):
    """Formats 2 (depth 2, 4) and 4 as programmatic dependents of the kernel that
    writes x: the plain launch's bits, and within the tolerance of the oracle."""
    M, K = 256, 2048
    W = gen.weights_student_t(M, K, 74, 4.0, 0.02, 0.001, 20.0, "bf16")
    if fmt == "q4":
        o = oracle.build_sketch_q4(W, None, 15)
        sk = sketch_from_oracle(o, M, K, 15, usk.FORMAT_Q4, 1)
        ref_fn = lambda xh: oracle.gemv_q4_f64(o["codes"], o["scales"], M, K, xh, 15)  # noqa: E731
    else:
        d = 2 if fmt == "amm2" else 4
        o = oracle.build_sketch_amm(W, 15, d)
        sk = sketch_from_oracle(o, M, K, 15, usk.FORMAT_ABSMAXMIN, d)
        ref_fn = lambda xh: oracle.gemv_amm_f64(o["codes"], o["scales"], M, K, xh, 15, d)  # noqa: E731
    xh = gen.activations(32, K, 75, "bf16")
    x_src = to_dev(xh)
    ref = usk.usk_gemm(sk, x_src).clone()
    x = torch.zeros_like(x_src)
    y = torch.full_like(ref, float("nan"))
    torch.cuda._sleep(1_000_000)
    torch.mul(x_src, 1, out=x)
    usk.usk_gemm(sk, x, y=y, pdl=True)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    assert rel_err(y.cpu().numpy(), ref_fn(xh)) <= TOL
