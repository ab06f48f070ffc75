"""Per-row-block rates on the GPU: every 64-row block of a format-1 sketch has
its own slot count (2, 4 or 8 hash slots per class), the table in a rate map
("UltraSketchLLM" explainer, Resumen Tecnico, Metodologia §2: rows of higher
importance E[a^2] receive larger sketch spaces).  Builds bit-exact against the
CPU oracle; products on ORACLE-built sketches within
max|y - y_ref| <= 1e-3 max|y_ref| of the oracle's float64 product."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _gpu_build(W, imp, seed, rm, status=None):
    sk = usk.usk_build(to_dev(W), None if imp is None else to_dev(imp), seed, status=status, rates=rm)
    torch.cuda.synchronize()
    return sk


def _compare_build(W, imp, seed, slots):
    o = oracle.build_sketch_vr(W, imp, seed, slots)
    assert o["status"] == oracle.OK
    rm = usk.usk_rate_map(W.shape[0], W.shape[1], slots)
    st = status_tensor()
    sk = _gpu_build(W, imp, seed, rm, st)
    assert int(st.item()) == 0
    assert np.array_equal(scales_np(sk), o["scales"]), "scales differ"
    bad = np.nonzero(codes_np(sk) != o["codes"])[0]
    assert bad.size == 0, "codes differ at %d, first %s" % (bad.size, bad[:8])
    return o


def _oracle_sketch(W, imp, seed, slots):
    o = oracle.build_sketch_vr(W, imp, seed, slots)
    assert o["status"] == oracle.OK
    M, K = W.shape
    codes = torch.from_numpy(o["codes"].copy()).cuda()
    scales = torch.from_numpy(o["scales"].view(np.int16).copy()).cuda()
    return usk.Sketch(M, K, seed, codes, scales, usk.FORMAT_MAXKEY, 1, 0, usk.usk_rate_map(M, K, slots)), o


def _check_product(sk, o, x, rows=None, gemm=False):
    st = status_tensor()
    xd = to_dev(x)
    y = (usk.usk_gemm(sk, xd, status=st) if gemm else usk.usk_gemv(sk, xd, status=st)).cpu().numpy()
    assert int(st.item()) == 0
    ref = oracle.gemv_vr_f64(o["codes"], o["scales"], sk.M, sk.K, x, sk.seed, sk.rates.slots, rows=rows)
    if rows is not None:
        y = y[:, rows]
    e = rel_err(y, ref)
    assert e <= TOL, "relative error %.3e" % e


TABLES = [[2, 8, 4], [8, 2, 2, 4, 8], [4, 4, 2], [8], [2, 2, 8, 8, 4, 4, 2]]


@pytest.mark.parametrize("slots", TABLES)
@pytest.mark.parametrize("K", [256, 1024, 2816, 4352])
@pytest.mark.parametrize("wdtype", ["bf16", "f32"])
@pytest.mark.parametrize("with_imp", [False, True])
def test_vr_build_bit_exact(slots, K, wdtype, with_imp):
    M = 64 * len(slots)
    W = gen.weights_student_t(M, K, 61, 4.0, 0.02, 0.001, 20.0, wdtype)
    imp = gen.importance_lognormal(K, 61) if with_imp else None
    _compare_build(W, imp, 17, slots)


@pytest.mark.parametrize("cluster", [1, 3, 8])
def test_vr_build_geometry_independent(cluster):
    slots = [8, 2, 4, 2]
    W = gen.weights_student_t(256, 4352, 62, 4.0, 0.02, 0.001, 20.0, "bf16")
    imp = gen.importance_lognormal(4352, 62)
    o = oracle.build_sketch_vr(W, imp, 3, slots)
    usk.usk_debug_set_geometry(cluster, 0)
    try:
        sk = _gpu_build(W, imp, 3, usk.usk_rate_map(256, 4352, slots))
    finally:
        usk.usk_debug_set_geometry(0, 0)
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])


def test_vr_uniform_table_equals_the_rate_sketch():
    """A table of one slot count gives the bytes of the per-sketch rate build."""
    W = gen.weights_student_t(192, 2048, 63, 4.0, 0.02, 0.001, 20.0, "bf16")
    for S in (2, 4, 8):
        a = _gpu_build(W, None, 5, usk.usk_rate_map(192, 2048, [S] * 3))
        b = usk.usk_build(to_dev(W), None, 5, slots=S)
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)


@pytest.mark.parametrize("slots", TABLES)
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
def test_vr_gemv_matches_oracle(slots, xdtype):
    M, K = 64 * len(slots), 2816
    W = gen.weights_student_t(M, K, 64, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 9, slots)
    for batch in (1, 4, 9, 15):
        _check_product(sk, o, gen.activations(batch, K, 65, xdtype))


@pytest.mark.parametrize("path", [1, 2, 3, 4])
def test_vr_gemv_paths_and_pdl(path):
    """Forced paths: the integer paths read uniform 4-slot sketches only, so a
    rate map takes a bf16 path; a PDL launch gives the same y."""
    slots = [8, 2, 4, 2, 8]
    W = gen.weights_student_t(320, 1024, 66, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 10, slots)
    usk.usk_debug_set_gemv_path(path)
    try:
        for batch in (1, 4):
            x = gen.activations(batch, 1024, 67, "bf16")
            _check_product(sk, o, x)
            a = usk.usk_gemv(sk, to_dev(x))
            assert torch.equal(a, usk.usk_gemv(sk, to_dev(x), pdl=True))
    finally:
        usk.usk_debug_set_gemv_path(0)


@pytest.mark.parametrize("tpc", [1, 3, 8])
def test_vr_gemv_geometries(tpc):
    slots = [2, 4, 8, 4]
    W = gen.weights_student_t(256, 4352, 68, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 11, slots)
    usk.usk_debug_set_geometry(0, tpc)
    try:
        for batch in (1, 5, 12):
            _check_product(sk, o, gen.activations(batch, 4352, 69, "bf16"))
    finally:
        usk.usk_debug_set_geometry(0, 0)


@pytest.mark.parametrize("slots", [[8, 2, 2, 4, 8], [2, 8, 4], [4, 4, 2, 2, 8, 8, 8]])
@pytest.mark.parametrize("K", [256, 2048, 4352])
@pytest.mark.parametrize("batch", [16, 64, 256])
def test_vr_gemm_matches_oracle(slots, K, batch):
    """Odd group sizes leave 128-row tiles with one row block."""
    M = 64 * len(slots)
    W = gen.weights_student_t(M, K, 70, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 12, slots)
    _check_product(sk, o, gen.activations(batch, K, 71, "bf16"), gemm=True)


def _block_importance(W, x):
    """E[a^2] of each 64-row block's outputs over calibration rows x: the mean
    of (W x^T)^2 over the block's rows and the samples."""
    Wf = gen.bf16_bits_to_f32(W) if W.dtype == np.uint16 else W
    xf = gen.bf16_bits_to_f32(x) if x.dtype == np.uint16 else x
    a = xf.astype(np.float64) @ Wf.astype(np.float64).T
    return (a ** 2).reshape(a.shape[0], -1, 64).mean(axis=(0, 2))


def test_vr_allocated_mlp_layer():
    """A 28672 x 8192 layer whose row blocks differ in output energy (a
    lognormal gain per block): the allocation at 0.5 bit/weight from the
    blocks' E[a^2], the whole build against the oracle, products on sampled
    rows."""
    M, K = 28672, 8192
    RB = M // 64
    W = gen.weights_normal(M, K, 72, 0.02, "f32")
    gain = np.exp(np.random.default_rng(73).normal(0.0, 0.5, size=RB)).astype(np.float32)
    W = gen.f32_to_bf16_bits((W.reshape(RB, 64, K) * gain[:, None, None]).reshape(M, K))
    xcal = gen.activations(8, K, 74, "f32")
    imp = _block_importance(W, xcal)
    slots = usk.usk_plan_slots([64 * K] * RB, imp.tolist(), 0.5)
    assert slots == oracle.plan_slots([64 * K] * RB, imp.tolist(), 0.5)
    assert len(set(slots)) >= 2 and K * sum(slots) * 8 <= 0.5 * M * K
    o = _compare_build(W, None, 7, slots)
    sk, _ = _oracle_sketch(W, None, 7, slots)
    rows = np.array([0, 63, 64, 4095, 12800, 20031, M - 65, M - 1])
    _check_product(sk, o, gen.activations(1, K, 75, "bf16"), rows=rows)
    _check_product(sk, o, gen.activations(7, K, 75, "f32"), rows=rows)
    _check_product(sk, o, gen.activations(64, K, 75, "bf16"), rows=rows, gemm=True)


def test_vr_bad_map_entries_are_skipped_and_flagged():
    """A device table entry out of range (row block 99 of 3; an offset past the
    codes) is caught by the kernels' own checks: that row block is skipped and
    USK_FLAG_RATE_MAP set; the other blocks are still right."""
    slots = [2, 8, 4]
    M, K = 192, 1024
    W = gen.weights_student_t(M, K, 76, 4.0, 0.02, 0.001, 20.0, "bf16")
    o = oracle.build_sketch_vr(W, None, 4, slots)
    good = usk.usk_rate_map(M, K, slots)
    bad_order = usk.RateMap(slots, good.offset.clone(), good.order.clone(), good.count, good.code_bytes)
    bad_order.order[0] = 99  # the 2-slot group's only entry
    bad_off = usk.RateMap(slots, good.offset.clone(), good.order.clone(), good.count, good.code_bytes)
    # row block 1 (8 slots) would end past the codes, and row block 0's extent
    # (up to row block 1's offset) no longer matches its 2 slots: both skipped
    bad_off.offset[1] = good.code_bytes
    off = good.offset.cpu().tolist()
    x1 = to_dev(gen.activations(1, K, 77, "bf16"))
    x16 = to_dev(gen.activations(16, K, 77, "bf16"))
    for rm, skipped in ((bad_order, {0}), (bad_off, {0, 1})):
        st = status_tensor()
        codes = torch.zeros(good.code_bytes, dtype=torch.int8, device="cuda")
        scales = torch.zeros(M // 64, dtype=torch.int16, device="cuda")
        usk.usk_build(to_dev(W), None, 4, codes=codes, scales=scales, status=st, rates=rm)
        torch.cuda.synchronize()
        assert int(st.item()) & usk.FLAG_RATE_MAP
        c = codes.cpu().numpy()
        for rb, S in enumerate(slots):
            seg = slice(off[rb], off[rb] + S * K)
            if rb in skipped:
                assert not c[seg].any()
            else:
                assert np.array_equal(c[seg], o["codes"][seg])
        sk = usk.Sketch(M, K, 4, torch.from_numpy(o["codes"].copy()).cuda(),
                        torch.from_numpy(o["scales"].view(np.int16).copy()).cuda(), usk.FORMAT_MAXKEY, 1, 0, rm)
        ref = oracle.gemv_vr_f64(o["codes"], o["scales"], M, K, gen.activations(1, K, 77, "bf16"), 4, slots)
        for gemm in (False, True):
            st = status_tensor()
            x = x16 if gemm else x1
            y = torch.full((x.shape[0], M), 7.0, device="cuda")
            (usk.usk_gemm if gemm else usk.usk_gemv)(sk, x, y=y, status=st)
            torch.cuda.synchronize()
            assert int(st.item()) & usk.FLAG_RATE_MAP
            yc = y.cpu().numpy()
            keep = np.ones(M, bool)
            for rb in skipped:
                assert np.all(yc[:, 64 * rb:64 * rb + 64] == 7.0)  # not written
                keep[64 * rb:64 * rb + 64] = False
            r = ref if not gemm else oracle.gemv_vr_f64(o["codes"], o["scales"], M, K,
                                                        gen.activations(16, K, 77, "bf16"), 4, slots)
            assert rel_err(yc[:, keep], r[:, keep]) <= TOL


def test_vr_gemm_pair_keeps_the_valid_block():
    """A 128-row GEMM tile pairs two row blocks of one slot group; when one of
    them has a bad entry, only its rows are skipped: the partner block's
    outputs are still computed (GEMV and GEMM against the oracle)."""
    slots = [4, 4, 2]
    M, K = 192, 1024
    W = gen.weights_student_t(M, K, 80, 4.0, 0.02, 0.001, 20.0, "bf16")
    o = oracle.build_sketch_vr(W, None, 5, slots)
    good = usk.usk_rate_map(M, K, slots)
    assert good.order.cpu().tolist() == [2, 0, 1]  # the 2-slot group, then the 4-slot pair
    bad = usk.RateMap(slots, good.offset.clone(), good.order.clone(), good.count, good.code_bytes)
    bad.order[2] = 99  # row block 1's entry: the second block of the 4-slot tile
    sk = usk.Sketch(M, K, 5, torch.from_numpy(o["codes"].copy()).cuda(),
                    torch.from_numpy(o["scales"].view(np.int16).copy()).cuda(), usk.FORMAT_MAXKEY, 1, 0, bad)
    for batch, gemm in ((1, False), (16, True)):
        x = gen.activations(batch, K, 81, "bf16")
        st = status_tensor()
        y = torch.full((batch, M), 7.0, device="cuda")
        (usk.usk_gemm if gemm else usk.usk_gemv)(sk, to_dev(x), y=y, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) & usk.FLAG_RATE_MAP
        yc = y.cpu().numpy()
        assert np.all(yc[:, 64:128] == 7.0)
        keep = np.r_[0:64, 128:192]
        ref = oracle.gemv_vr_f64(o["codes"], o["scales"], M, K, x, 5, slots)
        assert rel_err(yc[:, keep], ref[:, keep]) <= TOL


def test_vr_timeouts_reported_then_recover():
    slots = [8, 2]
    W = gen.weights_normal(128, 2048, 78, 0.02, "bf16")
    sk, o = _oracle_sketch(W, None, 0, slots)
    x1 = gen.activations(1, 2048, 79, "bf16")
    x16 = gen.activations(16, 2048, 79, "bf16")
    rm = usk.usk_rate_map(128, 2048, slots)
    for kind, fn in ((1, lambda s: usk.usk_build(to_dev(W), None, 0, status=s, rates=rm)),
                     (2, lambda s: usk.usk_gemm(sk, to_dev(x16), status=s)),
                     (3, lambda s: usk.usk_gemv(sk, to_dev(x1), status=s))):
        st = status_tensor()
        usk.usk_debug_inject_timeout(kind)
        try:
            fn(st)
            torch.cuda.synchronize()
        finally:
            usk.usk_debug_inject_timeout(0)
        assert int(st.item()) & usk.FLAG_TIMEOUT
    _compare_build(W, None, 0, slots)
    _check_product(sk, o, x1)
    _check_product(sk, o, x16, gemm=True)


@pytest.mark.parametrize("call", ["gemm16", "gemv9", "gemv_f32"])
def test_vr_long_k_products(call):
    """K = 11008 (43 tiles) with per-row-block rates: the launches are planned
    for the 8-slot layout; each product runs and matches the oracle."""
    slots = [8, 2, 4, 8]
    M, K = 256, 11008
    W = gen.weights_normal(M, K, 82, 0.02, "bf16")
    sk, o = _oracle_sketch(W, None, 6, slots)
    if call == "gemm16":
        _check_product(sk, o, gen.activations(16, K, 83, "bf16"), gemm=True)
    elif call == "gemv9":
        _check_product(sk, o, gen.activations(9, K, 83, "bf16"))
    else:
        _check_product(sk, o, gen.activations(2, K, 83, "f32"))


@pytest.mark.parametrize("batch", [16, 64])
def test_vr_gemm_pdl(batch):
    """A rate-mapped GEMM launched as a programmatic dependent of the kernel that
    writes its x gives the plain launch's bits."""
    slots = [8, 2, 4, 2, 8]
    W = gen.weights_student_t(320, 2048, 72, 4.0, 0.02, 0.001, 20.0, "bf16")
    sk, o = _oracle_sketch(W, None, 13, slots)
    x_src = to_dev(gen.activations(batch, 2048, 73, "bf16"))
    ref = usk.usk_gemm(sk, x_src).clone()
    x = torch.zeros_like(x_src)
    y = torch.full_like(ref, float("nan"))
    torch.cuda._sleep(1_000_000)
    torch.mul(x_src, 1, out=x)
    usk.usk_gemm(sk, x, y=y, pdl=True)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
