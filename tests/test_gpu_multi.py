"""usk_gemv_multi (several independent products in one persistent launch) on
the GPU against the float64 oracle products on the same sketches.

Tolerance: max|y - y_ref| <= 1e-3 max|y_ref| over every output of every
product.  Every product runs on a sketch the ORACLE built (uploaded), so no
expected value depends on the CUDA build.  Shapes span one-chunk rows (K <=
1024, no workspace), rows split over several 1024-column chunks (summed
through the workspace), a ragged last chunk (K = 11008 = 43 tiles), several
linears of different shapes in one list, batches 1..8 and every format the
call takes."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import rel_err, sketch_from_oracle, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _oracle_sketch(M, K, seed, fmt="f1", slots=4, depth=1):
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.001, 20.0, "bf16")
    if fmt == "f1" and slots == 4:
        o = oracle.build_sketch(W, None, seed)
        sk = sketch_from_oracle(o, M, K, seed)
        ref = lambda x, rows=None: oracle.gemv_f64(o["codes"], o["scales"], M, K, x, seed, rows=rows)  # noqa: E731
    elif fmt == "f1":
        o = oracle.build_sketch_rate(W, None, seed, slots)
        sk = sketch_from_oracle(o, M, K, seed)
        sk.slots = slots
        ref = lambda x, rows=None: oracle.gemv_rate_f64(o["codes"], o["scales"], M, K, x, seed, slots,  # noqa: E731
                                                        rows=rows)
    elif fmt == "amm":
        o = oracle.build_sketch_amm(W, seed, depth)
        sk = sketch_from_oracle(o, M, K, seed, usk.FORMAT_ABSMAXMIN, depth)
        ref = lambda x, rows=None: oracle.gemv_amm_f64(o["codes"], o["scales"], M, K, x, seed, depth,  # noqa: E731
                                                       rows=rows)
    else:
        o = oracle.build_sketch_q4(W, None, seed)
        sk = sketch_from_oracle(o, M, K, seed, usk.FORMAT_Q4, 1)
        ref = lambda x, rows=None: oracle.gemv_q4_f64(o["codes"], o["scales"], M, K, x, seed, rows=rows)  # noqa: E731
    return sk, ref


def _run_and_check(cases, batch, pdl=False, rows=None):
    sks = [c[0] for c in cases]
    xs = [gen.activations(batch, sk.K, 100 + i, "bf16") for i, sk in enumerate(sks)]
    st = status_tensor()
    need = usk.usk_gemv_multi_ws_bytes(sks, batch)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    xd = [to_dev(x) for x in xs]
    ys = usk.usk_gemv_multi(sks, xd, ws=ws, status=st, pdl=pdl)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # a second call on the same workspace (its counters must be back at zero)
    # overwrites every output with the same bits
    ys2 = [torch.full_like(y, float("nan")) for y in ys]
    usk.usk_gemv_multi(sks, xd, ys2, ws=ws, status=st, pdl=pdl)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for y, y2 in zip(ys, ys2):
        assert torch.equal(y, y2), "second call on the same workspace differs"
    out = []
    for (sk, ref), x, y in zip(cases, xs, ys):
        yy = y.cpu().numpy()
        r = ref(x, rows)
        if rows is not None:
            yy = yy[:, rows]
        e = rel_err(yy, r)
        assert e <= TOL, "relative error %.3e (M=%d K=%d batch=%d)" % (e, sk.M, sk.K, batch)
        out.append(yy)
    return out


@pytest.mark.parametrize("M,K", [(64, 256), (128, 1024), (192, 1280), (128, 4096), (64, 11008), (320, 2816)])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8])
def test_multi_single_linear(M, K, batch):
    _run_and_check([_oracle_sketch(M, K, 31)], batch)


@pytest.mark.parametrize("batch", [1, 4, 8])
def test_multi_mixed_list(batch):
    """Linears of different shapes in one launch, one-chunk and split rows mixed."""
    shapes = [(64, 256), (256, 4096), (128, 11008), (448, 1024), (64, 2816), (192, 4352)]
    _run_and_check([_oracle_sketch(M, K, 40 + i) for i, (M, K) in enumerate(shapes)], batch, pdl=True)


@pytest.mark.parametrize("fmt,slots,depth", [("f1", 2, 1), ("f1", 8, 1), ("amm", 4, 2), ("amm", 4, 4), ("q4", 8, 1)])
@pytest.mark.parametrize("batch", [1, 4])
def test_multi_formats(fmt, slots, depth, batch):
    cases = [_oracle_sketch(M, K, 50 + i, fmt, slots, depth) for i, (M, K) in enumerate([(128, 4096), (64, 1024),
                                                                                         (192, 2816)])]
    _run_and_check(cases, batch)


def test_multi_llama7b_layer_set_sampled():
    """q, k, v of a 7B layer in one call and gate+up in another (the grouping a
    transformer's data flow allows), sampled rows over every row block's end."""
    rows_q = np.array([0, 63, 64, 2048, 4031, 4095])
    q = [_oracle_sketch(4096, 4096, 60 + i) for i in range(3)]
    _run_and_check(q, 1, pdl=True, rows=rows_q)
    rows_g = np.array([0, 1, 5503, 11007])
    gu = [_oracle_sketch(11008, 4096, 70 + i) for i in range(2)]
    _run_and_check(gu, 1, rows=rows_g)


def test_multi_repeatable_and_matches_gemv():
    """Bitwise repeatable across calls that share one workspace; within the
    tolerance of usk_gemv on the same sketch."""
    sk, ref = _oracle_sketch(256, 11008, 81)
    x = to_dev(gen.activations(2, 11008, 82, "bf16"))
    ws = torch.zeros(usk.usk_gemv_multi_ws_bytes([sk], 2), dtype=torch.uint8, device="cuda")
    a = usk.usk_gemv_multi([sk], [x], ws=ws)[0].clone()
    for _ in range(3):
        b = usk.usk_gemv_multi([sk], [x], ws=ws, pdl=True)[0]
        assert torch.equal(a, b)
    y1 = usk.usk_gemv(sk, x)
    e = rel_err(a.cpu().numpy(), y1.cpu().numpy().astype(np.float64))
    assert e <= TOL


def test_multi_zero_sizes_and_empty():
    sk, _ = _oracle_sketch(64, 256, 90)
    empty = usk.Sketch(0, 256, 0, torch.zeros(0, dtype=torch.int8, device="cuda"),
                       torch.zeros(0, dtype=torch.int16, device="cuda"))
    x = to_dev(gen.activations(1, 256, 91, "bf16"))
    ys = usk.usk_gemv_multi([sk, empty], [x, x], ys=[torch.full((1, 64), 7.0, device="cuda"),
                                                     torch.empty((1, 0), device="cuda")])
    assert torch.isfinite(ys[0]).all()
    kz = usk.Sketch(64, 0, 0, torch.zeros(0, dtype=torch.int8, device="cuda"),
                    torch.zeros(1, dtype=torch.int16, device="cuda"))
    yz = torch.full((1, 64), 7.0, device="cuda")
    usk.usk_gemv_multi([kz], [torch.zeros((1, 0), dtype=torch.bfloat16, device="cuda")], ys=[yz])
    torch.cuda.synchronize()
    assert torch.count_nonzero(yz).item() == 0


def test_multi_argument_errors():
    sk, _ = _oracle_sketch(128, 4096, 93)
    x = to_dev(gen.activations(1, 4096, 94, "bf16"))
    with pytest.raises(usk.UskError) as e:  # workspace too small
        usk.usk_gemv_multi([sk], [x], ws=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 5
    cs = usk.usk_build(to_dev(gen.weights_normal(128, 4096, 1)), None, 1, version=usk.FORMAT_COLSHARED)
    with pytest.raises(usk.UskError) as e:
        usk.usk_gemv_multi([cs], [x])
    assert e.value.status == 6
    amm, _ = _oracle_sketch(128, 4096, 95, "amm", 4, 2)
    with pytest.raises(usk.UskError) as e:  # formats mixed in one list
        usk.usk_gemv_multi([sk, amm], [x, x])
    assert e.value.status == 6
    with pytest.raises(usk.UskError) as e:  # batch 9
        usk.usk_gemv_multi([sk], [to_dev(gen.activations(9, 4096, 1, "bf16"))])
    assert e.value.status == 4


def test_multi_injected_timeout_recovers():
    """Host-made failure: block 0 never issues one copy; its bounded wait gives
    up, USK_FLAG_TIMEOUT is set, and the context still computes correctly."""
    sk, ref = _oracle_sketch(128, 4096, 97)
    x = gen.activations(1, 4096, 98, "bf16")
    st = status_tensor()
    ws = torch.zeros(usk.usk_gemv_multi_ws_bytes([sk], 1), dtype=torch.uint8, device="cuda")
    usk.usk_debug_inject_timeout(4)
    try:
        usk.usk_gemv_multi([sk], [to_dev(x)], ws=ws, status=st)
        torch.cuda.synchronize()
    finally:
        usk.usk_debug_inject_timeout(0)
    assert int(st.item()) & usk.FLAG_TIMEOUT
    ws.zero_()
    _run_and_check([(sk, ref)], 1)
