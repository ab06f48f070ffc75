"""Failure path of the bounded device waits, injected from the host.

A test hook makes thread block (0, 0) skip one bulk or tensor copy (usk_build,
usk_gemv, usk_gemm); its bounded mbarrier wait gives up after about one second, sets USK_FLAG_TIMEOUT in the status word and the kernel completes.
No trap, no assert, no fault: the context stays usable, which the follow-up
call checks against the oracle."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sub_bit_weight_usk_b200 as usk
from tests.gpu_util import codes_np, rel_err, scales_np, status_tensor, to_dev

pytestmark = pytest.mark.gpu


def _inject(kind, fn):
    st = status_tensor()
    usk.usk_debug_inject_timeout(kind)
    try:
        fn(st)
        torch.cuda.synchronize()
    finally:
        usk.usk_debug_inject_timeout(0)
    return int(st.item())


def test_build_wait_timeout_reported_then_recovers():
    W = gen.weights_normal(64, 256, 1, 0.02, "bf16")  # one block, one tile
    flags = _inject(1, lambda st: usk.usk_build(to_dev(W), None, 0, status=st))
    assert flags & usk.FLAG_TIMEOUT
    st = status_tensor()
    sk = usk.usk_build(to_dev(W), None, 0, status=st)
    o = oracle.build_sketch(W, None, 0)
    assert int(st.item()) == 0
    assert np.array_equal(codes_np(sk), o["codes"]) and np.array_equal(scales_np(sk), o["scales"])


def test_gemm_wait_timeout_reported_then_recovers():
    W = gen.weights_normal(128, 256, 2, 0.02, "bf16")  # one block; the x copy of its first chunk is skipped
    sk = usk.usk_build(to_dev(W), None, 1)
    x = gen.activations(16, 256, 3, "bf16")
    flags = _inject(2, lambda st: usk.usk_gemm(sk, to_dev(x), status=st))
    assert flags & usk.FLAG_TIMEOUT
    st = status_tensor()
    y = usk.usk_gemm(sk, to_dev(x), status=st).cpu().numpy()
    assert int(st.item()) == 0
    o = oracle.build_sketch(W, None, 1)
    assert rel_err(y, oracle.gemv_f64(o["codes"], o["scales"], 128, 256, x, 1)) <= 1e-3


@pytest.mark.parametrize("path", [2, 3, 4])
def test_gemv_wait_timeout_reported_then_recovers(path):
    """Path 3 skips a code copy; paths 2 and 4 (no copies) have block 1 of row
    block 0 skip its partial sums, so the first block's wait gives up (K spans
    two blocks of the path's default tiles per block: 8 for path 2, 4 for 4)."""
    K = {2: 4096, 3: 256, 4: 2048}[path]
    W = gen.weights_normal(64, K, 4, 0.02, "bf16")
    sk = usk.usk_build(to_dev(W), None, 2)
    x = gen.activations(1, K, 5, "bf16")
    usk.usk_debug_set_gemv_path(path)
    try:
        flags = _inject(3, lambda st: usk.usk_gemv(sk, to_dev(x), status=st))
        assert flags & usk.FLAG_TIMEOUT
        st = status_tensor()
        y = usk.usk_gemv(sk, to_dev(x), status=st).cpu().numpy()
    finally:
        usk.usk_debug_set_gemv_path(0)
    assert int(st.item()) == 0
    o = oracle.build_sketch(W, None, 2)
    assert rel_err(y, oracle.gemv_f64(o["codes"], o["scales"], 64, K, x, 2)) <= (1e-3 if path == 4 else 1e-6)
