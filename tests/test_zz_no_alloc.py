"""usk_gemv_multi_static -- the products of usk_gemv_multi for callers that may
not allocate device memory (a host engine or plug-in that owns every device
buffer but the inputs and outputs it hands over, or a loop that must not call
cudaMalloc after start-up): its scratch is a fixed array inside the library.

Called here through the C ABI itself (ctypes on libusk.so), twice in a row,
and compared with usk_gemv_multi, the entry point that takes a caller
workspace, within the tolerance of every product test here:
max|y - y_ref| <= 1e-3 max|y_ref|.  A list whose scratch exceeds the fixed
array must be refused before anything runs.  This file is collected last so
that a stop at its first failure still runs every other test."""
import ctypes

import numpy as np
import pytest
import torch

import gen
import sub_bit_weight_usk_b200 as usk
from sub_bit_weight_usk_b200 import _native
from tests.gpu_util import rel_err, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3
STATIC_BYTES = 512 * 1024  # USK_GEMV_MULTI_STATIC_BYTES in include/usk.h


def _sketches(shapes, seed0):
    out = []
    for i, (M, K) in enumerate(shapes):
        W = gen.weights_student_t(M, K, seed0 + i, 4.0, 0.02, 0.001, 20.0, "bf16")
        out.append(usk.usk_build(to_dev(W), None, seed0 + i))
    torch.cuda.synchronize()
    return out


def _call_static(sks, xs, ys, status):
    """One raw C-ABI call of usk_gemv_multi_static on the current stream."""
    lib = _native.load_library()
    n = len(sks)
    cs = [sk.as_c() for sk in sks]
    arr = (_native.UskSketchC * n)(*cs)
    xp = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
    yp = (ctypes.c_void_p * n)(*[y.data_ptr() for y in ys])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.usk_gemv_multi_static(n, arr, xp, _native.USK_BF16, xs[0].shape[0], yp, 0,
                                     ctypes.c_void_p(status.data_ptr()), stream)


@pytest.mark.parametrize("shapes,batch", [
    ([(4096, 4096)], 1),                                   # one layer, rows split over the GPU
    ([(256, 4096), (128, 11008), (448, 1024)], 4),         # a mixed list, split and whole rows
    ([(4096, 4096), (4096, 4096), (4096, 4096)], 1),       # q, k, v of a 7B layer
])
def test_static_scratch_matches_the_workspace_call(shapes, batch):
    sks = _sketches(shapes, 300)
    xs = [to_dev(gen.activations(batch, sk.K, 400 + i, "bf16")) for i, sk in enumerate(sks)]
    need = usk.usk_gemv_multi_ws_bytes(sks, batch)
    assert need <= STATIC_BYTES
    ref = usk.usk_gemv_multi(sks, xs, ws=torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda"))
    st = status_tensor()
    for call in range(2):  # two calls in a row share the fixed array
        ys = [torch.full((batch, sk.M), float("nan"), device="cuda") for sk in sks]
        assert _call_static(sks, xs, ys, st) == 0
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for y, r in zip(ys, ref):
            e = rel_err(y.cpu().numpy(), r.cpu().numpy().astype(np.float64))
            assert e <= TOL, "call %d: relative error %.3e" % (call, e)


def test_static_scratch_refuses_lists_that_do_not_fit():
    sks = _sketches([(4096, 4096)], 500)
    x = to_dev(gen.activations(8, 4096, 501, "bf16"))
    need = usk.usk_gemv_multi_ws_bytes(sks, 8)
    y = torch.full((8, 4096), 7.0, device="cuda")
    st = status_tensor()
    rc = _call_static(sks, [x], [y], st)
    torch.cuda.synchronize()
    if need > STATIC_BYTES:
        assert rc == 5  # USK_ERR_WORKSPACE, nothing launched
        assert torch.all(y == 7.0)
    else:
        assert rc == 0
