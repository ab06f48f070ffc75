"""The C ABI without a GPU: the library loads, exports every symbol that
include/usk.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import sub_bit_weight_usk_b200 as usk
from sub_bit_weight_usk_b200 import _build, _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return _native.load_library()


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            with open(os.path.join(ROOT, "include", f)) as fh:
                names |= set(re.findall(r"USK_API\s+[\w\s\*]+?\b(usk_\w+)\s*\(", fh.read()))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"usk_build", "usk_gemv", "usk_gemm", "usk_sizes"} <= names
    raw = ctypes.CDLL(_native.LIB_PATH)
    for n in sorted(names):
        assert hasattr(raw, n), n
    assert names == set(_native.EXPORTED)


def test_sizes_and_strings(lib):
    assert usk.usk_format_version() == 4
    assert usk.usk_sizes(4096, 4096) == (4096 * 4096 // 16, 2 * 64)
    assert usk.usk_sizes(0, 0) == (0, 0)
    with pytest.raises(usk.UskError):
        usk.usk_sizes(63, 256)
    with pytest.raises(usk.UskError):
        usk.usk_sizes(64, 300)
    with pytest.raises(usk.UskError):
        usk.usk_sizes(64, 1 << 17)
    for st in range(13):
        assert lib.usk_status_str(st)
    assert lib.usk_status_str(99) == b"unknown status"


def test_argument_errors_return_before_any_launch(lib):
    p = _native.UskParams(1, 0, 0)
    fake = ctypes.c_void_p(16 * 1024)  # never dereferenced: validation fails first
    # shape
    assert lib.usk_build(fake, 1, 63, 256, 256, None, ctypes.byref(p), fake, fake, None, None) == 2
    assert lib.usk_build(fake, 1, 64, 200, 200, None, ctypes.byref(p), fake, fake, None, None) == 2
    # dtype, params, null
    assert lib.usk_build(fake, 7, 64, 256, 256, None, ctypes.byref(p), fake, fake, None, None) == 3
    assert lib.usk_build(fake, 1, 64, 256, 256, None, None, fake, fake, None, None) == 6
    # unknown format, bad depth for the format, reserved bits, importance with format 2
    for bad in (_native.UskParams(5, 0, 0, 1, 0), _native.UskParams(4, 0, 0, 2, 0), _native.UskParams(1, 0, 0, 1, 3),
                _native.UskParams(4, 0, 0, 1, 4), _native.UskParams(2, 0, 0, 2, 8), _native.UskParams(3, 0, 0, 2, 0), _native.UskParams(2, 0, 0, 0, 0), _native.UskParams(2, 0, 0, 3, 0),
                _native.UskParams(1, 0, 0, 2, 0), _native.UskParams(1, 1, 0, 1, 0)):
        assert lib.usk_build(fake, 1, 64, 256, 256, None, ctypes.byref(bad), fake, fake, None, None) == 6
    amm = _native.UskParams(2, 0, 0, 2, 0)
    assert lib.usk_build(fake, 1, 64, 256, 256, fake, ctypes.byref(amm), fake, fake, None, None) == 6
    assert lib.usk_build(None, 1, 64, 256, 256, None, ctypes.byref(p), fake, fake, None, None) == 1
    # alignment (W at an odd address, ldw not a multiple of 8 for bf16)
    odd = ctypes.c_void_p(16 * 1024 + 2)
    assert lib.usk_build(odd, 1, 64, 256, 256, None, ctypes.byref(p), fake, fake, None, None) == 10
    assert lib.usk_build(fake, 1, 64, 256, 260, None, ctypes.byref(p), fake, fake, None, None) == 10
    # M == 0 is a no-op
    assert lib.usk_build(None, 1, 0, 256, 256, None, ctypes.byref(p), None, None, None, None) == 0
    sk = _native.UskSketchC(64, 256, 0, 16 * 1024, 16 * 1024)
    assert lib.usk_gemv(None, fake, 1, 1, fake, None, None) == 1
    assert lib.usk_gemv(ctypes.byref(sk), fake, 1, 16, fake, None, None) == 4
    assert lib.usk_gemv(ctypes.byref(sk), fake, 5, 1, fake, None, None) == 3
    assert lib.usk_gemv_ex(ctypes.byref(sk), fake, 1, 1, fake, 8, None, None) == 6
    assert lib.usk_gemv(ctypes.byref(sk), fake, 1, 0, fake, None, None) == 0
    assert lib.usk_gemm(ctypes.byref(sk), fake, 8, fake, None, 0, None, None) == 4
    assert lib.usk_gemm(ctypes.byref(sk), fake, 24, fake, None, 0, None, None) == 4
    assert lib.usk_gemm(ctypes.byref(sk), fake, 512, fake, None, 0, None, None) == 4
    assert lib.usk_gemm_ex(ctypes.byref(sk), fake, 16, fake, 2, None, None) == 6  # unknown flag bit
    assert lib.usk_gemm_ex(ctypes.byref(sk), fake, 24, fake, 1, None, None) == 4
    for version, depth in ((2, 3), (2, 0), (1, 2), (5, 1)):
        bad_sk = _native.UskSketchC(64, 256, 0, 16 * 1024, 16 * 1024, version, depth)
        assert lib.usk_gemv(ctypes.byref(bad_sk), fake, 1, 1, fake, None, None) == 6
        assert lib.usk_gemm(ctypes.byref(bad_sk), fake, 16, fake, None, 0, None, None) == 6
    unaligned = _native.UskSketchC(64, 256, 0, 16 * 1024 + 1, 16 * 1024)
    assert lib.usk_gemv(ctypes.byref(unaligned), fake, 1, 1, fake, None, None) == 10


def test_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        usk.usk_build(torch.zeros((64, 256), dtype=torch.bfloat16))


def test_plan_slots_matches_the_oracle_procedure(lib):
    """The library's allocation (C++) against the oracle's (Python), written
    separately from the same definition: identical slot counts."""
    import numpy as np
    import oracle
    g = np.random.default_rng(17)
    for trial in range(200):
        n = int(g.integers(1, 60))
        w = [int(v) * 16384 for v in g.integers(1, 300, size=n)]
        imp = [float(v) for v in g.lognormal(0, 2, size=n)]
        if trial % 7 == 0:
            imp = [float(int(v)) for v in g.integers(0, 3, size=n)]  # many ties
        budget = float(g.uniform(0.25, 1.0))
        assert usk.usk_plan_slots(w, imp, budget) == oracle.plan_slots(w, imp, budget)
    assert usk.usk_plan_slots([], [], 0.5) == []
    for bad in ((0.2,), (1.5,)):
        with pytest.raises(usk.UskError):
            usk.usk_plan_slots([1], [1.0], bad[0])
    with pytest.raises(usk.UskError):
        usk.usk_plan_slots([1], [-1.0], 0.5)
    with pytest.raises(usk.UskError):
        usk.usk_plan_slots([0], [1.0], 0.5)


def test_sizes_ex(lib):
    assert usk.usk_sizes_ex(4096, 4096) == (4096 * 4096 // 16, 128)
    assert usk.usk_sizes_ex(4096, 4096, 1, 2) == (4096 * 4096 // 32, 128)
    assert usk.usk_sizes_ex(4096, 4096, 1, 8) == (4096 * 4096 // 8, 128)
    assert usk.usk_sizes_ex(4096, 4096, 4, 0) == (4096 * 4096 // 16, 128)
    assert usk.usk_sizes_ex(4096, 4096, 2, 4) == (4096 * 4096 // 16, 128)
    with pytest.raises(usk.UskError):
        usk.usk_sizes_ex(4096, 4096, 2, 8)
    with pytest.raises(usk.UskError):
        usk.usk_sizes_ex(4096, 4096, 1, 3)


def test_struct_layouts_match_the_header(lib, tmp_path):
    """sizeof and field offsets of the C structs (gcc on include/usk.h) equal
    the binding's ctypes mirrors."""
    import subprocess
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "usk.h"\n'
        'int main(void) {\n'
        '  printf("%zu %zu %zu\\n", sizeof(usk_params), offsetof(usk_params, slots), offsetof(usk_params, rates));\n'
        '  printf("%zu %zu %zu\\n", sizeof(usk_sketch), offsetof(usk_sketch, pad), offsetof(usk_sketch, rates));\n'
        '  printf("%zu %zu %zu\\n", sizeof(usk_rate_map), offsetof(usk_rate_map, count),'
        ' offsetof(usk_rate_map, code_bytes));\n'
        '  return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [list(map(int, ln.split())) for ln in subprocess.check_output([str(exe)]).decode().split("\n") if ln]
    P, S, R = _native.UskParams, _native.UskSketchC, _native.UskRateMapC
    assert got[0] == [ctypes.sizeof(P), P.slots.offset, P.rates.offset]
    assert got[1] == [ctypes.sizeof(S), S.pad.offset, S.rates.offset]
    assert got[2] == [ctypes.sizeof(R), R.count.offset, R.code_bytes.offset]


def test_rate_map_plan_matches_the_oracle_offsets(lib):
    import numpy as np
    import oracle
    g = np.random.default_rng(5)
    for _ in range(50):
        n = int(g.integers(1, 40))
        K = 256 * int(g.integers(1, 20))
        slots = [int(v) for v in g.choice([2, 4, 8], size=n)]
        off, order, count, total = usk.usk_rate_map_plan(64 * n, K, slots)
        ooff, ototal = oracle.vr_offsets(64 * n, K, slots)
        assert off == ooff.tolist() and total == ototal
        assert count == (slots.count(2), slots.count(4), slots.count(8))
        # grouped by slot count, increasing within a group, a permutation
        assert sorted(order) == list(range(n))
        keys = [(slots[rb], rb) for rb in order]
        assert keys == sorted(keys)
    assert usk.usk_rate_map_plan(0, 256, []) == ([], [], (0, 0, 0), 0)
    with pytest.raises(usk.UskError):
        usk.usk_rate_map_plan(128, 256, [2, 6])
    with pytest.raises(usk.UskError):
        usk.usk_rate_map_plan(100, 256, [2])


def test_rate_map_argument_errors(lib):
    fake = ctypes.c_void_p(16 * 1024)
    good = _native.UskRateMapC(16 * 1024, 16 * 1024)
    good.count[0], good.count[1], good.count[2] = 1, 0, 1
    good.code_bytes = 256 * (2 + 8)

    def params(rm, version=1, slots=0):
        p = _native.UskParams(version, 0, 0, 1, slots)
        p.rates = ctypes.pointer(rm)
        return p

    def sketch(rm, version=1, slots=0):
        s = _native.UskSketchC(128, 256, 0, 16 * 1024, 16 * 1024, version, 1, slots, 0)
        s.rates = ctypes.pointer(rm)
        return s

    bad_counts = _native.UskRateMapC(16 * 1024, 16 * 1024)
    bad_counts.count[0], bad_counts.code_bytes = 1, 512  # 1 of 2 row blocks
    bad_bytes = _native.UskRateMapC(16 * 1024, 16 * 1024)
    bad_bytes.count[0], bad_bytes.count[2], bad_bytes.code_bytes = 1, 1, 4096
    no_tables = _native.UskRateMapC(None, None)
    no_tables.count[1], no_tables.code_bytes = 2, 2048
    odd = _native.UskRateMapC(16 * 1024 + 4, 16 * 1024)
    odd.count[1], odd.code_bytes = 2, 2048
    for rm, want in ((bad_counts, 6), (bad_bytes, 6), (no_tables, 1), (odd, 10)):
        assert lib.usk_build(fake, 1, 128, 256, 256, None, ctypes.byref(params(rm)), fake, fake, None, None) == want
        assert lib.usk_gemv(ctypes.byref(sketch(rm)), fake, 1, 1, fake, None, None) == want
        assert lib.usk_gemm(ctypes.byref(sketch(rm)), fake, 16, fake, None, 0, None, None) == want
    # a rate map only with format 1 and the default slot count
    for version, slots in ((2, 0), (3, 0), (4, 0), (1, 8)):
        p = params(good, version, slots)
        assert lib.usk_build(fake, 1, 128, 256, 256, None, ctypes.byref(p), fake, fake, None, None) == 6
        assert lib.usk_gemv(ctypes.byref(sketch(good, version, slots)), fake, 1, 1, fake, None, None) == 6


def test_rate_map_binding_checks(lib):
    """The binding refuses rate tables that the kernels could not read."""
    import torch
    off, order, count, total = usk.usk_rate_map_plan(128, 256, [2, 8])
    cpu = usk.RateMap([2, 8], torch.tensor(off, dtype=torch.int64), torch.tensor(order, dtype=torch.int32),
                      count, total)
    with pytest.raises(ValueError):
        cpu.as_c()  # host tensors
    wrong = usk.RateMap([2, 8], torch.tensor(off, dtype=torch.int32), torch.tensor(order, dtype=torch.int32),
                        count, total)
    with pytest.raises(ValueError):
        wrong.as_c()
    short = usk.RateMap([2, 8], torch.tensor(off[:1], dtype=torch.int64), torch.tensor(order, dtype=torch.int32),
                        count, total)
    with pytest.raises(ValueError):
        short.as_c()
    empty = usk.RateMap([], torch.zeros(0, dtype=torch.int64), torch.zeros(0, dtype=torch.int32), (0, 0, 0), 0)
    c = empty.as_c()
    assert c.code_bytes == 0 and list(c.count) == [0, 0, 0]
