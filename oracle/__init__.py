"""CPU oracle of the UltraSketchLLM sketch -- TEST INFRASTRUCTURE ONLY.

This package wraps ``usk_oracle.c`` (plain sequential C, IEEE fp32/fp64, no
fast-math) with ctypes and numpy.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the library under
``sub_bit_weight_usk_b200/`` never does, and the two share no code.

What it computes is written out in ``usk_oracle.c`` with its sources:
"UltraSketchLLM: Sub-1-Bit LLM Compression via Sketch and Hardware-Friendly
Operators" (gist.science/es/paper/2506.17255), Resumen Tecnico, Metodologia §1
(AbsMaxMin sketch) and §4 (decompression as W_hat = S . P^T), plus the frozen
format readings listed there: format 1 (one hash row, largest key kept) and
format 2 (the multi-row AbsMaxMin sketch: smallest magnitude kept per bucket,
largest magnitude over the hash rows on decode; the ``*_amm`` functions) and
format 3 (the column-shared projection W_hat = S . P^T; the ``*_cs`` functions)
and format 4 (format 1 with 4-bit codes and 8 weights per bucket; ``*_q4``).

Parity pins (tests/test_oracle_*.py): SplitMix64 published outputs, binary16
conversion against numpy's, round-half-even against numpy.rint, an independent
pure-Python brute-force bucket enumeration, closed-form special cases and
invariants, and numpy float64 matmul for the products.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "usk_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# status values (same meanings as the library's usk_status)
OK = 0
ERR_NULL = 1
ERR_SHAPE = 2
ERR_DTYPE = 3
ERR_NONFINITE = 8
ERR_IMPORTANCE = 11
ERR_SCALE_OVERFLOW = 12

F32 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compile usk_oracle.c into liboracle.so next to it (gcc, IEEE-strict)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, u64, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
        lib.orc_build.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, u64, vp, vp, vp, vp]
        lib.orc_build.restype = ctypes.c_int
        lib.orc_build_rows.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, u64, i64, vp, vp, vp, vp]
        lib.orc_build_rows.restype = ctypes.c_int
        lib.orc_decode.argtypes = [vp, vp, i64, i64, u64, vp]
        lib.orc_decode.restype = ctypes.c_int
        lib.orc_gemv_f64.argtypes = [vp, vp, i64, i64, u64, vp, ctypes.c_int, i64, vp, i64, vp]
        lib.orc_gemv_f64.restype = ctypes.c_int
        lib.orc_bucket_index.argtypes = [i64, u64, i64, i64]
        lib.orc_bucket_index.restype = i64
        lib.orc_splitmix64.argtypes = [u64, u64]
        lib.orc_splitmix64.restype = u64
        lib.orc_tile_hash_params.argtypes = [u64, u64, vp, vp]
        lib.orc_tile_hash_params.restype = None
        lib.orc_f32_to_f16.argtypes = [ctypes.c_float]
        lib.orc_f32_to_f16.restype = ctypes.c_uint16
        lib.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.orc_f16_to_f32.restype = ctypes.c_float
        lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_f32.restype = ctypes.c_float
        lib.orc_storage_bytes.argtypes = [i64, i64, vp, vp]
        lib.orc_storage_bytes.restype = None
        lib.orc_amm_bucket_index.argtypes = [i64, u64, ctypes.c_int, ctypes.c_int, i64, i64]
        lib.orc_amm_bucket_index.restype = i64
        lib.orc_amm_build_rows.argtypes = [vp, ctypes.c_int, i64, i64, i64, u64, ctypes.c_int, i64, vp, vp,
                                           vp, vp]
        lib.orc_amm_build_rows.restype = ctypes.c_int
        lib.orc_amm_decode.argtypes = [vp, vp, i64, i64, u64, ctypes.c_int, vp]
        lib.orc_amm_decode.restype = ctypes.c_int
        lib.orc_amm_gemv_f64.argtypes = [vp, vp, i64, i64, u64, ctypes.c_int, vp, ctypes.c_int, i64, vp, i64,
                                         vp]
        lib.orc_amm_gemv_f64.restype = ctypes.c_int
        lib.orc_cs_sigma.argtypes = [u64, i64, ctypes.c_int]
        lib.orc_cs_sigma.restype = ctypes.c_int
        lib.orc_cs_bucket.argtypes = [i64, u64, i64]
        lib.orc_cs_bucket.restype = i64
        lib.orc_cs_build.argtypes = [vp, ctypes.c_int, i64, i64, i64, u64, vp, vp, vp, vp]
        lib.orc_cs_build.restype = ctypes.c_int
        lib.orc_cs_decode.argtypes = [vp, vp, i64, i64, u64, vp]
        lib.orc_cs_decode.restype = ctypes.c_int
        lib.orc_cs_gemv_f64.argtypes = [vp, vp, i64, i64, u64, vp, ctypes.c_int, i64, vp, i64, vp]
        lib.orc_cs_gemv_f64.restype = ctypes.c_int
        lib.orc_q4_bucket.argtypes = [i64, u64, i64, i64]
        lib.orc_q4_bucket.restype = i64
        lib.orc_q4_build_rows.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, u64, i64, vp, vp, vp, vp]
        lib.orc_q4_build_rows.restype = ctypes.c_int
        lib.orc_q4_decode.argtypes = [vp, vp, i64, i64, u64, vp]
        lib.orc_q4_decode.restype = ctypes.c_int
        lib.orc_q4_gemv_f64.argtypes = [vp, vp, i64, i64, u64, vp, ctypes.c_int, i64, vp, i64, vp]
        lib.orc_q4_gemv_f64.restype = ctypes.c_int
        lib.orc_rate_bucket.argtypes = [i64, u64, ctypes.c_int, i64, i64]
        lib.orc_rate_bucket.restype = i64
        lib.orc_rate_build.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, u64, ctypes.c_int, vp, vp]
        lib.orc_rate_build.restype = ctypes.c_int
        lib.orc_rate_gemv_f64.argtypes = [vp, vp, i64, i64, u64, ctypes.c_int, vp, ctypes.c_int, i64, vp, i64, vp]
        lib.orc_rate_gemv_f64.restype = ctypes.c_int
        lib.orc_vr_offsets.argtypes = [i64, i64, vp, vp]
        lib.orc_vr_offsets.restype = i64
        lib.orc_vr_bucket.argtypes = [i64, u64, vp, i64, i64]
        lib.orc_vr_bucket.restype = i64
        lib.orc_vr_build.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, u64, vp, vp, vp]
        lib.orc_vr_build.restype = ctypes.c_int
        lib.orc_vr_gemv_f64.argtypes = [vp, vp, i64, i64, u64, vp, vp, ctypes.c_int, i64, vp, i64, vp]
        lib.orc_vr_gemv_f64.restype = ctypes.c_int
        lib.orc_f32_to_f16_array.argtypes = [vp, vp, i64]
        lib.orc_f32_to_f16_array.restype = None
        lib.orc_f16_to_f32_array.argtypes = [vp, vp, i64]
        lib.orc_f16_to_f32_array.restype = None
        lib.orc_threads.argtypes = [ctypes.c_int]
        lib.orc_threads.restype = ctypes.c_int
        lib.orc_build_mt.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, u64, vp, vp, ctypes.c_int]
        lib.orc_build_mt.restype = ctypes.c_int
        lib.orc_gemv_f64_mt.argtypes = [vp, vp, i64, i64, u64, vp, ctypes.c_int, i64, vp, ctypes.c_int]
        lib.orc_gemv_f64_mt.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _weights(W):
    """(array, dtype code): float32 arrays are fp32, uint16 arrays are bf16 bits."""
    W = np.ascontiguousarray(W)
    if W.dtype == np.float32:
        return W, F32
    if W.dtype == np.uint16:
        return W, BF16
    raise TypeError("weights must be float32 or uint16 (bf16 bit patterns)")


def build_sketch(W, importance=None, seed=0, want_winners=False, row_block0=0):
    """Sketch of W [M, K].  Returns dict(status, codes, scales[, winner, value]).

    row_block0 > 0: W holds the rows starting at row block row_block0 of a
    larger matrix with the same K (the hash uses the true row blocks)."""
    W, dt = _weights(W)
    M, K = W.shape
    imp = None if importance is None else np.ascontiguousarray(importance, dtype=np.float32)
    nb = M * K // 16 if (M % 64 == 0 and K % 256 == 0 and M >= 0 and K >= 0) else 0
    codes = np.zeros(max(nb, 1), dtype=np.int8)
    scales = np.zeros(max(M // 64, 1), dtype=np.uint16)
    winner = np.full(max(nb, 1), -2, dtype=np.int64) if want_winners else None
    value = np.zeros(max(nb, 1), dtype=np.float32) if want_winners else None
    st = _load().orc_build_rows(_ptr(W), dt, M, K, K, _ptr(imp), seed, row_block0, _ptr(codes),
                                _ptr(scales), _ptr(winner), _ptr(value))
    out = {"status": st, "codes": codes[:nb], "scales": scales[: M // 64]}
    if want_winners:
        out["winner"] = winner[:nb]
        out["value"] = value[:nb]
    return out


def build_sketch_amm(W, seed=0, depth=2, want_winners=False, row_block0=0):
    """Depth-`depth` AbsMaxMin sketch of W [M, K] (format 2: min-|w| store,
    max-magnitude decode over the hash rows).  Returns dict as build_sketch."""
    W, dt = _weights(W)
    M, K = W.shape
    nb = M * K // 16 if (M % 64 == 0 and K % 256 == 0 and M >= 0 and K >= 0) else 0
    codes = np.zeros(max(nb, 1), dtype=np.int8)
    scales = np.zeros(max(M // 64, 1), dtype=np.uint16)
    winner = np.full(max(nb, 1), -2, dtype=np.int64) if want_winners else None
    value = np.zeros(max(nb, 1), dtype=np.float32) if want_winners else None
    st = _load().orc_amm_build_rows(_ptr(W), dt, M, K, K, seed, depth, row_block0, _ptr(codes),
                                    _ptr(scales), _ptr(winner), _ptr(value))
    out = {"status": st, "codes": codes[:nb], "scales": scales[: M // 64]}
    if want_winners:
        out["winner"] = winner[:nb]
        out["value"] = value[:nb]
    return out


def decode_amm(codes, scales, M, K, seed=0, depth=2):
    """W_hat [M, K] float32 of a format-2 sketch."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    out = np.zeros((M, K), dtype=np.float32)
    st = _load().orc_amm_decode(_ptr(codes), _ptr(scales), M, K, seed, depth, _ptr(out))
    if st:
        raise ValueError("orc_amm_decode status %d" % st)
    return out


def gemv_amm_f64(codes, scales, M, K, x, seed=0, depth=2, rows=None):
    """y = W_hat x^T in float64 for a format-2 sketch (arguments as gemv_f64)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    xdt = F32 if x.dtype == np.float32 else BF16 if x.dtype == np.uint16 else None
    if xdt is None:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    batch = x.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else len(r)
    y = np.zeros((batch, nr), dtype=np.float64)
    st = _load().orc_amm_gemv_f64(_ptr(codes), _ptr(scales), M, K, seed, depth, _ptr(x), xdt, batch,
                                  _ptr(r), 0 if r is None else len(r), _ptr(y))
    if st:
        raise ValueError("orc_amm_gemv_f64 status %d" % st)
    return y


def amm_bucket_index(K, seed, depth, rho, i, j):
    """Global code index of weight (i, j) in hash row rho of a format-2 sketch."""
    return int(_load().orc_amm_bucket_index(K, seed, depth, rho, i, j))


def build_sketch_cs(W, seed=0, want_winners=False):
    """Column-shared projection sketch of W [M, K] (format 3: W_hat = S . P^T with
    a one-hot P shared by all rows; S keeps the smallest |w| per row and
    bucket).  Returns dict as build_sketch; codes are row-major [M, K/16]."""
    W, dt = _weights(W)
    M, K = W.shape
    nb = M * K // 16 if (M % 64 == 0 and K % 256 == 0 and M >= 0 and K >= 0) else 0
    codes = np.zeros(max(nb, 1), dtype=np.int8)
    scales = np.zeros(max(M // 64, 1), dtype=np.uint16)
    winner = np.full(max(nb, 1), -2, dtype=np.int64) if want_winners else None
    value = np.zeros(max(nb, 1), dtype=np.float32) if want_winners else None
    st = _load().orc_cs_build(_ptr(W), dt, M, K, K, seed, _ptr(codes), _ptr(scales), _ptr(winner), _ptr(value))
    out = {"status": st, "codes": codes[:nb], "scales": scales[: M // 64]}
    if want_winners:
        out["winner"] = winner[:nb]
        out["value"] = value[:nb]
    return out


def decode_cs(codes, scales, M, K, seed=0):
    """W_hat [M, K] float32 of a format-3 sketch."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    out = np.zeros((M, K), dtype=np.float32)
    st = _load().orc_cs_decode(_ptr(codes), _ptr(scales), M, K, seed, _ptr(out))
    if st:
        raise ValueError("orc_cs_decode status %d" % st)
    return out


def gemv_cs_f64(codes, scales, M, K, x, seed=0, rows=None):
    """y = W_hat x^T in float64 for a format-3 sketch (arguments as gemv_f64)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    xdt = F32 if x.dtype == np.float32 else BF16 if x.dtype == np.uint16 else None
    if xdt is None:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    batch = x.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else len(r)
    y = np.zeros((batch, nr), dtype=np.float64)
    st = _load().orc_cs_gemv_f64(_ptr(codes), _ptr(scales), M, K, seed, _ptr(x), xdt, batch,
                                 _ptr(r), 0 if r is None else len(r), _ptr(y))
    if st:
        raise ValueError("orc_cs_gemv_f64 status %d" % st)
    return y


def cs_sigma(seed, tc, u):
    """sigma_tc(u): position u of tile column tc's column list (format 3)."""
    return int(_load().orc_cs_sigma(seed & (2**64 - 1), tc, u))


def cs_bucket(K, seed, j):
    """Global bucket of column j in a format-3 sketch."""
    return int(_load().orc_cs_bucket(K, seed, j))


def build_sketch_q4(W, importance=None, seed=0, want_winners=False, row_block0=0):
    """Format-4 sketch of W [M, K]: the format-1 rule with 8 weights per bucket
    and 4-bit codes (two per byte).  Returns dict as build_sketch; winner and
    value have M*K/8 entries (buckets)."""
    W, dt = _weights(W)
    M, K = W.shape
    ok = M % 64 == 0 and K % 256 == 0 and M >= 0 and K >= 0
    nbytes = M * K // 16 if ok else 0
    nb = M * K // 8 if ok else 0
    imp = None if importance is None else np.ascontiguousarray(importance, dtype=np.float32)
    codes = np.zeros(max(nbytes, 1), dtype=np.int8)
    scales = np.zeros(max(M // 64, 1), dtype=np.uint16)
    winner = np.full(max(nb, 1), -2, dtype=np.int64) if want_winners else None
    value = np.zeros(max(nb, 1), dtype=np.float32) if want_winners else None
    st = _load().orc_q4_build_rows(_ptr(W), dt, M, K, K, _ptr(imp), seed, row_block0, _ptr(codes),
                                   _ptr(scales), _ptr(winner), _ptr(value))
    out = {"status": st, "codes": codes[:nbytes], "scales": scales[: M // 64]}
    if want_winners:
        out["winner"] = winner[:nb]
        out["value"] = value[:nb]
    return out


def decode_q4(codes, scales, M, K, seed=0):
    """W_hat [M, K] float32 of a format-4 sketch."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    out = np.zeros((M, K), dtype=np.float32)
    st = _load().orc_q4_decode(_ptr(codes), _ptr(scales), M, K, seed, _ptr(out))
    if st:
        raise ValueError("orc_q4_decode status %d" % st)
    return out


def gemv_q4_f64(codes, scales, M, K, x, seed=0, rows=None):
    """y = W_hat x^T in float64 for a format-4 sketch (arguments as gemv_f64)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    xdt = F32 if x.dtype == np.float32 else BF16 if x.dtype == np.uint16 else None
    if xdt is None:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    batch = x.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else len(r)
    y = np.zeros((batch, nr), dtype=np.float64)
    st = _load().orc_q4_gemv_f64(_ptr(codes), _ptr(scales), M, K, seed, _ptr(x), xdt, batch,
                                 _ptr(r), 0 if r is None else len(r), _ptr(y))
    if st:
        raise ValueError("orc_q4_gemv_f64 status %d" % st)
    return y


def q4_bucket(K, seed, i, j):
    """Bucket of weight (i, j) within its 64-row block (format 4): 2048 tc + b."""
    return int(_load().orc_q4_bucket(K, seed, i, j))


def build_sketch_rate(W, importance=None, seed=0, slots=4):
    """Format-1 sketch with `slots` (2, 4 or 8) hash slots per class: 32, 16 or 8
    weights per bucket, 0.25, 0.5 or 1 bit/weight.  Returns dict(status, codes,
    scales); codes [M*K*slots/64]."""
    W, dt = _weights(W)
    M, K = W.shape
    ok = M % 64 == 0 and K % 256 == 0 and M >= 0 and K >= 0 and slots in (2, 4, 8)
    nb = M * K * slots // 64 if ok else 0
    imp = None if importance is None else np.ascontiguousarray(importance, dtype=np.float32)
    codes = np.zeros(max(nb, 1), dtype=np.int8)
    scales = np.zeros(max(M // 64, 1), dtype=np.uint16)
    st = _load().orc_rate_build(_ptr(W), dt, M, K, K, _ptr(imp), seed, slots, _ptr(codes), _ptr(scales))
    return {"status": st, "codes": codes[:nb], "scales": scales[: M // 64]}


def gemv_rate_f64(codes, scales, M, K, x, seed=0, slots=4, rows=None):
    """y = W_hat x^T in float64 for a `slots`-slot format-1 sketch."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    xdt = F32 if x.dtype == np.float32 else BF16 if x.dtype == np.uint16 else None
    if xdt is None:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    batch = x.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else len(r)
    y = np.zeros((batch, nr), dtype=np.float64)
    st = _load().orc_rate_gemv_f64(_ptr(codes), _ptr(scales), M, K, seed, slots, _ptr(x), xdt, batch,
                                   _ptr(r), 0 if r is None else len(r), _ptr(y))
    if st:
        raise ValueError("orc_rate_gemv_f64 status %d" % st)
    return y


def rate_bucket(K, seed, slots, i, j):
    """Global code index of weight (i, j) in a `slots`-slot format-1 sketch."""
    return int(_load().orc_rate_bucket(K, seed, slots, i, j))


def _slots_u32(slots):
    return np.ascontiguousarray(np.asarray(slots, dtype=np.uint32))


def vr_offsets(M, K, slots):
    """Per-row-block rates: (offsets, total code bytes); row block rb's codes
    start at K * (slots[0] + ... + slots[rb - 1])."""
    sl = _slots_u32(slots)
    off = np.zeros(max(M // 64, 1), dtype=np.int64)
    total = int(_load().orc_vr_offsets(M, K, _ptr(sl), _ptr(off)))
    if total < 0:
        raise ValueError("slot counts must be 2, 4 or 8")
    return off[: M // 64], total


def build_sketch_vr(W, importance=None, seed=0, slots=None):
    """Format-1 sketch whose 64-row block rb has slots[rb] (2, 4 or 8) hash
    slots per class, codes of the blocks back to back in matrix order.
    Returns dict(status, codes, scales)."""
    W, dt = _weights(W)
    M, K = W.shape
    sl = _slots_u32(slots)
    if sl.shape != (M // 64,):
        raise ValueError("one slot count per 64-row block")
    ok = M % 64 == 0 and K % 256 == 0 and all(v in (2, 4, 8) for v in sl.tolist())
    nb = int(K * int(sl.astype(np.int64).sum())) if ok else 0
    imp = None if importance is None else np.ascontiguousarray(importance, dtype=np.float32)
    codes = np.zeros(max(nb, 1), dtype=np.int8)
    scales = np.zeros(max(M // 64, 1), dtype=np.uint16)
    st = _load().orc_vr_build(_ptr(W), dt, M, K, K, _ptr(imp), seed, _ptr(sl), _ptr(codes), _ptr(scales))
    return {"status": st, "codes": codes[:nb], "scales": scales[: M // 64]}


def gemv_vr_f64(codes, scales, M, K, x, seed=0, slots=None, rows=None):
    """y = W_hat x^T in float64 for a per-row-block-rate sketch."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    sl = _slots_u32(slots)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    xdt = F32 if x.dtype == np.float32 else BF16 if x.dtype == np.uint16 else None
    if xdt is None:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    batch = x.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else len(r)
    y = np.zeros((batch, nr), dtype=np.float64)
    st = _load().orc_vr_gemv_f64(_ptr(codes), _ptr(scales), M, K, seed, _ptr(sl), _ptr(x), xdt, batch,
                                 _ptr(r), 0 if r is None else len(r), _ptr(y))
    if st:
        raise ValueError("orc_vr_gemv_f64 status %d" % st)
    return y


def vr_bucket(K, seed, slots, i, j):
    """Global code index of weight (i, j) in a per-row-block-rate sketch."""
    sl = _slots_u32(slots)
    return int(_load().orc_vr_bucket(K, seed, _ptr(sl), i, j))


# bits per weight of each slot count (8-bit codes)
SLOT_BITS = {2: 0.25, 4: 0.5, 8: 1.0}


def plan_slots(weights, importance, budget_bits):
    """Importance-aware space allocation (Metodologia §2: units of higher
    importance get more buckets), written as a plain greedy procedure:

    every unit starts at 2 slots; the upgrades 2 -> 4 and 4 -> 8 of every unit
    are visited in decreasing order of importance gained per bit -- with the
    distortion of a unit taken as importance x weights / slots, upgrade s -> 2s
    gains importance x weights / (2 s) for (bits(2s) - bits(s)) x weights bits,
    i.e. a ratio of importance (2 -> 4) or importance / 4 (4 -> 8) -- ties in
    the order go to the lower level, then to the lower index; an upgrade is
    taken when the unit is at its starting level and the total stays within
    budget_bits x total weights.  Returns a list of slot counts."""
    n = len(weights)
    w = [int(v) for v in weights]
    imp = [float(v) for v in importance]
    total = sum(w)
    cap = budget_bits * total
    slots = [2] * n
    used = sum(0.25 * wi for wi in w)
    cands = []
    for i in range(n):
        cands.append((-imp[i], 0, i))        # 2 -> 4, ratio imp
        cands.append((-imp[i] / 4.0, 1, i))  # 4 -> 8, ratio imp / 4
    cands.sort()
    for _, level, i in cands:
        frm = 2 if level == 0 else 4
        if slots[i] != frm:
            continue
        cost = (SLOT_BITS[2 * frm] - SLOT_BITS[frm]) * w[i]
        if used + cost <= cap:
            slots[i] = 2 * frm
            used += cost
    return slots


def decode(codes, scales, M, K, seed=0):
    """W_hat [M, K] float32 rebuilt from the sketch."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    out = np.zeros((M, K), dtype=np.float32)
    st = _load().orc_decode(_ptr(codes), _ptr(scales), M, K, seed, _ptr(out))
    if st:
        raise ValueError("orc_decode status %d" % st)
    return out


def gemv_f64(codes, scales, M, K, x, seed=0, rows=None):
    """y [batch, M] (or [batch, len(rows)]) = W_hat x^T in float64.

    x is [batch, K] float32 (fp32) or uint16 (bf16 bit patterns)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    xdt = F32 if x.dtype == np.float32 else BF16 if x.dtype == np.uint16 else None
    if xdt is None:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    batch = x.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else len(r)
    y = np.zeros((batch, nr), dtype=np.float64)
    st = _load().orc_gemv_f64(_ptr(codes), _ptr(scales), M, K, seed, _ptr(x), xdt, batch,
                              _ptr(r), 0 if r is None else len(r), _ptr(y))
    if st:
        raise ValueError("orc_gemv_f64 status %d" % st)
    return y


def threads(n: int = 0) -> int:
    """Host threads the all-core functions use for `n` (0 = all available)."""
    return int(_load().orc_threads(int(n)))


def build_sketch_mt(W, importance=None, seed=0, threads=0):
    """build_sketch (format 1) with the row blocks spread over host threads:
    the same sequential code per row block, so the same codes and scales.
    Returns dict(status, codes, scales)."""
    W, dt = _weights(W)
    M, K = W.shape
    imp = None if importance is None else np.ascontiguousarray(importance, dtype=np.float32)
    nb = M * K // 16 if (M % 64 == 0 and K % 256 == 0 and M >= 0 and K >= 0) else 0
    codes = np.empty(max(nb, 1), dtype=np.int8)
    scales = np.zeros(max(M // 64, 1), dtype=np.uint16)
    st = _load().orc_build_mt(_ptr(W), dt, M, K, K, _ptr(imp), seed, _ptr(codes), _ptr(scales), int(threads))
    return {"status": st, "codes": codes[:nb], "scales": scales[: M // 64]}


def gemv_f64_mt(codes, scales, M, K, x, seed=0, threads=0):
    """gemv_f64 over all rows with runs of 64 rows spread over host threads
    (the same float64 sums row by row)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    xdt = F32 if x.dtype == np.float32 else BF16 if x.dtype == np.uint16 else None
    if xdt is None:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    batch = x.shape[0]
    y = np.zeros((batch, M), dtype=np.float64)
    st = _load().orc_gemv_f64_mt(_ptr(codes), _ptr(scales), M, K, seed, _ptr(x), xdt, batch, _ptr(y),
                                 int(threads))
    if st:
        raise ValueError("orc_gemv_f64_mt status %d" % st)
    return y


def bucket_index(K, seed, i, j):
    """Global code index of weight (i, j)."""
    return int(_load().orc_bucket_index(K, seed, i, j))


def splitmix64(seed, n):
    """Output n (1-based) of SplitMix64 seeded with `seed`."""
    return int(_load().orc_splitmix64(seed & (2**64 - 1), n))


def tile_hash_params(seed, tile_id):
    a = ctypes.c_uint32()
    c = ctypes.c_uint32()
    _load().orc_tile_hash_params(seed, tile_id, ctypes.byref(a), ctypes.byref(c))
    return a.value, c.value


def f32_to_f16(x):
    return int(_load().orc_f32_to_f16(float(np.float32(x))))


def f16_to_f32(h):
    return float(_load().orc_f16_to_f32(int(h)))


def f32_to_f16_array(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, dtype=np.uint16)
    _load().orc_f32_to_f16_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_to_f32_array(h):
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.zeros(h.shape, dtype=np.float32)
    _load().orc_f16_to_f32_array(_ptr(h), _ptr(out), h.size)
    return out


def bf16_to_f32(h):
    return float(_load().orc_bf16_to_f32(int(h)))


def storage_bytes(M, K):
    c = ctypes.c_int64()
    s = ctypes.c_int64()
    _load().orc_storage_bytes(M, K, ctypes.byref(c), ctypes.byref(s))
    return c.value, s.value
