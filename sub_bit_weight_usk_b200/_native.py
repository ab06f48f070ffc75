"""ctypes binding of libusk.so (include/usk.h): argument marshalling only.

Every step of the sketch build and of the sketch-decode products runs in the
library's CUDA kernels; this module only turns torch tensors into device
pointers, picks the current CUDA stream and raises on a non-OK status.  There
is no CPU fallback: if the library or a GPU is missing, calls fail loudly.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libusk.so")

USK_OK = 0
USK_F32 = 0
USK_BF16 = 1
FORMAT_MAXKEY = 1      # format 1: one hash row, the largest key kept per bucket
FORMAT_ABSMAXMIN = 2   # format 2: multi-row AbsMaxMin (smallest |w| kept, largest over rows decoded)
FORMAT_COLSHARED = 3   # format 3: column-shared projection, W_hat = S . P^T, product as S (P^T x)
FORMAT_Q4 = 4          # format 4: format 1 with 4-bit codes, 8 weights per bucket
FORMAT_VERSION = 4     # highest format the library builds and reads
GEMV_MAX_BATCH = 15
GEMM_MIN_BATCH = 16
GEMM_MAX_BATCH = 256

FLAG_NONFINITE_W = 1 << 0
FLAG_BAD_IMPORTANCE = 1 << 1
FLAG_SCALE_OVERFLOW = 1 << 2
FLAG_TIMEOUT = 1 << 3
FLAG_RATE_MAP = 1 << 4

STATUS_NAMES = {
    0: "USK_OK", 1: "USK_ERR_NULL", 2: "USK_ERR_SHAPE", 3: "USK_ERR_DTYPE", 4: "USK_ERR_BATCH",
    5: "USK_ERR_WORKSPACE", 6: "USK_ERR_PARAMS", 7: "USK_ERR_CUDA", 8: "USK_ERR_NONFINITE",
    9: "USK_ERR_TIMEOUT", 10: "USK_ERR_ALIGN", 11: "USK_ERR_IMPORTANCE", 12: "USK_ERR_SCALE_OVERFLOW",
}


class UskError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (what, STATUS_NAMES.get(status, status), usk_status_str(status)))


class UskRateMapC(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_void_p), ("order", ctypes.c_void_p), ("count", ctypes.c_int64 * 3),
                ("code_bytes", ctypes.c_int64)]


class UskParams(ctypes.Structure):
    _fields_ = [("version", ctypes.c_uint32), ("flags", ctypes.c_uint32), ("seed", ctypes.c_uint64),
                ("depth", ctypes.c_uint32), ("slots", ctypes.c_uint32), ("rates", ctypes.POINTER(UskRateMapC))]


class UskSketchC(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("K", ctypes.c_int64), ("seed", ctypes.c_uint64),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("version", ctypes.c_uint32), ("depth", ctypes.c_uint32), ("slots", ctypes.c_uint32),
                ("pad", ctypes.c_uint32), ("rates", ctypes.POINTER(UskRateMapC))]


_lib = None

EXPORTED = ["usk_sizes", "usk_sizes_ex", "usk_plan_slots", "usk_rate_map_plan", "usk_build", "usk_gemv", "usk_gemv_ex",
            "usk_gemv_multi", "usk_gemv_multi_ws_bytes", "usk_gemv_multi_static", "usk_gemm", "usk_gemm_ex",
            "usk_status_str",
            "usk_format_version", "usk_debug_set_geometry", "usk_debug_set_gemv_path", "usk_debug_set_gemv_rows",
            "usk_debug_set_gemm_splits", "usk_debug_set_gemm_issuers", "usk_debug_inject_timeout"]
GEMV_PDL = 1
GEMM_PDL = 1


def load_library(path: str = LIB_PATH):
    """Load libusk.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError("libusk.so not found at %s: build it with __graft_entry__.build() "
                      "or python -m sub_bit_weight_usk_b200._build" % path)
    lib = ctypes.CDLL(path)
    vp, i64, u32p = ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_uint32)
    lib.usk_sizes.argtypes = [i64, i64, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
    lib.usk_sizes.restype = ctypes.c_int
    lib.usk_sizes_ex.argtypes = [i64, i64, ctypes.c_uint32, ctypes.c_uint32, ctypes.POINTER(ctypes.c_size_t),
                                 ctypes.POINTER(ctypes.c_size_t)]
    lib.usk_sizes_ex.restype = ctypes.c_int
    lib.usk_plan_slots.argtypes = [i64, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double),
                                   ctypes.c_double, ctypes.POINTER(ctypes.c_uint32)]
    lib.usk_plan_slots.restype = ctypes.c_int
    lib.usk_rate_map_plan.argtypes = [i64, i64, u32p, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)]
    lib.usk_rate_map_plan.restype = ctypes.c_int
    lib.usk_build.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, ctypes.POINTER(UskParams), vp, vp, vp, vp]
    lib.usk_build.restype = ctypes.c_int
    lib.usk_gemv.argtypes = [ctypes.POINTER(UskSketchC), vp, ctypes.c_int, i64, vp, vp, vp]
    lib.usk_gemv.restype = ctypes.c_int
    lib.usk_gemv_ex.argtypes = [ctypes.POINTER(UskSketchC), vp, ctypes.c_int, i64, vp, ctypes.c_uint32, vp, vp]
    lib.usk_gemv_ex.restype = ctypes.c_int
    lib.usk_gemv_multi_ws_bytes.argtypes = [i64, ctypes.POINTER(UskSketchC), i64, ctypes.POINTER(ctypes.c_size_t)]
    lib.usk_gemv_multi_ws_bytes.restype = ctypes.c_int
    lib.usk_gemv_multi.argtypes = [i64, ctypes.POINTER(UskSketchC), ctypes.POINTER(vp), ctypes.c_int, i64,
                                   ctypes.POINTER(vp), vp, ctypes.c_size_t, ctypes.c_uint32, vp, vp]
    lib.usk_gemv_multi.restype = ctypes.c_int
    lib.usk_gemv_multi_static.argtypes = [i64, ctypes.POINTER(UskSketchC), ctypes.POINTER(vp), ctypes.c_int, i64,
                                          ctypes.POINTER(vp), ctypes.c_uint32, vp, vp]
    lib.usk_gemv_multi_static.restype = ctypes.c_int
    lib.usk_gemm.argtypes = [ctypes.POINTER(UskSketchC), vp, i64, vp, vp, ctypes.c_size_t, vp, vp]
    lib.usk_gemm.restype = ctypes.c_int
    lib.usk_gemm_ex.argtypes = [ctypes.POINTER(UskSketchC), vp, i64, vp, ctypes.c_uint32, vp, vp]
    lib.usk_gemm_ex.restype = ctypes.c_int
    lib.usk_status_str.argtypes = [ctypes.c_int]
    lib.usk_status_str.restype = ctypes.c_char_p
    lib.usk_format_version.argtypes = []
    lib.usk_format_version.restype = ctypes.c_uint32
    lib.usk_debug_set_geometry.argtypes = [ctypes.c_int, ctypes.c_int]
    lib.usk_debug_set_geometry.restype = None
    lib.usk_debug_set_gemv_path.argtypes = [ctypes.c_int]
    lib.usk_debug_set_gemv_path.restype = None
    lib.usk_debug_set_gemv_rows.argtypes = [ctypes.c_int]
    lib.usk_debug_set_gemv_rows.restype = None
    lib.usk_debug_set_gemm_splits.argtypes = [ctypes.c_int]
    lib.usk_debug_set_gemm_splits.restype = None
    lib.usk_debug_set_gemm_issuers.argtypes = [ctypes.c_int]
    lib.usk_debug_set_gemm_issuers.restype = None
    lib.usk_debug_inject_timeout.argtypes = [ctypes.c_int]
    lib.usk_debug_inject_timeout.restype = None
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(st: int, what: str):
    if st != USK_OK:
        raise UskError(st, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return USK_BF16
    if t.dtype == torch.float32:
        return USK_F32
    raise TypeError("expected a bfloat16 or float32 tensor, got %s" % t.dtype)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libusk works on CUDA tensors only (no CPU fallback)")


def usk_status_str(status: int) -> str:
    return load_library().usk_status_str(int(status)).decode()


def usk_format_version() -> int:
    return int(load_library().usk_format_version())


def usk_plan_slots(weights, importance, budget_bits: float):
    """Hash slots per unit (2, 4 or 8) from importance under a bits-per-weight
    budget (host computation in the library; see include/usk.h)."""
    n = len(weights)
    w = (ctypes.c_int64 * max(n, 1))(*[int(v) for v in weights])
    imp = (ctypes.c_double * max(n, 1))(*[float(v) for v in importance])
    out = (ctypes.c_uint32 * max(n, 1))()
    _check(load_library().usk_plan_slots(n, w, imp, ctypes.c_double(budget_bits), out), "usk_plan_slots")
    return [int(out[i]) for i in range(n)]


def usk_sizes_ex(M: int, K: int, version: int = FORMAT_MAXKEY, slots: int = 0):
    c = ctypes.c_size_t()
    s = ctypes.c_size_t()
    _check(load_library().usk_sizes_ex(M, K, version, slots, ctypes.byref(c), ctypes.byref(s)), "usk_sizes_ex")
    return c.value, s.value


def usk_sizes(M: int, K: int):
    c = ctypes.c_size_t()
    s = ctypes.c_size_t()
    _check(load_library().usk_sizes(M, K, ctypes.byref(c), ctypes.byref(s)), "usk_sizes")
    return c.value, s.value


def usk_rate_map_plan(M: int, K: int, slots):
    """Host rate table of a per-row-block-rate sketch: (offset list, order list,
    (count2, count4, count8), code_bytes) from one slot count per 64-row block."""
    n = M // 64 if M > 0 else 0
    sl = (ctypes.c_uint32 * max(n, 1))(*[int(v) for v in slots])
    off = (ctypes.c_int64 * max(n, 1))()
    order = (ctypes.c_int32 * max(n, 1))()
    cnt = (ctypes.c_int64 * 3)()
    total = ctypes.c_int64()
    if len(slots) != n:
        raise ValueError("one slot count per 64-row block")
    _check(load_library().usk_rate_map_plan(M, K, sl, off, order, cnt, ctypes.byref(total)), "usk_rate_map_plan")
    return [int(off[i]) for i in range(n)], [int(order[i]) for i in range(n)], tuple(int(c) for c in cnt), total.value


@dataclass
class RateMap:
    """Per-row-block rates of a format-1 sketch: slot counts (2, 4 or 8) per
    64-row block and the device tables the kernels read (byte offset of each
    block's codes; row blocks grouped by slot count)."""
    slots: list
    offset: torch.Tensor  # int64 [M/64], device
    order: torch.Tensor   # int32 [M/64], device
    count: tuple
    code_bytes: int

    def as_c(self) -> UskRateMapC:
        n = len(self.slots)
        for t, dt, name in ((self.offset, torch.int64, "offset"), (self.order, torch.int32, "order")):
            if t.dtype != dt or not t.is_contiguous() or t.numel() != n:
                raise ValueError("RateMap.%s must be a contiguous %s tensor of %d entries" % (name, dt, n))
            if n and not t.is_cuda:
                raise ValueError("RateMap.%s must be on the GPU (the kernels read it)" % name)
        if sum(self.count) != n:
            raise ValueError("RateMap.count must add up to the row blocks")
        c = UskRateMapC(self.offset.data_ptr() if self.offset.numel() else None,
                        self.order.data_ptr() if self.order.numel() else None)
        for g in range(3):
            c.count[g] = int(self.count[g])
        c.code_bytes = int(self.code_bytes)
        return c


def usk_rate_map(M: int, K: int, slots, device="cuda") -> RateMap:
    """RateMap for an M x K sketch: the library plans the table on the host,
    torch copies it to the device."""
    off, order, count, total = usk_rate_map_plan(M, K, slots)
    return RateMap([int(v) for v in slots], torch.tensor(off, dtype=torch.int64, device=device),
                   torch.tensor(order, dtype=torch.int32, device=device), count, total)


@dataclass
class Sketch:
    """A built sketch: int8 codes [M*K/16] and binary16 scales [M/64] on the GPU,
    with its format (1 or 2) and number of hash rows."""
    M: int
    K: int
    seed: int
    codes: torch.Tensor
    scales: torch.Tensor  # int16 storage of binary16 bit patterns
    version: int = FORMAT_MAXKEY
    depth: int = 1
    slots: int = 0  # hash slots per class as built (0 = the format's default)
    rates: RateMap | None = None  # per-row-block rates (format 1)

    def as_c(self) -> UskSketchC:
        c = UskSketchC(self.M, self.K, self.seed & (2**64 - 1), self.codes.data_ptr() if self.codes.numel() else None,
                       self.scales.data_ptr() if self.scales.numel() else None, self.version, self.depth,
                       self.slots, 0)
        if self.rates is not None:
            c._rates = self.rates.as_c()  # kept alive with the struct
            c.rates = ctypes.pointer(c._rates)
        return c


def usk_build(W: torch.Tensor, importance: torch.Tensor | None = None, seed: int = 0,
              codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
              status: torch.Tensor | None = None, stream=None, version: int = FORMAT_MAXKEY,
              depth: int = 1, slots: int = 0, rates: RateMap | None = None) -> Sketch:
    """Sketch of W [M, K] (bf16 or fp32, CUDA).  Outputs are allocated with torch
    when not given.  `status` is an optional int32 CUDA tensor of 1 element into
    which device-detected USK_FLAG_* bits are OR-ed.  version=FORMAT_ABSMAXMIN
    builds the multi-row AbsMaxMin sketch with `depth` (1, 2 or 4) hash rows,
    version=FORMAT_COLSHARED the column-shared projection sketch (no importance
    for either), version=FORMAT_Q4 the format-1 sketch with 4-bit codes.  slots
    (format 1): 2, 4 or 8 hash slots per class, 0.25, 0.5 or 1 bit/weight.
    rates (format 1, slots 0): a RateMap giving every 64-row block its own slot
    count (usk_rate_map)."""
    _need_cuda(W, importance, codes, scales, status)
    if W.dim() != 2 or W.stride(1) != 1:
        raise ValueError("W must be a 2-D row-major tensor")
    M, K = W.shape
    nb = M * K * (slots if (version == FORMAT_MAXKEY and slots in (2, 8)) else 4) // 64
    if rates is not None:
        nb = int(rates.code_bytes)
    if codes is None:
        codes = torch.empty(max(nb, 1), dtype=torch.int8, device=W.device)[:nb]
    if scales is None:
        scales = torch.empty(max(M // 64, 1), dtype=torch.int16, device=W.device)[: M // 64]
    if importance is not None and (importance.dtype != torch.float32 or not importance.is_contiguous()):
        raise TypeError("importance must be a contiguous float32 tensor")
    p = UskParams(version, 0, seed & (2**64 - 1), depth, slots)
    if rates is not None:
        rc = rates.as_c()
        p.rates = ctypes.pointer(rc)
    st = load_library().usk_build(_ptr(W), _dtype_code(W), M, K, W.stride(0), _ptr(importance), ctypes.byref(p),
                                  _ptr(codes) if nb else None, _ptr(scales) if M // 64 else None,
                                  _ptr(status), _stream(stream))
    _check(st, "usk_build")
    return Sketch(M, K, seed, codes, scales, version, depth, slots, rates)


def usk_gemv(sketch: Sketch, x: torch.Tensor, y: torch.Tensor | None = None,
             status: torch.Tensor | None = None, stream=None, pdl: bool = False) -> torch.Tensor:
    """y [batch, M] fp32 = W_hat x^T for x [batch, K] (bf16 or fp32), batch 1..15.

    pdl=True launches as a programmatic dependent of the previous kernel in the
    stream (usk_gemv_ex with USK_GEMV_PDL): the sketch codes are prefetched
    before that kernel finishes, so no kernel still running may write them."""
    _need_cuda(x, y, status)
    if x.dim() == 1:
        x = x[None, :]
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, sketch.M), dtype=torch.float32, device=x.device)
    sk = sketch.as_c()
    st = load_library().usk_gemv_ex(ctypes.byref(sk), _ptr(x), _dtype_code(x), batch, _ptr(y),
                                    GEMV_PDL if pdl else 0, _ptr(status), _stream(stream))
    _check(st, "usk_gemv")
    return y


class MultiCall:
    """Marshalled arguments of one usk_gemv_multi list (built once, reusable:
    the ctypes arrays stay alive with this object)."""

    def __init__(self, sketches, xs, ys):
        n = len(sketches)
        self.n = n
        self._c = [sk.as_c() for sk in sketches]
        self.sk = (UskSketchC * max(n, 1))(*self._c)
        self.x = (ctypes.c_void_p * max(n, 1))(*[x.data_ptr() for x in xs])
        self.y = (ctypes.c_void_p * max(n, 1))(*[y.data_ptr() for y in ys])


def usk_gemv_multi_ws_bytes(sketches, batch: int) -> int:
    """Workspace bytes usk_gemv_multi needs for this list of sketches and batch."""
    n = len(sketches)
    arr = (UskSketchC * max(n, 1))(*[sk.as_c() for sk in sketches])
    out = ctypes.c_size_t()
    _check(load_library().usk_gemv_multi_ws_bytes(n, arr, int(batch), ctypes.byref(out)), "usk_gemv_multi_ws_bytes")
    return out.value


def usk_gemv_multi(sketches, xs, ys=None, ws: torch.Tensor | None = None, status: torch.Tensor | None = None,
                   stream=None, pdl: bool = False, call: MultiCall | None = None):
    """y[l] = W_hat_l x[l]^T for several sketches in one launch (batch 1..8, bf16
    x).  ys are allocated when not given.  ws: a zero-filled uint8 CUDA tensor of
    at least usk_gemv_multi_ws_bytes bytes (allocated with torch.zeros when None;
    pass the same one to consecutive calls on a stream).  Returns ys."""
    xs = [x if x.dim() == 2 else x[None, :] for x in xs]
    _need_cuda(*xs, ws, status)
    for x in xs:
        if x.dtype != torch.bfloat16 or not x.is_contiguous():
            raise TypeError("usk_gemv_multi takes contiguous bfloat16 x")
    batch = xs[0].shape[0] if xs else 0
    if any(x.shape[0] != batch for x in xs):
        raise ValueError("every x of one call has the same batch")
    if ys is None:
        ys = [torch.empty((batch, sk.M), dtype=torch.float32, device=x.device) for sk, x in zip(sketches, xs)]
    if ws is None:
        need = usk_gemv_multi_ws_bytes(sketches, batch)
        ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=xs[0].device) if xs else None
    if call is None:
        call = MultiCall(sketches, xs, ys)
    st = load_library().usk_gemv_multi(call.n, call.sk, call.x, USK_BF16, batch, call.y, _ptr(ws),
                                       ws.numel() if ws is not None else 0, GEMV_PDL if pdl else 0, _ptr(status),
                                       _stream(stream))
    _check(st, "usk_gemv_multi")
    return ys


def usk_gemm(sketch: Sketch, x: torch.Tensor, y: torch.Tensor | None = None,
             status: torch.Tensor | None = None, stream=None, pdl: bool = False) -> torch.Tensor:
    """y [batch, M] fp32 = W_hat x^T for bf16 x [batch, K], batch 16..256 (multiple of 16).

    pdl=True launches as a programmatic dependent of the previous kernel in the
    stream (usk_gemm_ex with USK_GEMM_PDL): set-up, code copies and decoding
    overlap that kernel; x, scales, y and status wait for it.  The caller
    guarantees that no kernel still running in the stream writes the sketch."""
    _need_cuda(x, y, status)
    if x.dtype != torch.bfloat16 or not x.is_contiguous() or x.dim() != 2:
        raise TypeError("x must be a contiguous 2-D bfloat16 tensor")
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, sketch.M), dtype=torch.float32, device=x.device)
    sk = sketch.as_c()
    st = load_library().usk_gemm_ex(ctypes.byref(sk), _ptr(x), batch, _ptr(y), GEMM_PDL if pdl else 0,
                                    _ptr(status), _stream(stream))
    _check(st, "usk_gemm")
    return y


def usk_debug_set_geometry(build_cluster: int = 0, gemv_tiles_per_block: int = 0) -> None:
    load_library().usk_debug_set_geometry(int(build_cluster), int(gemv_tiles_per_block))


def usk_debug_set_gemv_path(path: int = 0) -> None:
    """0 automatic, 1 bf16 tensor path, 2 integer path with clusters, 3 integer
    row-slab path (2 and 3 where eligible)."""
    load_library().usk_debug_set_gemv_path(int(path))


def usk_debug_set_gemv_rows(rows: int = 0) -> None:
    """Rows per block of the row-slab path (16, 32, 64; other values = automatic)."""
    load_library().usk_debug_set_gemv_rows(int(rows))


def usk_debug_set_gemm_splits(splits: int = 0) -> None:
    """Blocks along K per 128-row tile of usk_gemm (0 = automatic)."""
    load_library().usk_debug_set_gemm_splits(int(splits))


def usk_debug_set_gemm_issuers(issuers: int = 0) -> None:
    """MMA issuer warps of usk_gemm (1, 2 or 4; 0 = automatic)."""
    load_library().usk_debug_set_gemm_issuers(int(issuers))


def usk_debug_inject_timeout(kernel: int = 0) -> None:
    """Test hook: 1 build, 2 gemm, 3 gemv (integer path) skip one copy/commit in
    block (0, 0) so its bounded wait gives up (USK_FLAG_TIMEOUT); 0 = off."""
    load_library().usk_debug_inject_timeout(int(kernel))
