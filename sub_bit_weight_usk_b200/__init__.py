"""UltraSketchLLM sketch weights on NVIDIA B200 (sm_100a).

Thin Python face of libusk.so (C ABI in include/usk.h): ``usk_build`` compresses
a weight matrix into a 0.5 bit/weight hashed sketch (format 1: one hash row,
largest key kept; format 2: the multi-row AbsMaxMin sketch; format 3: the
column-shared projection W_hat = S . P^T, multiplied as S (P^T x); format 4:
format 1 with 4-bit codes and 8 weights per bucket; format 1 at 2, 4 or 8 hash
slots per class, per sketch or per 64-row block); ``usk_gemv`` (batch 1-15)
and ``usk_gemm`` (batch 16-256) multiply the sketch with activations, rebuilding
every weight on the fly; ``usk_gemv_multi`` runs several independent batch 1-8
products in one persistent launch.  PyTorch supplies device memory and streams only.
"""
from ._native import (  # noqa: F401
    FLAG_BAD_IMPORTANCE,
    FLAG_NONFINITE_W,
    FLAG_RATE_MAP,
    FLAG_SCALE_OVERFLOW,
    FLAG_TIMEOUT,
    FORMAT_ABSMAXMIN,
    FORMAT_COLSHARED,
    FORMAT_MAXKEY,
    FORMAT_Q4,
    FORMAT_VERSION,
    GEMM_MAX_BATCH,
    GEMM_MIN_BATCH,
    GEMV_MAX_BATCH,
    LIB_PATH,
    RateMap,
    Sketch,
    UskError,
    load_library,
    usk_build,
    usk_debug_inject_timeout,
    usk_debug_set_gemv_path,
    usk_debug_set_gemv_rows,
    usk_debug_set_gemm_splits,
    usk_debug_set_gemm_issuers,
    usk_debug_set_geometry,
    usk_format_version,
    usk_gemm,
    usk_gemv,
    usk_gemv_multi,
    usk_gemv_multi_ws_bytes,
    MultiCall,
    usk_plan_slots,
    usk_rate_map,
    usk_rate_map_plan,
    usk_sizes,
    usk_sizes_ex,
    usk_status_str,
)
