"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds none of the sketch's arithmetic: it only draws weights,
importance vectors and activations with numpy's PCG64 generator and rounds
float32 draws to bfloat16 bit patterns (``device_weights_normal`` draws with
torch's seeded CUDA generator instead: a fast fill of the largest matrices for
timing runs only, where the values do not change the work).  Both the CPU oracle and the CUDA path
consume the arrays it returns, so neither side generates its own inputs.

bf16 arrays are returned as numpy uint16 bit patterns (numpy has no bfloat16).

Workloads (weights of LLM-shaped layers; no trained checkpoints exist here, so
Student-t(4) with injected x20 outliers stands in for heavy-tailed trained
weights):
  * small   -- one 256x1024 fp32 matrix N(0, 0.02^2), lognormal(0, 1) per-column
               importance, x ~ N(0, 1) at batch 1 (fp32 and bf16 copies).
  * layer   -- one 4096x4096 bf16 layer, 0.02 * t(4) with 0.1 % of entries x20,
               importance per column = mean |x| over 128 N(0, 1) calibration
               rows; x bf16 N(0, 1) at batch 1 and 4.
  * llama7b -- q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008,
               bf16 N(0, 0.02^2), no importance; batch 1, 4, 16.
  * mlp70b  -- 28672x8192 and 8192x28672 bf16 0.02 * t(4); batch 16, 32, 64.
  * stack7b -- 32 layers x {q, k, v, o, gate, up, down} of the llama7b shapes,
               bf16 N(0, 0.02^2); one independent N(0, 1) x per linear, batch 1.
"""
from __future__ import annotations

import numpy as np

# stream ids inside one workload seed
_W, _IMP, _X, _OUT = 0, 1, 2, 3


def rng(seed: int, stream: int) -> np.random.Generator:
    """Independent PCG64 stream `stream` of workload seed `seed`."""
    return np.random.default_rng([int(seed), int(stream)])


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # 32-bit arithmetic cannot wrap for non-NaN patterns (at most 0xFF807FFF)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _cast(a32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(a32, dtype=np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(a32)
    raise ValueError(dtype)


def weights_normal(M: int, K: int, seed: int, std: float = 0.02, dtype: str = "bf16"):
    g = rng(seed, _W)
    return _cast(g.standard_normal((M, K), dtype=np.float32) * np.float32(std), dtype)


def weights_student_t(M: int, K: int, seed: int, df: float = 4.0, scale: float = 0.02,
                      outlier_frac: float = 0.0, outlier_mult: float = 20.0, dtype: str = "bf16"):
    g = rng(seed, _W)
    w = (g.standard_t(df, size=(M, K)) * scale).astype(np.float32)
    if outlier_frac > 0:
        mask = g.random((M, K)) < outlier_frac
        w = np.where(mask, w * np.float32(outlier_mult), w).astype(np.float32)
    return _cast(w, dtype)


def importance_lognormal(K: int, seed: int) -> np.ndarray:
    return rng(seed, _IMP).lognormal(0.0, 1.0, size=K).astype(np.float32)


def importance_calibration(K: int, seed: int, rows: int = 128) -> np.ndarray:
    """Per-column mean |x| over `rows` N(0, 1) calibration rows (float64 mean)."""
    x = rng(seed, _IMP).standard_normal((rows, K))
    return np.abs(x).mean(axis=0).astype(np.float32)


def activations(batch: int, K: int, seed: int, dtype: str = "bf16", stream: int = _X):
    g = rng(seed, stream)
    return _cast(g.standard_normal((batch, K), dtype=np.float32), dtype)


# --------------------------------------------------------------- workloads

LLAMA7B_SHAPES = {
    "q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
    "gate": (11008, 4096), "up": (11008, 4096), "down": (4096, 11008),
}
LLAMA7B_ORDER = ["q", "k", "v", "o", "gate", "up", "down"]
MLP70B_SHAPES = {"up": (28672, 8192), "down": (8192, 28672)}


def small(dtype_x: str = "f32"):
    """256x1024 fp32 weights, lognormal importance, x at batch 1 (seed 0)."""
    seed = 0
    return {
        "seed": seed,
        "W": weights_normal(256, 1024, seed, 0.02, "f32"),
        "importance": importance_lognormal(1024, seed),
        "x": activations(1, 1024, seed, dtype_x),
    }


def layer(batch: int = 1, M: int = 4096, K: int = 4096):
    """One bf16 layer with outliers and calibration importance (seed 1)."""
    seed = 1
    return {
        "seed": seed,
        "W": weights_student_t(M, K, seed, 4.0, 0.02, 0.001, 20.0, "bf16"),
        "importance": importance_calibration(K, seed, 128),
        "x": activations(batch, K, seed, "bf16"),
    }


def row_block_gains(RB: int, seed: int, sigma: float = 0.5) -> np.ndarray:
    """One lognormal gain exp(N(0, sigma^2)) per 64-row block: rows of unequal
    output energy (stream of its own)."""
    return np.exp(rng(seed, 7).normal(0.0, sigma, size=RB)).astype(np.float32)


def scale_row_blocks(W: np.ndarray, gains: np.ndarray) -> np.ndarray:
    """W (bf16 bits or float32) with 64-row block rb multiplied by gains[rb],
    rounded back to the input type."""
    M, K = W.shape
    Wf = bf16_bits_to_f32(W) if W.dtype == np.uint16 else W
    out = (Wf.reshape(M // 64, 64, K) * gains[:, None, None].astype(np.float32)).reshape(M, K)
    return f32_to_bf16_bits(out) if W.dtype == np.uint16 else out.astype(np.float32)


def llama7b_layer(name: str, batch: int = 1):
    """One linear of the 7B layer set (seed 2 + its index)."""
    idx = LLAMA7B_ORDER.index(name)
    seed = 2 + idx
    M, K = LLAMA7B_SHAPES[name]
    return {"seed": seed, "W": weights_normal(M, K, seed, 0.02, "bf16"), "importance": None,
            "x": activations(batch, K, seed, "bf16")}


def mlp70b(name: str, batch: int = 16):
    """70B-MLP-shaped matrix (seed 3; 'down' uses stream offset via seed 3 + 100)."""
    seed = 3 if name == "up" else 103
    M, K = MLP70B_SHAPES[name]
    return {"seed": seed, "W": weights_student_t(M, K, seed, 4.0, 0.02, 0.0, 20.0, "bf16"),
            "importance": None, "x": activations(batch, K, seed, "bf16")}


def device_weights_normal(M: int, K: int, seed: int, std: float = 0.02, device="cuda"):
    """bf16 N(0, std^2) [M, K] drawn on the device by torch's seeded generator
    (timing inputs only; not reproducible against the numpy streams)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return (torch.randn((M, K), generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def stack7b_seed(layer_idx: int, linear: str) -> int:
    return 4 + 7 * layer_idx + LLAMA7B_ORDER.index(linear)
