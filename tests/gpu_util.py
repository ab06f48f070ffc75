"""Helpers for the GPU tests: numpy <-> torch CUDA transfers of the seeded inputs."""
import numpy as np
import torch


def to_dev(a: np.ndarray) -> torch.Tensor:
    """uint16 arrays are bf16 bit patterns; float32 stays float32."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    if a.dtype == np.float32:
        return torch.from_numpy(a).cuda()
    raise TypeError(a.dtype)


def codes_np(sk) -> np.ndarray:
    return sk.codes.cpu().numpy().view(np.int8)


def scales_np(sk) -> np.ndarray:
    return sk.scales.cpu().numpy().view(np.uint16)


def status_tensor() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    """max |y - ref| / max |ref| (the products' tolerance measure)."""
    den = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(y.astype(np.float64) - ref)))
    return num / den if den > 0 else num


def sketch_from_oracle(o, M: int, K: int, seed: int, version: int = 1, depth: int = 1):
    """A device sketch holding the ORACLE's codes and scales (uploaded), so that a
    product test's expected value never depends on the CUDA build."""
    import sub_bit_weight_usk_b200 as usk
    codes = torch.from_numpy(np.ascontiguousarray(o["codes"]).copy()).cuda()
    scales = torch.from_numpy(np.ascontiguousarray(o["scales"]).view(np.int16).copy()).cuda()
    return usk.Sketch(M, K, seed, codes, scales, version, depth)
