"""Independent pure-Python restatement of the sketch, for tiny matrices.

It pins the C oracle from a second, separately written reading of the format:
Python integers for the hash, explicit member lists per bucket sorted by
(key descending, row-major index ascending) instead of a running maximum, and
numpy's own float16 conversion and rint for the scale and the codes.  It shares
no code with the oracle or with the CUDA library.

Format (64x256 hash tiles, 64-row scale blocks; "UltraSketchLLM" explainer,
Metodologia §1 AbsMaxMin sketch, with the library's frozen readings):
  tile key z = SplitMix64(seed) output number tile_id + 1, tile_id = rb*(K/256)+tc
  A = low32(z) | 1, C = high32(z)
  octet o = c // 8, m = 32*r + o, h = (A*m + C) mod 2^32, slot = (4*h) >> 32
  class = (o + r) % 32, bucket = (slot*32 + class)*8 + c % 8
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1


def splitmix64_output(seed: int, n: int) -> int:
    z = (seed + n * 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def bucket_of(K: int, seed: int, i: int, j: int) -> int:
    rb, r = divmod(i, 64)
    tc, c = divmod(j, 256)
    tile_id = rb * (K // 256) + tc
    z = splitmix64_output(seed, tile_id + 1)
    A = (z & 0xFFFFFFFF) | 1
    C = z >> 32
    o = c // 8
    m = 32 * r + o
    h = (A * m + C) & 0xFFFFFFFF
    slot = (4 * h) >> 32
    cls = (o + r) % 32
    b = (slot * 32 + cls) * 8 + (c % 8)
    return rb * 4 * K + 1024 * tc + b


def to_f32(W: np.ndarray) -> np.ndarray:
    if W.dtype == np.float32:
        return W
    return (W.astype(np.uint32) << 16).view(np.float32)


def build(W: np.ndarray, importance=None, seed: int = 0):
    """Returns (codes int8, scales uint16, winner int64 flat index or -1)."""
    Wf = to_f32(np.ascontiguousarray(W))
    M, K = Wf.shape
    imp = np.ones(K, np.float32) if importance is None else np.asarray(importance, np.float32)
    nb = M * K // 16
    members = [[] for _ in range(nb)]
    for i in range(M):
        for j in range(K):
            members[bucket_of(K, seed, i, j)].append(i * K + j)
    winner = np.full(nb, -1, dtype=np.int64)
    value = np.zeros(nb, dtype=np.float32)
    flat = Wf.reshape(-1)
    for b, mem in enumerate(members):
        if not mem:
            continue
        keyed = [(-float(np.float32(abs(flat[q])) * imp[q % K]), q) for q in mem]
        keyed.sort()
        winner[b] = keyed[0][1]
        value[b] = flat[winner[b]]
    codes = np.zeros(nb, dtype=np.int8)
    scales = np.zeros(M // 64, dtype=np.uint16)
    per = 4 * K
    for rb in range(M // 64):
        v = value[rb * per:(rb + 1) * per]
        mx = np.float32(np.max(np.abs(v))) if per else np.float32(0)
        s16 = np.float16(np.float32(mx) / np.float32(127.0))
        scales[rb] = s16.view(np.uint16)
        s = np.float32(s16)
        if s != 0:
            q = np.rint(v / s)
            codes[rb * per:(rb + 1) * per] = np.clip(q, -127, 127).astype(np.int8)
    return codes, scales, winner


# ---- format 2: the multi-row AbsMaxMin sketch (Metodologia §1: a bucket keeps
# its member of smallest magnitude; decompression takes the largest magnitude
# over the hash rows).  depth D rows share the tile's 1024 buckets; row rho is
# keyed by SplitMix64 output tile_id*D + rho + 1; class = (o + r) % (32 // D).

def bucket_of_amm(K: int, seed: int, depth: int, rho: int, i: int, j: int) -> int:
    rb, r = divmod(i, 64)
    tc, c = divmod(j, 256)
    tile_id = rb * (K // 256) + tc
    z = splitmix64_output(seed, tile_id * depth + rho + 1)
    A = (z & 0xFFFFFFFF) | 1
    C = z >> 32
    o = c // 8
    h = (A * (32 * r + o) + C) & 0xFFFFFFFF
    slot = (4 * h) >> 32
    ncls = 32 // depth
    b = rho * (1024 // depth) + (slot * ncls + (o + r) % ncls) * 8 + (c % 8)
    return rb * 4 * K + 1024 * tc + b


def build_amm(W: np.ndarray, seed: int = 0, depth: int = 2):
    """Returns (codes, scales, winner).  Members listed per bucket and sorted by
    (|w|, row-major index); codes by exact rational arithmetic (Fraction):
    sign(v) * min(127, floor(|v| / s))."""
    from fractions import Fraction
    Wf = to_f32(np.ascontiguousarray(W))
    M, K = Wf.shape
    nb = M * K // 16
    members = [[] for _ in range(nb)]
    for i in range(M):
        for j in range(K):
            for rho in range(depth):
                members[bucket_of_amm(K, seed, depth, rho, i, j)].append(i * K + j)
    flat = Wf.reshape(-1)
    winner = np.full(nb, -1, dtype=np.int64)
    value = np.zeros(nb, dtype=np.float32)
    for b, mem in enumerate(members):
        if mem:
            winner[b] = min(mem, key=lambda q: (abs(float(flat[q])), q))
            value[b] = flat[winner[b]]
    codes = np.zeros(nb, dtype=np.int8)
    scales = np.zeros(M // 64, dtype=np.uint16)
    per = 4 * K
    for rb in range(M // 64):
        v = value[rb * per:(rb + 1) * per]
        mx = np.float32(np.max(np.abs(v)))
        s16 = np.float16(mx / np.float32(127.0))
        scales[rb] = s16.view(np.uint16)
        s = Fraction(float(s16))
        if s != 0:
            for q in range(per):
                a = Fraction(float(abs(v[q])))
                n = min(127, int(a / s))  # floor of a non-negative rational
                codes[rb * per + q] = -n if v[q] < 0 else n
    return codes, scales, winner


def decode_amm(codes, scales, M: int, K: int, seed: int = 0, depth: int = 2) -> np.ndarray:
    """W_hat: per weight the code of largest magnitude over the rows, ties to
    the lowest row, times the block scale."""
    out = np.zeros((M, K), dtype=np.float64)
    for i in range(M):
        s = float(np.uint16(scales[i // 64]).view(np.float16))
        for j in range(K):
            cs = [int(codes[bucket_of_amm(K, seed, depth, rho, i, j)]) for rho in range(depth)]
            best = cs[0]
            for c in cs[1:]:
                if abs(c) > abs(best):
                    best = c
            out[i, j] = best * s
    return out


# ---- format 3: the column-shared projection (Metodologia §4: W_hat = S . P^T,
# compression a MIN reduction over |w|).  Bucket b' of tile tc holds the columns
# sigma_tc(16 b' + k); S keeps per row and bucket the member of smallest |w|.

def sigma_cs(seed: int, tc: int, u: int) -> int:
    z = splitmix64_output(seed, tc + 1)
    A, B, C = (z & 255) | 1, (z >> 8) & 255, ((z >> 16) & 255) | 1
    v1 = (A * u + B) % 256
    v2 = v1 ^ (v1 >> 4)
    v3 = (C * v2) % 256
    return v3 ^ (v3 >> 3)


def build_cs(W: np.ndarray, seed: int = 0):
    """Returns (codes row-major [M*K/16], scales, winner flat index)."""
    from fractions import Fraction
    Wf = to_f32(np.ascontiguousarray(W))
    M, K = Wf.shape
    nb = K // 16
    groups = []  # global bucket -> its 16 columns
    for tc in range(K // 256):
        for bp in range(16):
            groups.append([256 * tc + sigma_cs(seed, tc, 16 * bp + k) for k in range(16)])
    winner = np.zeros(M * nb, dtype=np.int64)
    value = np.zeros(M * nb, dtype=np.float32)
    for i in range(M):
        for b, cols in enumerate(groups):
            j = min(cols, key=lambda c: (abs(float(Wf[i, c])), c))
            winner[i * nb + b] = i * K + j
            value[i * nb + b] = Wf[i, j]
    codes = np.zeros(M * nb, dtype=np.int8)
    scales = np.zeros(M // 64, dtype=np.uint16)
    for rb in range(M // 64):
        sl = slice(rb * 64 * nb, (rb + 1) * 64 * nb)
        v = value[sl]
        s16 = np.float16(np.float32(np.max(np.abs(v))) / np.float32(127.0))
        scales[rb] = s16.view(np.uint16)
        s = Fraction(float(s16))
        if s != 0:
            out = codes[sl]
            for q in range(len(v)):
                n = min(127, int(Fraction(float(abs(v[q]))) / s))
                out[q] = -n if v[q] < 0 else n
    return codes, scales, winner


# ---- format 4: the format-1 rule with 8 weights per bucket and 4-bit codes
# (Resultados: 0.5 bit/weight with 4-bit quantisation).  8 slots per class.

def bucket_of_q4(K: int, seed: int, i: int, j: int) -> int:
    """Global bucket index rb * 8K + 2048 tc + b."""
    rb, r = divmod(i, 64)
    tc, c = divmod(j, 256)
    z = splitmix64_output(seed, rb * (K // 256) + tc + 1)
    A = (z & 0xFFFFFFFF) | 1
    C = z >> 32
    o = c // 8
    h = (A * (32 * r + o) + C) & 0xFFFFFFFF
    slot = (8 * h) >> 32
    b = (slot * 32 + (o + r) % 32) * 8 + (c % 8)
    return rb * 8 * K + 2048 * tc + b


def build_q4(W: np.ndarray, importance=None, seed: int = 0):
    """Returns (packed codes [M*K/16] int8, scales, winner per bucket)."""
    Wf = to_f32(np.ascontiguousarray(W))
    M, K = Wf.shape
    imp = np.ones(K, np.float32) if importance is None else np.asarray(importance, np.float32)
    nb = M * K // 8
    members = [[] for _ in range(nb)]
    for i in range(M):
        for j in range(K):
            members[bucket_of_q4(K, seed, i, j)].append(i * K + j)
    flat = Wf.reshape(-1)
    winner = np.full(nb, -1, dtype=np.int64)
    value = np.zeros(nb, dtype=np.float32)
    for b, mem in enumerate(members):
        if mem:
            keyed = sorted((-float(np.float32(abs(flat[q])) * imp[q % K]), q) for q in mem)
            winner[b] = keyed[0][1]
            value[b] = flat[winner[b]]
    nib = np.zeros(nb, dtype=np.int64)
    scales = np.zeros(M // 64, dtype=np.uint16)
    per = 8 * K
    for rb in range(M // 64):
        v = value[rb * per:(rb + 1) * per]
        s16 = np.float16(np.float32(np.max(np.abs(v))) / np.float32(7.0))
        scales[rb] = s16.view(np.uint16)
        s = np.float32(s16)
        if s != 0:
            nib[rb * per:(rb + 1) * per] = np.clip(np.rint(v / s), -7, 7).astype(np.int64)
    u = (nib & 15).astype(np.uint8)
    packed = (u[0::2] | (u[1::2] << 4)).astype(np.uint8).view(np.int8)
    return packed, scales, winner


def bucket_of_vr(K: int, seed: int, slots, i: int, j: int) -> int:
    """Per-row-block rates: row block rb has slots[rb] hash slots per class
    (slot = (slots[rb] * h) >> 32) and its codes start after those of the
    blocks above it (K * slots[q] bytes each)."""
    rb, r = divmod(i, 64)
    tc, c = divmod(j, 256)
    S = int(slots[rb])
    z = splitmix64_output(seed, rb * (K // 256) + tc + 1)
    A = (z & 0xFFFFFFFF) | 1
    C = z >> 32
    o = c // 8
    h = (A * (32 * r + o) + C) & 0xFFFFFFFF
    b = (((S * h) >> 32) * 32 + (o + r) % 32) * 8 + c % 8
    start = sum(int(s) * K for s in slots[:rb])
    return start + 256 * S * tc + b


def build_vr(W: np.ndarray, importance=None, seed: int = 0, slots=None):
    """Returns (codes int8, scales uint16) of the per-row-block-rate sketch."""
    Wf = to_f32(np.ascontiguousarray(W))
    M, K = Wf.shape
    imp = np.ones(K, np.float32) if importance is None else np.asarray(importance, np.float32)
    nb = K * sum(int(s) for s in slots)
    members = [[] for _ in range(nb)]
    for i in range(M):
        for j in range(K):
            members[bucket_of_vr(K, seed, slots, i, j)].append(i * K + j)
    flat = Wf.reshape(-1)
    value = np.zeros(nb, np.float32)
    for b, mem in enumerate(members):
        if mem:
            best = sorted((-float(np.float32(np.float32(abs(flat[m])) * imp[m % K])), m) for m in mem)[0][1]
            value[b] = flat[best]
    codes = np.zeros(nb, np.int8)
    scales = np.zeros(M // 64, np.uint16)
    start = 0
    for rb in range(M // 64):
        n = int(slots[rb]) * K
        v = value[start:start + n]
        s16 = np.float16(np.float32(np.max(np.abs(v))) / np.float32(127.0))
        scales[rb] = s16.view(np.uint16)
        s = np.float32(s16)
        if s != 0:
            codes[start:start + n] = np.clip(np.rint(v / s), -127, 127).astype(np.int8)
        start += n
    return codes, scales
