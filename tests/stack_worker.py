"""Host half of the whole-stack parity test (32 layers x 7 linears of the
7B-shaped stack): one linear's seeded weights, the oracle's sketch of them and
the oracle's float64 products on a full 64-row block plus the first and last
rows.  Runs in spawned worker processes; it imports numpy, the input
generators and the oracle only (no CUDA), so a pool of them can start after the
parent has initialised its GPU."""
import numpy as np

import gen
import oracle


def check_rows(M: int, layer: int, idx: int) -> np.ndarray:
    """Rows whose products are compared: the whole row block (layer * 7 + idx)
    mod (M / 64), so that the 224 linears cover row blocks all over the
    matrices, and the first and last rows."""
    rb = (layer * 7 + idx) % (M // 64)
    return np.concatenate([np.arange(64 * rb, 64 * rb + 64), [0, M - 1]]).astype(np.int64)


def linear_case(job):
    layer, name = job
    idx = gen.LLAMA7B_ORDER.index(name)
    seed = gen.stack7b_seed(layer, name)
    M, K = gen.LLAMA7B_SHAPES[name]
    W = gen.weights_normal(M, K, seed, 0.02, "bf16")
    o = oracle.build_sketch(W, None, seed)
    x = gen.activations(1, K, seed, "bf16")
    rows = check_rows(M, layer, idx)
    ref = oracle.gemv_f64(o["codes"], o["scales"], M, K, x, seed, rows=rows)
    return {"layer": layer, "name": name, "seed": seed, "W": W, "status": o["status"], "codes": o["codes"],
            "scales": o["scales"], "x": x, "rows": rows, "ref": ref}
