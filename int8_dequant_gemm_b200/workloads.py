"""Seeded synthetic inputs with the shapes of the RT-J block projections.

This module draws random numbers and nothing else: no quantization, packing,
dequantization or matrix product lives here.  Both the CUDA path (through the
benchmark and the tests) and the CPU oracle take their inputs from it.

Shapes follow the RT-J hyper-parameters printed in the "Backends" page of the
relational-transformers docs (12 blocks, d_model 512, d_ff 2048) and the
projection names of the RT-J int4 / int8 model cards (wq, wk, wv, wg, wo,
ffn.w1, ffn.w2, ffn.w3).  Distributions: activations X ~ N(0, 1) fp32,
weights W ~ N(0, 0.02^2) fp32, drawn with numpy's PCG64 from
``seed = 1000 * config + 10 * block + tensor_id``.
"""
from __future__ import annotations

import numpy as np

NUM_BLOCKS = 12
D_MODEL = 512
D_FF = 2048
W_SIGMA = 0.02

# tensor ids used in the seed formula
TENSOR_IDS = {"wq": 0, "wk": 1, "wv": 2, "wg": 3, "wo": 4, "w1": 5, "w2": 6, "w3": 7,
              "x_qkvg": 8, "x_o": 9, "x_ffn": 10, "x_w2": 11}

# The mixed-precision recipe of the int4 card: attention q/k/v/gate and the
# ffn up-projections are q4 g32; the residual-writing wo and w2 stay q8.
# Fused groups concatenate rows in the listed order.
BLOCK_PROJECTIONS = {
    "qkvg": {"fmt": "q4", "parts": ("wq", "wk", "wv", "wg"), "N": 4 * D_MODEL, "K": D_MODEL,
             "x": "x_qkvg"},
    "wo": {"fmt": "q8", "parts": ("wo",), "N": D_MODEL, "K": D_MODEL, "x": "x_o"},
    "w13": {"fmt": "q4", "parts": ("w1", "w3"), "N": 2 * D_FF, "K": D_MODEL, "x": "x_ffn"},
    "w2": {"fmt": "q8", "parts": ("w2",), "N": D_MODEL, "K": D_FF, "x": "x_w2"},
}
PART_SHAPES = {"wq": (D_MODEL, D_MODEL), "wk": (D_MODEL, D_MODEL), "wv": (D_MODEL, D_MODEL),
               "wg": (D_MODEL, D_MODEL), "wo": (D_MODEL, D_MODEL), "w1": (D_FF, D_MODEL),
               "w3": (D_FF, D_MODEL), "w2": (D_MODEL, D_FF)}


def seed_for(config: int, block: int, tensor: str | int) -> int:
    tid = TENSOR_IDS[tensor] if isinstance(tensor, str) else int(tensor)
    return 1000 * int(config) + 10 * int(block) + tid


def generator(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def activations(M: int, K: int, seed: int) -> np.ndarray:
    """X ~ N(0, 1), fp32 [M, K]."""
    return generator(seed).standard_normal((M, K), dtype=np.float32)


def weights(N: int, K: int, seed: int, sigma: float = W_SIGMA) -> np.ndarray:
    """W ~ N(0, sigma^2), fp32 [N, K]."""
    w = generator(seed).standard_normal((N, K), dtype=np.float32)
    return (w * np.float32(sigma)).astype(np.float32)


def with_outliers(W: np.ndarray, seed: int, frac: float = 0.01, factor: float = 20.0,
                  span: int = 32) -> np.ndarray:
    """Copy of W where a seeded `frac` of the (row, span-of-32) cells has one
    seeded element multiplied by `factor` (the outlier stress of the M sweep)."""
    W = np.array(W, dtype=np.float32, copy=True)
    N, K = W.shape
    span = min(span, K)
    n_spans = K // span
    g = generator(seed + 7_919)
    cells = N * n_spans
    n_pick = max(1, int(round(frac * cells)))
    picked = g.choice(cells, size=n_pick, replace=False)
    elem = g.integers(0, span, size=n_pick)
    rows = picked // n_spans
    cols = (picked % n_spans) * span + elem
    W[rows, cols] *= np.float32(factor)
    return W


def projection_weights(config: int, block: int, name: str, outliers: bool = False) -> np.ndarray:
    """fp32 weights of one block projection group (rows of fused parts concatenated)."""
    spec = BLOCK_PROJECTIONS[name]
    parts = []
    for part in spec["parts"]:
        n, k = PART_SHAPES[part]
        s = seed_for(config, block, part)
        w = weights(n, k, s)
        if outliers:
            w = with_outliers(w, s)
        parts.append(w)
    return np.ascontiguousarray(np.concatenate(parts, axis=0))


def projection_input(config: int, block: int, name: str, M: int) -> np.ndarray:
    spec = BLOCK_PROJECTIONS[name]
    return activations(M, spec["K"], seed_for(config, block, spec["x"]))


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """Sorted seeded subset of n row indices of [0, M) that always holds 0 and M-1."""
    if M <= n:
        return np.arange(M, dtype=np.int64)
    if n < 2:
        raise ValueError(f"a row sample holds rows 0 and M-1, so n >= 2 (got n = {n})")
    g = generator(seed)
    inner = g.choice(np.arange(1, M - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, M - 1], inner]).astype(np.int64))
