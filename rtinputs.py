"""Seeded synthetic inputs for the Recurrent Transformer (RT) layer.

This module is the ONLY code shared by the CPU oracle side and the CUDA side.
It draws numbers and rounds them to the storage grid; it holds none of the
layer's arithmetic.

Generator: numpy's Philox4x32-10 counter-based bit generator (Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3", SC'11), one independent stream
per (seed, tensor id, sequence index), keyed through numpy's SeedSequence.
Each sequence b of x has its own stream, so a sampled subset of sequences can
be regenerated on its own (sequences of an RT layer never interact).

Workload recipe (the pages' single-layer latency setting: batch 512, width
1024, 16 heads; no dataset is used because the layer's cost depends only on
shapes): x ~ N(0, 1); every weight ~ N(0, sigma^2) with sigma = 0.02; no
biases; token ids uniform in [0, vocab).
"""
from __future__ import annotations

import numpy as np

# Stream ids, one per tensor.
_TID = {"W_q": 1, "W_k": 2, "W_v": 3, "W_o": 4, "W_1": 5, "W_2": 6,
        "x": 7, "E": 8, "ids": 9}

WEIGHT_NAMES = ("W_q", "W_k", "W_v", "W_o", "W_1", "W_2")


def _stream(seed: int, tid: int, sub: int = 0, layer: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed), int(tid), int(sub), int(layer)])
    return np.random.Generator(np.random.Philox(ss))


# --------------------------------------------------------------------------
# storage grids
# --------------------------------------------------------------------------
def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (round-to-nearest-even via fp32) and return the raw
    16-bit patterns as uint16."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    u = (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16))
    return u.view(np.float32).astype(np.float64)


def to_grid(a: np.ndarray, dtype: str) -> np.ndarray:
    """Values of `a` rounded to the storage grid of `dtype` ('f32' or 'bf16'),
    returned as float64 so that the oracle consumes exactly what the GPU gets."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f64(bf16_bits(a))
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# tensors
# --------------------------------------------------------------------------
def weights(seed: int, d: int, d_ff: int, sigma: float = 0.02,
            dtype: str = "f32", layer: int = 0) -> dict[str, np.ndarray]:
    """Weights in nn.Linear orientation [out][in]: W_q, W_k, W_v, W_o [d][d],
    W_1 [d_ff][d], W_2 [d][d_ff]; float64 values on the `dtype` grid."""
    shapes = {"W_q": (d, d), "W_k": (d, d), "W_v": (d, d), "W_o": (d, d),
              "W_1": (d_ff, d), "W_2": (d, d_ff)}
    out = {}
    for name in WEIGHT_NAMES:
        g = _stream(seed, _TID[name], 0, layer)
        out[name] = to_grid(g.standard_normal(shapes[name]) * sigma, dtype)
    return out


def x_seq(seed: int, b: int, N: int, d: int, dtype: str = "f32") -> np.ndarray:
    """Layer input of sequence b: [N][d] ~ N(0, 1), on the `dtype` grid."""
    g = _stream(seed, _TID["x"], b)
    return to_grid(g.standard_normal((N, d)), dtype)


def x_batch(seed: int, seqs, N: int, d: int, dtype: str = "f32") -> np.ndarray:
    """Stack of x_seq for the sequence indices in `seqs`: [len(seqs)][N][d]."""
    return np.stack([x_seq(seed, b, N, d, dtype) for b in seqs])


def embedding(seed: int, vocab: int, d: int, sigma: float = 0.02,
              dtype: str = "bf16") -> np.ndarray:
    g = _stream(seed, _TID["E"])
    return to_grid(g.standard_normal((vocab, d)) * sigma, dtype)


def token_ids(seed: int, b: int, N: int, vocab: int) -> np.ndarray:
    g = _stream(seed, _TID["ids"], b)
    return g.integers(0, vocab, size=N, dtype=np.int64).astype(np.int32)
