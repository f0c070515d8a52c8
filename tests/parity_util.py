"""Shared helpers of the parity tests: seeded problems (from rtinputs) on both
sides, oracle runs on sampled sequences, and the error metric.

Error metric (per output tensor): max |gpu - ref| / max |ref|; where the
reference is identically zero (for example the gradients of W_q and W_k of a
one-token sequence, whose single softmax weight is constant) the metric is
the absolute max |gpu|.
Bars: 1e-4 for the fp32 storage mode, 2e-2 for bf16 storage with fp32
accumulation."""
from __future__ import annotations

import numpy as np

import rtinputs

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    diff = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return diff / scale if scale > 0.0 else diff


def torch_dtype(dtype: str):
    import torch
    return torch.float32 if dtype == "f32" else torch.bfloat16


def to_device(a: np.ndarray, dtype: str, device="cuda"):
    """fp64 values on the storage grid -> torch tensor of the storage type
    (exact: the values are already representable)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device=device, dtype=torch_dtype(dtype))


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def problem(B, N, d, H, d_ff, dtype, seed=0, sigma=0.02, seqs=None, layer=0):
    """Weights and x for the sequences `seqs` (default all B) as fp64 arrays on
    the storage grid."""
    W = rtinputs.weights(seed, d, d_ff, sigma=sigma, dtype=dtype, layer=layer)
    seqs = list(range(B)) if seqs is None else list(seqs)
    x = rtinputs.x_batch(seed, seqs, N, d, dtype=dtype)
    return x, W
