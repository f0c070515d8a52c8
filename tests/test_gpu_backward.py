"""GPU parity of the layer's backward pass (RT paper §6.4; the exact
derivatives of the forward of paper §2.2, with the forward's intermediates
rebuilt from its stored inputs and outputs as in paper §6.1) through the C
ABI, against the oracle's fp64 gradient reference rt_layer_backward (itself
pinned by central finite differences). fp32 arithmetic; bar per gradient
tensor max|gpu-ref|/max|ref| <= 1e-4 with fp32 storage, <= 2e-2 with bf16
storage (inputs on the bf16 grid on both sides)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import rtinputs  # noqa: E402
from oracle import rt_oracle as O  # noqa: E402
from tests.parity_util import TOL, problem, rel_err, to_device, to_np  # noqa: E402

pytestmark = pytest.mark.gpu

NAMES = ("W_q", "W_k", "W_v", "W_o", "W_1", "W_2")


@pytest.fixture(scope="module")
def rt():
    from blocked_attention_b200 import rtlayer as R
    R.lib()
    return R


@pytest.mark.parametrize("dtype,B,N,d,H,d_ff,sigma", [
    ("f32", 2, 64, 64, 2, 256, 0.02), ("f32", 3, 17, 96, 3, 128, 0.02), ("f32", 2, 24, 64, 2, 128, 0.2),
    ("f32", 1, 1, 64, 1, 64, 0.02), ("bf16", 2, 40, 128, 2, 256, 0.02), ("bf16", 3, 33, 64, 1, 128, 0.2)])
def test_backward_matches_oracle_gradients(rt, dtype, B, N, d, H, d_ff, sigma):
    x, W = problem(B, N, d, H, d_ff, dtype, sigma=sigma)
    rng = np.random.default_rng(B * 100 + N)
    grid = lambda a: rtinputs.to_grid(a, dtype)
    dz = grid(rng.standard_normal((B, N, d)))
    dK = grid(rng.standard_normal((B, N, d)))
    dV = grid(rng.standard_normal((B, N, d)))
    dx_r, dW_r, (z, K, V) = O.rt_layer_backward(x, W, H, dz, dK, dV)
    # the stored forward outputs the backward starts from, on the storage grid
    z, K, V = grid(z), grid(K), grid(V)
    pm = lambda a: np.ascontiguousarray(a.transpose(1, 0, 2))        # [B, N, d] -> position-major
    dev = lambda a: to_device(a, dtype)
    dx, dW = rt.layer_backward(dev(x), {k: dev(v) for k, v in W.items()}, H, dev(z), dev(pm(K)), dev(pm(V)),
                               dev(dz), dev(pm(dK)), dev(pm(dV)))
    torch.cuda.synchronize()
    errs = {"dx": rel_err(to_np(dx), dx_r)}
    errs.update({n: rel_err(to_np(dW[n]), dW_r[n]) for n in NAMES})
    assert max(errs.values()) <= TOL[dtype], errs
