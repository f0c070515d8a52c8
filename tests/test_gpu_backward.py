"""GPU parity of the layer's backward pass (RT paper §6.4; the exact
derivatives of the forward of paper §2.2, with the forward's intermediates
rebuilt from its stored inputs and outputs as in paper §6.1) through the C
ABI, against the oracle's fp64 gradient reference rt_layer_backward (itself
pinned by central finite differences). fp32 storage and arithmetic; bar:
max|gpu-ref|/max|ref| <= 1e-4 per gradient tensor."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import rt_oracle as O  # noqa: E402
from tests.parity_util import TOL, problem, rel_err, to_device, to_np  # noqa: E402

pytestmark = pytest.mark.gpu

NAMES = ("W_q", "W_k", "W_v", "W_o", "W_1", "W_2")


@pytest.fixture(scope="module")
def rt():
    from blocked_attention_b200 import rtlayer as R
    R.lib()
    return R


@pytest.mark.parametrize("B,N,d,H,d_ff,sigma", [(2, 64, 64, 2, 256, 0.02), (3, 17, 96, 3, 128, 0.02),
                                                (2, 24, 64, 2, 128, 0.2), (1, 1, 64, 1, 64, 0.02)])
def test_backward_matches_oracle_gradients(rt, B, N, d, H, d_ff, sigma):
    x, W = problem(B, N, d, H, d_ff, "f32", sigma=sigma)
    rng = np.random.default_rng(B * 100 + N)
    dz = rng.standard_normal((B, N, d))
    dK = rng.standard_normal((B, N, d))
    dV = rng.standard_normal((B, N, d))
    dx_r, dW_r, (z, K, V) = O.rt_layer_backward(x, W, H, dz, dK, dV)
    pm = lambda a: np.ascontiguousarray(a.transpose(1, 0, 2))        # [B, N, d] -> position-major
    dx, dW = rt.layer_backward(to_device(x, "f32"), {k: to_device(v, "f32") for k, v in W.items()}, H,
                               to_device(z, "f32"), to_device(pm(K), "f32"), to_device(pm(V), "f32"),
                               to_device(dz, "f32"), to_device(pm(dK), "f32"), to_device(pm(dV), "f32"))
    torch.cuda.synchronize()
    errs = {"dx": rel_err(to_np(dx), dx_r)}
    errs.update({n: rel_err(to_np(dW[n]), dW_r[n]) for n in NAMES})
    assert max(errs.values()) <= TOL["f32"], errs
