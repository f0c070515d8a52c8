"""GPU parity of the autoregressive decode step (RT paper §7.3) through the C
ABI: against the fp64 oracle's decode step on identical inputs (the cache
rounded to bf16 as the GPU holds it), and against the GPU's own
whole-sequence forward at the same position. Bar: max|gpu-ref|/max|ref| <=
2e-2 per output (bf16 storage, fp32 accumulation)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import rtinputs  # noqa: E402
from oracle import rt_oracle as O  # noqa: E402
from tests.parity_util import TOL, problem, rel_err, to_device, to_np  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    from blocked_attention_b200 import rtlayer as R
    return R


def _wdev(W):
    return {k: to_device(v, "bf16") for k, v in W.items()}


@pytest.mark.parametrize("B,t,cap,sigma", [(3, 1, 4, 0.02), (3, 2, 2, 0.02), (5, 17, 40, 0.02),
                                           (2, 40, 40, 0.2), (130, 33, 33, 0.02)])
def test_decode_step_matches_oracle_step(rt, B, t, cap, sigma):
    d, H, d_ff = 128, 2, 256
    x, W = problem(B, t, d, H, d_ff, "bf16", sigma=sigma)
    # a cache of persistent pairs for positions 1..t-1: the oracle's own, on the bf16 grid
    _, K, V = O.rt_layer(x, W, H)
    Kc = rtinputs.to_grid(K[:, :t - 1], "bf16")          # [B, t-1, d]
    Vc = rtinputs.to_grid(V[:, :t - 1], "bf16")
    zr, kr, vr = O.rt_decode_step(x[:, t - 1], W, H, Kc, Vc)
    K_dev = torch.zeros((cap, B, d), dtype=torch.bfloat16, device="cuda")
    V_dev = torch.zeros((cap, B, d), dtype=torch.bfloat16, device="cuda")
    K_dev[:t - 1] = to_device(Kc.transpose(1, 0, 2), "bf16")
    V_dev[:t - 1] = to_device(Vc.transpose(1, 0, 2), "bf16")
    sentinel = K_dev[t:].clone()
    ws = rt.alloc_workspace(rt.decode_workspace_bytes(B, d, H, d_ff))
    z = rt.layer_decode_step(to_device(x[:, t - 1], "bf16"), _wdev(W), H, t, K_dev, V_dev, workspace=ws)
    torch.cuda.synchronize()
    assert rt.sync_status(ws) == 0
    assert rel_err(to_np(z), zr) <= TOL["bf16"]
    assert rel_err(to_np(K_dev[t - 1]), kr) <= TOL["bf16"]
    assert rel_err(to_np(V_dev[t - 1]), vr) <= TOL["bf16"]
    # earlier rows unchanged, later rows untouched
    assert torch.equal(K_dev[:t - 1], to_device(Kc.transpose(1, 0, 2), "bf16"))
    assert torch.equal(K_dev[t:], sentinel)


def test_decode_continues_the_gpu_forward(rt):
    # the whole-sequence forward of positions 1..N-1, then one decode step for
    # position N, against the whole-sequence forward of 1..N at position N
    B, N, d, H, d_ff = 4, 24, 128, 2, 256
    x, W = problem(B, N, d, H, d_ff, "bf16")
    Wd = _wdev(W)
    xd = to_device(x, "bf16")
    z_all, K_all, V_all = rt.layer_forward(xd, Wd, H)
    _, K_pre, V_pre = rt.layer_forward(xd[:, :N - 1].contiguous(), Wd, H)
    K_dev = torch.zeros((N, B, d), dtype=torch.bfloat16, device="cuda")
    V_dev = torch.zeros_like(K_dev)
    K_dev[:N - 1] = K_pre
    V_dev[:N - 1] = V_pre
    z = rt.layer_decode_step(xd[:, N - 1].contiguous(), Wd, H, N, K_dev, V_dev)
    torch.cuda.synchronize()
    assert rel_err(to_np(z), to_np(z_all[:, N - 1])) <= TOL["bf16"]
    assert rel_err(to_np(K_dev[N - 1]), to_np(K_all[N - 1])) <= TOL["bf16"]
    assert rel_err(to_np(V_dev[N - 1]), to_np(V_all[N - 1])) <= TOL["bf16"]
    # and against the oracle at that position
    zr, Kr, Vr = O.rt_layer(x, W, H)
    assert rel_err(to_np(z), zr[:, N - 1]) <= TOL["bf16"]
    assert rel_err(to_np(K_dev[N - 1]), Kr[:, N - 1]) <= TOL["bf16"]
