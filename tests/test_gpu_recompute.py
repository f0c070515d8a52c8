"""GPU parity of the activation-checkpoint recompute (RT paper §6.1: the
persistent pairs of every position rebuilt from the stored layer outputs in
one parallel step) through the C ABI, against the fp64 oracle's
recompute_kv on the same bf16 outputs, and against the pairs the forward
itself produced. Bar: max|gpu-ref|/max|ref| <= 2e-2 (bf16 storage, fp32
accumulation)."""
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
    R.lib()
    return R


@pytest.mark.parametrize("B,N,d", [(3, 37, 128), (5, 300, 256), (1, 1, 64), (130, 9, 192)])
def test_recompute_matches_oracle(rt, B, N, d):
    # stored outputs: any bf16 array of the layer's shape (the recompute is a
    # per-position map); here seeded N(0, 1) values on the bf16 grid
    rng = np.random.default_rng(B * 1000 + N + d)
    z = rtinputs.to_grid(rng.standard_normal((B, N, d)), "bf16")
    W = rtinputs.weights(0, d, 2 * d, dtype="bf16")
    ws = torch.zeros(rt.lib().rt_layer_recompute_workspace_bytes(B, N, d), dtype=torch.uint8, device="cuda")
    K, V = rt.recompute_kv(to_device(z, "bf16"), to_device(W["W_k"], "bf16"), to_device(W["W_v"], "bf16"),
                           workspace=ws)
    assert rt.sync_status(ws) == 0
    Kr, Vr = O.recompute_kv(z, W)
    assert rel_err(to_np(K).transpose(1, 0, 2), Kr) <= TOL["bf16"]
    assert rel_err(to_np(V).transpose(1, 0, 2), Vr) <= TOL["bf16"]


def test_recompute_reproduces_the_forward_pairs(rt):
    # the forward's own persistent pairs, rebuilt from its stored outputs
    B, N, d, H, d_ff = 8, 130, 256, 4, 512
    x, W = problem(B, N, d, H, d_ff, "bf16")
    Wd = {k: to_device(v, "bf16") for k, v in W.items()}
    z, K, V = rt.layer_forward(to_device(x, "bf16"), Wd, H)
    K2, V2 = rt.recompute_kv(z, Wd["W_k"], Wd["W_v"])
    torch.cuda.synchronize()
    assert rel_err(to_np(K2), to_np(K)) <= TOL["bf16"]
    assert rel_err(to_np(V2), to_np(V)) <= TOL["bf16"]
