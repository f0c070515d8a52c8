"""GPU parity of the block-wise (chunked) recurrence (RT paper §9 / notes §8
name it as the depth-for-speed trade-off; the reading -- persistent pairs
visible from the next chunk on, causal temporary pairs inside a chunk -- is
the oracle's rt_layer_chunked, pinned at both ends) through the C ABI, on
the same bf16 inputs. Bar: max|gpu-ref|/max|ref| <= 2e-2 per output tensor."""
import pytest

torch = pytest.importorskip("torch")

from oracle import rt_oracle as O  # noqa: E402
from tests.parity_util import TOL, problem, rel_err, to_device, to_np  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    from blocked_attention_b200 import rtlayer as R
    R.lib()
    return R


@pytest.mark.parametrize("B,N,d,H,d_ff,C", [(3, 37, 128, 2, 256, 1), (3, 37, 128, 2, 256, 3),
                                            (2, 100, 128, 2, 256, 16), (130, 20, 192, 3, 320, 4),
                                            (2, 30, 128, 2, 256, 30), (2, 30, 128, 2, 256, 64)])
def test_chunked_recurrence_matches_oracle(rt, B, N, d, H, d_ff, C):
    x, W = problem(B, N, d, H, d_ff, "bf16")
    z, K, V = rt.layer_forward_chunked(to_device(x, "bf16"), {k: to_device(v, "bf16") for k, v in W.items()}, H, C)
    torch.cuda.synchronize()
    zr, Kr, Vr = O.rt_layer_chunked(x, W, H, C)
    errs = (rel_err(to_np(z), zr), rel_err(to_np(K).transpose(1, 0, 2), Kr), rel_err(to_np(V).transpose(1, 0, 2), Vr))
    assert max(errs) <= TOL["bf16"], errs


def test_chunks_of_one_match_the_layer_forward(rt):
    B, N, d, H, d_ff = 4, 70, 128, 2, 256
    x, W = problem(B, N, d, H, d_ff, "bf16")
    Wd = {k: to_device(v, "bf16") for k, v in W.items()}
    a = rt.layer_forward_chunked(to_device(x, "bf16"), Wd, H, 1)
    b = rt.layer_forward(to_device(x, "bf16"), Wd, H)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert rel_err(to_np(u), to_np(v)) < 1e-2
