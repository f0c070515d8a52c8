"""GPU parity of the layer in the paper's own parameterisation ("Recurrent
Transformer" paper page, paper §2 notation, §2.1, §2.2: per-head unit-RMS
queries and keys, softmax without a scale, RMS without eps, residual
branches scaled by 1/sqrt(L)) through the C ABI, against the fp64 oracle's
rt_layer_pages on the same bf16 inputs. Bar: max|gpu-ref|/max|ref| <= 2e-2
per output tensor (bf16 storage, fp32 accumulation)."""
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


@pytest.mark.parametrize("driver", ["graph", "persistent"])
@pytest.mark.parametrize("B,N,d,H,d_ff,L", [(3, 37, 128, 2, 256, 1), (2, 70, 128, 2, 256, 6),
                                            (130, 20, 192, 3, 320, 2), (1, 1, 64, 1, 64, 1)])
def test_pages_parameterisation_matches_oracle(rt, B, N, d, H, d_ff, L, driver):
    x, W = problem(B, N, d, H, d_ff, "bf16")
    z, K, V = rt.layer_forward_pages(to_device(x, "bf16"), {k: to_device(v, "bf16") for k, v in W.items()}, H, L,
                                     driver=driver)
    torch.cuda.synchronize()
    zr, Kr, Vr = O.rt_layer_pages(x, W, H, L)
    errs = (rel_err(to_np(z), zr), rel_err(to_np(K).transpose(1, 0, 2), Kr), rel_err(to_np(V).transpose(1, 0, 2), Vr))
    assert max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("driver", ["graph", "persistent"])
def test_pages_config_B64_N1024_d512_sampled(rt, driver):
    # the bf16 single-layer widths (B=64, N=1024, d=512, 8 heads of 64, d_ff=2048),
    # sampled sequences against the oracle; every fold kernel runs
    B, N, d, H, d_ff = 64, 1024, 512, 8, 2048
    x, W = problem(B, N, d, H, d_ff, "bf16")
    z, K, V = rt.layer_forward_pages(to_device(x, "bf16"), {k: to_device(v, "bf16") for k, v in W.items()}, H, 1,
                                     driver=driver)
    torch.cuda.synchronize()
    seqs = [0, 63]
    zr, Kr, Vr = O.rt_layer_pages(x[seqs], W, H, 1)
    errs = (rel_err(to_np(z)[seqs], zr), rel_err(to_np(K).transpose(1, 0, 2)[seqs], Kr),
            rel_err(to_np(V).transpose(1, 0, 2)[seqs], Vr))
    assert max(errs) <= TOL["bf16"], errs
