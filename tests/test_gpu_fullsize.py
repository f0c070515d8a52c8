"""Full-size parity in the launch configuration the benchmark times.

Sequences of an RT layer never interact, so the oracle can check sampled
sequences of a full batch exactly: the sampled sequences' inputs come from the
seeded generator (rtinputs), the other sequences are filled on the device with
N(0, 1) values. Bar: 2e-2 (bf16 storage, fp32 accumulation) per tensor."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import rtinputs  # noqa: E402
from oracle import rt_oracle as O  # noqa: E402
from tests.parity_util import TOL, rel_err, to_device, to_np  # noqa: E402

pytestmark = pytest.mark.gpu


def _filled_batch(B, N, d, seqs, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    x = torch.randn((B, N, d), generator=g, device="cuda", dtype=torch.bfloat16)
    xs = rtinputs.x_batch(seed, seqs, N, d, dtype="bf16")
    for i, b in enumerate(seqs):
        x[b] = to_device(xs[i], "bf16")
    return x, xs


@pytest.mark.parametrize("driver", ["graph", "persistent"])
def test_headline_config_sampled_sequences(driver):
    from blocked_attention_b200 import rtlayer as R
    B, N, d, H, dff = 512, 2048, 1024, 16, 4096
    seqs = [0, 511]
    W = rtinputs.weights(0, d, dff, dtype="bf16")
    x, xs = _filled_batch(B, N, d, seqs, 0)
    z, K, V = R.layer_forward(x, {k: to_device(v, "bf16") for k, v in W.items()}, H, driver=driver)
    torch.cuda.synchronize()
    zg, Kg, Vg = to_np(z[seqs]), to_np(K[:, seqs]).transpose(1, 0, 2), to_np(V[:, seqs]).transpose(1, 0, 2)
    del x, z, K, V
    zr, Kr, Vr = O.rt_layer(xs, W, H)
    errs = rel_err(zg, zr), rel_err(Kg, Kr), rel_err(Vg, Vr)
    assert max(errs) <= TOL["bf16"], errs


def test_long_sequence_exercises_blocks_of_2048_keys():
    # N = 4096 at the headline widths: the fold of step 2048 folds a block of
    # 2048 keys into 2048 queries (and step 1024 one of 1024), the block sizes
    # of the sequence-length sweep's longer runs. One sequence is checked
    # against the oracle; the other is filled on the device.
    from blocked_attention_b200 import rtlayer as R
    B, N, d, H, dff = 2, 4096, 1024, 16, 4096
    seqs = [1]
    W = rtinputs.weights(0, d, dff, dtype="bf16")
    x, xs = _filled_batch(B, N, d, seqs, 0)
    z, K, V = R.layer_forward(x, {k: to_device(v, "bf16") for k, v in W.items()}, H, driver="graph")
    torch.cuda.synchronize()
    zg, Kg, Vg = to_np(z[seqs]), to_np(K[:, seqs]).transpose(1, 0, 2), to_np(V[:, seqs]).transpose(1, 0, 2)
    zr, Kr, Vr = O.rt_layer(xs, W, H)
    errs = rel_err(zg, zr), rel_err(Kg, Kr), rel_err(Vg, Vr)
    assert max(errs) <= TOL["bf16"], errs


def test_stack_config_sampled_sequence():
    # 6 layers, d=1280 (20 heads of 64), d_ff=5120, vocab 32000, B=64, N=2048
    from blocked_attention_b200 import rtlayer as R
    B, N, d, H, dff, L, vocab = 64, 2048, 1280, 20, 5120, 6, 32000
    seq = 5
    E = rtinputs.embedding(0, vocab, d, dtype="bf16")
    ids = np.stack([rtinputs.token_ids(0, b, N, vocab) for b in range(B)])
    layers = [rtinputs.weights(0, d, dff, dtype="bf16", layer=i) for i in range(L)]
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    x = R.embed_forward(torch.tensor(ids, device="cuda"), to_device(E, "bf16"), workspace=ws)
    kv = []
    for W in layers:
        x, K, V = R.layer_forward(x, {k: to_device(v, "bf16") for k, v in W.items()}, H)
        kv.append((to_np(K[:, seq]), to_np(V[:, seq])))
    torch.cuda.synchronize()
    assert R.sync_status(ws) == 0
    zg = to_np(x[seq])
    zr, kvr = O.rt_stack(ids[seq:seq + 1], E, layers, H)
    assert rel_err(zg, zr[0]) <= TOL["bf16"]
    for (Kg, Vg), (Kr, Vr) in zip(kv, kvr):
        assert rel_err(Kg, Kr[0]) <= TOL["bf16"]
        assert rel_err(Vg, Vr[0]) <= TOL["bf16"]
