"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs. Bars: max|gpu-ref|/max|ref| <= 1e-4 (fp32 storage),
<= 2e-2 (bf16 storage, fp32 accumulation), per output tensor z, K, V."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import rtinputs  # noqa: E402
from oracle import rt_oracle as O  # noqa: E402
from tests.parity_util import TOL, problem, rel_err, to_device, to_np  # noqa: E402

pytestmark = pytest.mark.gpu

LOG2E = 1.0 / math.log(2.0)


@pytest.fixture(scope="module")
def rt():
    from blocked_attention_b200 import rtlayer
    rtlayer.lib()
    return rtlayer


def _weights_dev(W, dtype):
    return {k: to_device(v, dtype) for k, v in W.items()}


def _check_layer(rt, B, N, d, H, d_ff, dtype, schedule="blocked", driver="graph", sigma=0.02, seqs=None):
    x, W = problem(B, N, d, H, d_ff, dtype, sigma=sigma)
    z, K, V = rt.layer_forward(to_device(x, dtype), _weights_dev(W, dtype), H, schedule=schedule, driver=driver)
    torch.cuda.synchronize()
    sel = list(range(B)) if seqs is None else list(seqs)
    zr, Kr, Vr = O.rt_layer(x[sel], W, H)
    zg = to_np(z)[sel]
    Kg = to_np(K).transpose(1, 0, 2)[sel]
    Vg = to_np(V).transpose(1, 0, 2)[sel]
    errs = (rel_err(zg, zr), rel_err(Kg, Kr), rel_err(Vg, Vr))
    assert max(errs) <= TOL[dtype], errs
    return errs, (z, K, V)


# --------------------------------------------------------------------------
# components
# --------------------------------------------------------------------------
@pytest.mark.parametrize("M,Nout,Kd", [(128, 256, 64), (300, 192, 128), (64, 1024, 512), (1000, 96, 320),
                                       (2048, 3072, 1024), (1, 32, 64)])
def test_tcgen05_gemm_matches_fp64_matmul(rt, M, Nout, Kd):
    rng = np.random.default_rng(M + Nout + Kd)
    A = rtinputs.to_grid(rng.standard_normal((M, Kd)), "bf16")
    W = rtinputs.to_grid(rng.standard_normal((Nout, Kd)), "bf16")
    C = rt.gemm_bf16(to_device(A, "bf16"), to_device(W, "bf16"))
    torch.cuda.synchronize()
    ref = A @ W.T
    assert rel_err(to_np(C), ref) < 1e-5


@pytest.mark.parametrize("dtype,B,N,d", [("bf16", 3, 37, 128), ("bf16", 2, 300, 512), ("f32", 2, 64, 64),
                                         ("f32", 3, 17, 96)])
def test_batched_projection_matches_oracle(rt, dtype, B, N, d):
    x, W = problem(B, N, d, 2 if d % 64 == 0 else 3, 2 * d, dtype)
    Wqkv = np.concatenate([W["W_q"], W["W_k"], W["W_v"]], axis=0)
    qkv = rt.project_qkv(to_device(x, dtype), to_device(Wqkv, dtype))
    torch.cuda.synchronize()
    ref = O.rms(x) @ Wqkv.T                      # [B, N, 3d]
    got = to_np(qkv).transpose(1, 0, 2)          # position-major -> [B, N, 3d]
    assert rel_err(got, ref) <= (5e-3 if dtype == "bf16" else 1e-5)


@pytest.mark.parametrize("dtype,nk,nq,init_empty", [
    ("bf16", 1, 1, False), ("bf16", 2, 2, True), ("bf16", 8, 5, False),      # small-block kernel (nk <= 8)
    ("bf16", 8, 1, False), ("bf16", 3, 1, True), ("bf16", 5, 12, False),     # (query slots per pair 8 / 4 / 16)
    ("bf16", 4, 70, False), ("bf16", 8, 33, True),                           # (a pair's queries over 3 / 2 CTAs)
    ("bf16", 16, 16, False), ("bf16", 32, 7, False), ("bf16", 64, 64, True),  # mma.sync kernel
    ("bf16", 16, 40, False), ("bf16", 32, 70, True), ("bf16", 96, 65, False),  # (4 / 2 / 1 pairs per CTA)
    ("bf16", 48, 20, False), ("bf16", 12, 3, False), ("bf16", 27, 9, True),    # generic warp kernel (12, 27)
    ("bf16", 256, 100, False), ("bf16", 1024, 130, False),                     # tcgen05 kernels (nk % 128 == 0)
    ("bf16", 256, 256, False), ("bf16", 1024, 700, True), ("bf16", 256, 129, False),
    ("bf16", 128, 77, False), ("bf16", 128, 128, True), ("bf16", 512, 300, True), ("bf16", 384, 1, False),
    ("bf16", 40, 6, False),                                                      # generic warp kernel
    ("bf16", 2048, 300, False), ("bf16", 4096, 129, True),                     # the blocks of N >= 4096
    ("bf16", 1024, 100, False), ("bf16", 1024, 128, True),                     # one-tile tcgen05 kernel
    ("f32", 3, 4, False), ("f32", 16, 16, True), ("f32", 64, 33, False)])
def test_block_fold_matches_oracle(rt, dtype, nk, nq, init_empty):
    B, H, dh = 3, 2, 64 if dtype == "bf16" else 32
    d = H * dh
    npos = nk + nq + 2
    rng = np.random.default_rng(nk * 7 + nq)
    Q = rtinputs.to_grid(rng.standard_normal((npos, B, d)), dtype)
    Kc = rtinputs.to_grid(rng.standard_normal((npos, B, d)), dtype)
    Vc = rtinputs.to_grid(rng.standard_normal((npos, B, d)), dtype)
    scale = 1.0 / math.sqrt(dh)
    # prior accumulator state of the queries (natural-log units for the oracle)
    m0 = rng.standard_normal((npos, B, H)) * 2
    l0 = rng.uniform(0.5, 3.0, (npos, B, H))
    o0 = rng.standard_normal((npos, B, d))
    if init_empty:
        m0[:] = -np.inf; l0[:] = 0; o0[:] = 0
    k0, q0 = 1, 1 + nk
    mg = torch.tensor((m0 * LOG2E).astype(np.float32), device="cuda")
    lg = torch.tensor(l0.astype(np.float32), device="cuda")
    og = torch.tensor(o0.astype(np.float32), device="cuda")
    rt.block_fold(to_device(Q, dtype), to_device(Kc, dtype), to_device(Vc, dtype), mg, lg, og, H, dh, q0, nq, k0, nk)
    torch.cuda.synchronize()
    # oracle, per (b, h)
    qh = Q[q0:q0 + nq].reshape(nq, B, H, dh).transpose(1, 2, 0, 3)     # [B,H,nq,dh]
    kh = Kc[k0:k0 + nk].reshape(nk, B, H, dh).transpose(1, 2, 0, 3)
    vh = Vc[k0:k0 + nk].reshape(nk, B, H, dh).transpose(1, 2, 0, 3)
    mr = m0[q0:q0 + nq].transpose(1, 2, 0).copy()
    lr = l0[q0:q0 + nq].transpose(1, 2, 0).copy()
    orr = o0[q0:q0 + nq].reshape(nq, B, H, dh).transpose(1, 2, 0, 3).copy()
    mr, lr, orr = O.block_fold(qh, kh, vh, mr, lr, orr, scale)
    m_got = to_np(mg)[q0:q0 + nq].transpose(1, 2, 0) / LOG2E
    l_got = to_np(lg)[q0:q0 + nq].transpose(1, 2, 0)
    o_got = to_np(og)[q0:q0 + nq].reshape(nq, B, H, dh).transpose(1, 2, 0, 3)
    assert np.max(np.abs(m_got - mr)) < 1e-4 * max(1.0, np.max(np.abs(mr)))
    # compare normalised outputs and the normaliser. In bf16 the kernels round
    # the probabilities P to bf16 (unit roundoff 2^-9) before the PV product
    # while the normaliser sums them in fp32, so each normalised output
    # element is a convex combination of the block's v values with weights
    # off by at most 2^-9 relative: |error| <= 2^-9 * max|v| (+ fp32 sums).
    if dtype == "bf16":
        bound = 2.0 ** -9 * np.max(np.abs(Vc[k0:k0 + nk])) * 1.01 + 1e-5
        assert np.max(np.abs(o_got / l_got[..., None] - orr / lr[..., None])) <= bound
        assert rel_err(l_got, lr) < 2.0 ** -9 * 1.01
    else:
        assert rel_err(o_got / l_got[..., None], orr / lr[..., None]) < 1e-5
        assert rel_err(l_got, lr) < 1e-5
    # rows outside the query range are untouched
    untouched = np.ones(npos, bool); untouched[q0:q0 + nq] = False
    np.testing.assert_array_equal(to_np(og)[untouched], o0[untouched].astype(np.float32))


@pytest.mark.parametrize("nk,init_empty", [(256, False), (256, True), (384, False)])
def test_block_fold_many_items_per_cta(rt, nk, init_empty):
    # The two-tile tcgen05 fold with several (pair, 256-query) items per CTA
    # (1280 items over the SMs) and two or three 128-key chunks per item: each
    # item's merge must see every PV product of the item. Sampled pairs are
    # checked against the oracle with the bound of test_block_fold_matches_oracle.
    B, H, dh, nq = 64, 20, 64, 256
    d = H * dh
    npos = nk + nq + 2
    rng = np.random.default_rng(nk * 11 + int(init_empty))
    Q = rtinputs.to_grid(rng.standard_normal((npos, B, d)), "bf16")
    Kc = rtinputs.to_grid(rng.standard_normal((npos, B, d)), "bf16")
    Vc = rtinputs.to_grid(rng.standard_normal((npos, B, d)), "bf16")
    m0 = rng.standard_normal((npos, B, H)) * 2
    l0 = rng.uniform(0.5, 3.0, (npos, B, H))
    o0 = rng.standard_normal((npos, B, d))
    if init_empty:
        m0[:] = -np.inf; l0[:] = 0; o0[:] = 0
    k0, q0 = 1, 1 + nk
    mg = torch.tensor((m0 * LOG2E).astype(np.float32), device="cuda")
    lg = torch.tensor(l0.astype(np.float32), device="cuda")
    og = torch.tensor(o0.astype(np.float32), device="cuda")
    rt.block_fold(to_device(Q, "bf16"), to_device(Kc, "bf16"), to_device(Vc, "bf16"), mg, lg, og, H, dh,
                  q0, nq, k0, nk)
    torch.cuda.synchronize()
    m_all, l_all, o_all = to_np(mg) / LOG2E, to_np(lg), to_np(og)
    for pair in range(0, B * H, 37):
        b, h = divmod(pair, H)
        sl = slice(h * dh, (h + 1) * dh)
        v = Vc[k0:k0 + nk, b, sl]
        mr, lr, orr = O.block_fold(Q[q0:q0 + nq, b, sl], Kc[k0:k0 + nk, b, sl], v, m0[q0:q0 + nq, b, h].copy(),
                                   l0[q0:q0 + nq, b, h].copy(), o0[q0:q0 + nq, b, sl].copy(), 1.0 / math.sqrt(dh))
        m_got, l_got, o_got = m_all[q0:q0 + nq, b, h], l_all[q0:q0 + nq, b, h], o_all[q0:q0 + nq, b, sl]
        assert np.max(np.abs(m_got - mr)) < 1e-4 * max(1.0, np.max(np.abs(mr)))
        bound = 2.0 ** -9 * np.max(np.abs(v)) * 1.01 + 1e-5
        assert np.max(np.abs(o_got / l_got[:, None] - orr / lr[:, None])) <= bound, (b, h)
        assert rel_err(l_got, lr) < 2.0 ** -9 * 1.01


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------
@pytest.mark.parametrize("schedule", ["blocked", "naive"])
@pytest.mark.parametrize("driver", ["graph", "stream"])
def test_layer_f32_tiny_config(rt, schedule, driver):
    # B=2 sequences, N=64, d=64, H=2 heads of 32, d_ff=256, fp32
    _check_layer(rt, 2, 64, 64, 2, 256, "f32", schedule=schedule, driver=driver)


@pytest.mark.parametrize("driver", ["graph", "persistent"])
@pytest.mark.parametrize("B,N,d,H,d_ff", [(3, 37, 128, 2, 256), (5, 100, 192, 3, 320), (1, 1, 64, 1, 64),
                                          (2, 2, 64, 1, 128), (130, 20, 128, 2, 256)])
def test_layer_bf16_ragged_shapes(rt, B, N, d, H, d_ff, driver):
    _check_layer(rt, B, N, d, H, d_ff, "bf16", driver=driver)


def test_layer_f32_peaky_attention(rt):
    _check_layer(rt, 2, 48, 64, 2, 128, "f32", sigma=0.2)


def test_layer_bf16_peaky_attention(rt):
    _check_layer(rt, 2, 70, 128, 2, 256, "bf16", sigma=0.1)


@pytest.mark.parametrize("schedule", ["blocked", "naive"])
def test_layer_bf16_config_B64_N1024_d512(rt, schedule):
    # B=64, N=1024, d=512, H=8 heads of 64, d_ff=2048; sequences sampled for the oracle
    _check_layer(rt, 64, 1024, 512, 8, 2048, "bf16", schedule=schedule, seqs=[0, 31, 63])


def test_blocked_equals_naive_on_gpu(rt):
    B, N, d, H, d_ff = 4, 200, 128, 2, 256
    x, W = problem(B, N, d, H, d_ff, "bf16")
    xd, Wd = to_device(x, "bf16"), _weights_dev(W, "bf16")
    a = rt.layer_forward(xd, Wd, H, schedule="blocked")
    b = rt.layer_forward(xd, Wd, H, schedule="naive")
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert rel_err(to_np(u), to_np(v)) < 1e-2


def test_prefix_property_on_gpu(rt):
    B, N, d, H, d_ff = 3, 90, 128, 2, 256
    x, W = problem(B, N, d, H, d_ff, "f32")
    Wd = _weights_dev(W, "f32")
    z, K, V = rt.layer_forward(to_device(x, "f32"), Wd, H)
    zp, Kp, Vp = rt.layer_forward(to_device(x[:, :50].copy(), "f32"), Wd, H)
    torch.cuda.synchronize()
    assert rel_err(to_np(zp), to_np(z)[:, :50]) < 1e-6
    assert rel_err(to_np(Kp), to_np(K)[:50]) < 1e-6


def test_graph_replay_is_deterministic_and_matches_stream(rt):
    B, N, d, H, d_ff = 8, 130, 256, 4, 512
    x, W = problem(B, N, d, H, d_ff, "bf16")
    xd, Wd = to_device(x, "bf16"), _weights_dev(W, "bf16")
    ws = rt.alloc_workspace(rt.workspace_bytes(B, N, d, H, d_ff))
    outs = [torch.empty((B, N, d), dtype=torch.bfloat16, device="cuda"),
            torch.empty((N, B, d), dtype=torch.bfloat16, device="cuda"),
            torch.empty((N, B, d), dtype=torch.bfloat16, device="cuda")]
    rt.layer_forward(xd, Wd, H, out=outs, workspace=ws, driver="graph")
    first = [t.clone() for t in outs]
    rt.layer_forward(xd, Wd, H, out=outs, workspace=ws, driver="graph")     # cached graph replay
    assert rt.sync_status(ws) == 0
    for a, b in zip(first, outs):
        assert torch.equal(a, b)
    s = rt.layer_forward(xd, Wd, H, driver="stream")
    torch.cuda.synchronize()
    for a, b in zip(first, s):
        assert torch.equal(a, b)
    # the persistent step kernel: replays are bitwise equal too (its W_2
    # split partials are summed in split order), and it agrees with the
    # per-kernel path up to rounding order
    rt.layer_forward(xd, Wd, H, out=outs, workspace=ws, driver="persistent")
    pfirst = [t.clone() for t in outs]
    rt.layer_forward(xd, Wd, H, out=outs, workspace=ws, driver="persistent")
    assert rt.sync_status(ws) == 0
    for a, b, c in zip(pfirst, outs, first):
        assert torch.equal(a, b)
        assert rel_err(to_np(a), to_np(c)) < TOL["bf16"]


def test_host_buffer_entry_point(rt):
    B, N, d, H, d_ff = 4, 40, 128, 2, 256
    x, W = problem(B, N, d, H, d_ff, "bf16")
    xh = to_device(x, "bf16", device="cpu").pin_memory()
    Wh = {k: to_device(v, "bf16", device="cpu").pin_memory() for k, v in W.items()}
    out = [torch.empty((B, N, d), dtype=torch.bfloat16).pin_memory(),
           torch.empty((N, B, d), dtype=torch.bfloat16).pin_memory(),
           torch.empty((N, B, d), dtype=torch.bfloat16).pin_memory()]
    ws = rt.alloc_workspace(rt.host_workspace_bytes(B, N, d, H, d_ff))
    rt.layer_forward_host(xh, Wh, H, out, ws)
    torch.cuda.synchronize()
    zr, Kr, Vr = O.rt_layer(x, W, H)
    assert rel_err(to_np(out[0]), zr) < TOL["bf16"]
    assert rel_err(to_np(out[1]).transpose(1, 0, 2), Kr) < TOL["bf16"]
    assert rel_err(to_np(out[2]).transpose(1, 0, 2), Vr) < TOL["bf16"]


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("driver", ["graph", "stream", "persistent"])
def test_host_entry_matches_device_entry(rt, pinned, driver):
    # B=11 splits unevenly into the sequence chunks of the overlapped upload
    # and N=37 into its output ranges; pinned buffers take the overlapped
    # path, pageable ones the sequential one. Both must equal the
    # device-buffer entry point bit for bit.
    B, N, d, H, d_ff = 11, 37, 128, 2, 256
    x, W = problem(B, N, d, H, d_ff, "bf16")
    xd = to_device(x, "bf16")
    z0, K0, V0 = rt.layer_forward(xd, _weights_dev(W, "bf16"), H, driver=driver)

    def host(t):
        return t.pin_memory() if pinned else t

    xh = host(to_device(x, "bf16", device="cpu"))
    Wh = {k: host(to_device(v, "bf16", device="cpu")) for k, v in W.items()}
    out = [host(torch.full((B, N, d), 7.0, dtype=torch.bfloat16)),
           host(torch.full((N, B, d), 7.0, dtype=torch.bfloat16)),
           host(torch.full((N, B, d), 7.0, dtype=torch.bfloat16))]
    ws = rt.alloc_workspace(rt.host_workspace_bytes(B, N, d, H, d_ff))
    for _ in range(2):   # the second call replays the cached graph
        rt.layer_forward_host(xh, Wh, H, out, ws, driver=driver)
        torch.cuda.synchronize()
        assert rt.sync_status(ws) == 0
        assert torch.equal(out[0], z0.cpu())
        assert torch.equal(out[1], K0.cpu())
        assert torch.equal(out[2], V0.cpu())
        for t in out:
            t.fill_(7.0)


def test_stack_of_layers_with_embedding(rt):
    # reduced stack: vocab 500, d=128 (2 heads of 64), d_ff=256, 3 layers, B=3, N=33
    vocab, d, H, d_ff, B, N, L = 500, 128, 2, 256, 3, 33, 3
    E = rtinputs.embedding(0, vocab, d, dtype="bf16")
    ids = np.stack([rtinputs.token_ids(0, b, N, vocab) for b in range(B)])
    layers = [rtinputs.weights(0, d, d_ff, dtype="bf16", layer=i) for i in range(L)]
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    x = rt.embed_forward(torch.tensor(ids, device="cuda"), to_device(E, "bf16"), workspace=ws)
    kv = []
    for W in layers:
        x, K, V = rt.layer_forward(x, _weights_dev(W, "bf16"), H)
        kv.append((K, V))
    torch.cuda.synchronize()
    assert rt.sync_status(ws) == 0
    zr, kvr = O.rt_stack(ids, E, layers, H)
    assert rel_err(to_np(x), zr) < TOL["bf16"]
    for (K, V), (Kr, Vr) in zip(kv, kvr):
        assert rel_err(to_np(K).transpose(1, 0, 2), Kr) < TOL["bf16"]
        assert rel_err(to_np(V).transpose(1, 0, 2), Vr) < TOL["bf16"]


def test_embedding_out_of_range_id_is_reported(rt):
    E = to_device(rtinputs.embedding(0, 10, 64, dtype="bf16"), "bf16")
    ids = torch.tensor([[1, 2, 10]], dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    x = rt.embed_forward(ids, E, workspace=ws)
    assert rt.sync_status(ws) == rt.RT_ERR_INVALID_ARG
    assert torch.count_nonzero(x[0, 2]) == 0


def test_bounded_wait_reports_timeout_and_context_stays_usable(rt):
    # a barrier nothing arrives on: the wait gives up after 1 ms and reports it
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    rt.selftest_wait_timeout(1_000_000, ws)
    assert rt.sync_status(ws) == rt.RT_ERR_TIMEOUT
    assert rt.sync_status(ws) == 0                       # the word was cleared
    # the context is still usable: a normal forward runs and passes parity
    _check_layer(rt, 2, 20, 128, 2, 256, "bf16")


def test_component_entry_point_reports_through_its_error_word(rt):
    # the error word a component entry point's tensor-core kernel records into
    # is the one rt_layer_sync_status reads: a timeout recorded there (by the
    # bounded-wait self-test) surfaces, is cleared, and a GEMM enqueued on the
    # same word afterwards completes with the word still clear
    err = torch.zeros(256, dtype=torch.uint8, device="cuda")
    rt.selftest_wait_timeout(1_000_000, err)
    assert rt.sync_status(err) == rt.RT_ERR_TIMEOUT
    rng = np.random.default_rng(5)
    A = rtinputs.to_grid(rng.standard_normal((300, 256)), "bf16")
    W = rtinputs.to_grid(rng.standard_normal((192, 256)), "bf16")
    C = rt.gemm_bf16(to_device(A, "bf16"), to_device(W, "bf16"), err=err)
    assert rt.sync_status(err) == 0
    assert rel_err(to_np(C), A @ W.T) < 1e-5


@pytest.mark.parametrize("nk,nq", [(1024, 64), (1024, 300)])
def test_tcgen05_fold_with_several_items_per_cta(rt, nk, nq):
    # 28 sequences x 16 heads: every persistent CTA of the tcgen05 folds takes
    # three or more (pair, query tile) items, so the query buffers are
    # refilled (the buffer release by the softmax warps is exercised); the
    # error word must stay clear and sampled pairs match the oracle
    B, H, dh = 28, 16, 64
    d = H * dh
    npos = nk + nq
    rng = np.random.default_rng(nk + nq)
    Q = rtinputs.to_grid(rng.standard_normal((npos, B, d)), "bf16")
    Kc = rtinputs.to_grid(rng.standard_normal((npos, B, d)), "bf16")
    Vc = rtinputs.to_grid(rng.standard_normal((npos, B, d)), "bf16")
    mg = torch.full((npos, B, H), -float("inf"), device="cuda")
    lg = torch.zeros((npos, B, H), device="cuda")
    og = torch.zeros((npos, B, d), device="cuda")
    err = torch.zeros(256, dtype=torch.uint8, device="cuda")
    rt.block_fold(to_device(Q, "bf16"), to_device(Kc, "bf16"), to_device(Vc, "bf16"), mg, lg, og, H, dh, nk, nq, 0, nk,
                  err=err)
    assert rt.sync_status(err) == 0
    sb = [0, 27]
    qh = Q[nk:, sb].reshape(nq, 2, H, dh).transpose(1, 2, 0, 3)
    kh = Kc[:nk, sb].reshape(nk, 2, H, dh).transpose(1, 2, 0, 3)
    vh = Vc[:nk, sb].reshape(nk, 2, H, dh).transpose(1, 2, 0, 3)
    mr = np.full((2, H, nq), -np.inf)
    lr = np.zeros((2, H, nq))
    orr = np.zeros((2, H, nq, dh))
    mr, lr, orr = O.block_fold(qh, kh, vh, mr, lr, orr, 1.0 / math.sqrt(dh))
    l_got = to_np(lg)[nk:, sb].transpose(1, 2, 0)
    o_got = to_np(og)[nk:, sb].reshape(nq, 2, H, dh).transpose(1, 2, 0, 3)
    bound = 2.0 ** -9 * np.max(np.abs(Vc[:nk, sb])) * 1.01 + 1e-5
    assert np.max(np.abs(o_got / l_got[..., None] - orr / lr[..., None])) <= bound
