"""The no-allocation projection entry point against the allocating one.

rt_project_qkv_noalloc serves callers that cannot allocate device memory
where they call the library (runtimes that plan all device memory at
start-up, code running while another framework's caching allocator holds the
free memory, latency-critical loops): its per-row scratch lives in a fixed
array inside the library. This file is collected last on purpose.

Both entry points run the same kernels with the same tile choice, so their
outputs must agree bit for bit. Two calls in a row with different shapes
check that the shared array, which keeps the previous call's contents, does
not leak into the next result; the largest size the array allows (B*N =
2^20 rows) writes and reads its last row.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from tests.parity_util import problem, to_device  # noqa: E402

pytestmark = pytest.mark.gpu


def _inputs(B, N, d, seed):
    x, W = problem(B, N, d, 2, 2 * d, "bf16", seed=seed)
    Wqkv = np.concatenate([W["W_q"], W["W_k"], W["W_v"]], axis=0)
    return to_device(x, "bf16"), to_device(Wqkv, "bf16")


def _check_against_allocating(R, x, Wqkv):
    B, N, d = x.shape
    ref = R.project_qkv(x, Wqkv)
    out = torch.full((N, B, 3 * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    R.project_qkv_noalloc(x, Wqkv, out)
    assert R.project_qkv_noalloc_status() == R.RT_OK
    assert torch.equal(out, ref)


def test_noalloc_projection_matches_allocating_entry_point_twice():
    from blocked_attention_b200 import rtlayer as R
    R.lib()
    # the larger shape first, then a smaller one whose rows were written by call 1
    for B, N, d, seed in ((6, 300, 256, 1), (3, 37, 128, 2)):
        _check_against_allocating(R, *_inputs(B, N, d, seed))


def test_noalloc_projection_at_the_array_limit():
    from blocked_attention_b200 import rtlayer as R
    B, N, d = 1024, 1024, 64          # B*N = 2^20 rows: every row of the array
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    x = torch.randn((B, N, d), generator=g, device="cuda", dtype=torch.bfloat16)
    Wqkv = (torch.randn((3 * d, d), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    _check_against_allocating(R, x, Wqkv)


def test_noalloc_projection_rejects_sizes_beyond_its_array():
    from blocked_attention_b200 import rtlayer as R
    x = torch.empty((1, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.empty((192, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, dtype=torch.bfloat16, device="cuda")
    # B*N = 2^20 + 1 rows: refused on the host before anything is enqueued
    rc = R.lib().rt_project_qkv_noalloc(R._ptr(x), R._ptr(w), 1025, 1024, 64, R._ptr(out), None)
    assert rc == R.RT_ERR_WORKSPACE
