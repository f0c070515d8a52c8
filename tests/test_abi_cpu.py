"""The C ABI on the host: the library loads, exports every function the header
declares, and its host-side logic (validation, workspace plan, launch count)
behaves as documented. No kernel runs here."""
import ctypes
import os
import re

import pytest

from blocked_attention_b200 import build as B
from blocked_attention_b200 import rtlayer as R

HEADER = os.path.join(B.INCLUDE, "rtlayer.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return R.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rt_[a-z0-9_]+)\s*\(", text)))


def test_header_declarations_are_all_exported(L):
    names = _declared()
    assert "rt_layer_forward" in names and len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in rtlayer.h but not exported"
    assert set(R.EXPORTS) == set(names)


def test_version_and_status_strings(L):
    assert L.rt_version() >= 100
    for s in range(-6, 1):
        assert R.status_string(s) not in ("", "unknown status")
    assert R.status_string(-99) == "unknown status"


def test_cuda_error_detail(L):
    # no CUDA-runtime failure has happened on this thread yet
    assert L.rt_last_cuda_error() == 0
    assert L.rt_cuda_error_string(0).decode() == "no error"
    # any code maps to some text (never NULL), including unknown ones
    assert L.rt_cuda_error_string(2).decode()
    assert L.rt_cuda_error_string(123456).decode()
    # the binding's exception carries the CUDA error only for RT_ERR_CUDA
    e = R.RTError("rt_layer_forward", R.RT_ERR_INVALID_ARG)
    assert e.cuda_error == 0 and "CUDA error" not in str(e)
    e = R.RTError("rt_layer_forward", R.RT_ERR_CUDA)
    assert "CUDA error 0" in str(e)


def test_decode_step_validation_happens_before_any_launch(L):
    B, d, H, d_ff = 4, 128, 2, 256
    assert L.rt_layer_decode_workspace_bytes(B, d, H, d_ff) > 0
    assert L.rt_layer_decode_workspace_bytes(B, 96, 2, d_ff) == 0    # d_h = 48: bf16 path needs 64
    assert L.rt_layer_decode_workspace_bytes(0, d, H, d_ff) == 0
    p = ctypes.c_void_p(1 << 40)   # never dereferenced: every call below fails validation first

    def call(t, cap, Bv=B, dv=d, ws_bytes=1 << 30):
        return L.rt_layer_decode_step(*([p] * 7), Bv, t, cap, dv, H, d_ff, p, p, p, p,
                                      ctypes.c_size_t(ws_bytes), None)
    assert call(0, 8) == R.RT_ERR_INVALID_ARG          # positions are 1-based
    assert call(9, 8) == R.RT_ERR_INVALID_ARG          # beyond the cache capacity
    assert call(1, 8, Bv=0) == R.RT_ERR_INVALID_ARG
    assert call(1, 8, dv=96) == R.RT_ERR_UNSUPPORTED
    assert call(1, 8, ws_bytes=16) == R.RT_ERR_WORKSPACE
    assert L.rt_layer_decode_step(None, *([p] * 6), B, 1, 8, d, H, d_ff, p, p, p, p,
                                  ctypes.c_size_t(1 << 30), None) == R.RT_ERR_INVALID_ARG


def test_workspace_plan(L):
    bf, f32 = R.RT_BF16, R.RT_F32
    ws = L.rt_layer_workspace_bytes
    assert ws(512, 2048, 1024, 16, 4096, bf, 0) > 0
    # bf16 storage needs d_h = 64
    assert ws(2, 64, 64, 2, 256, bf, 0) == 0
    assert ws(2, 64, 64, 2, 256, f32, 0) > 0
    assert ws(2, 64, 64, 3, 256, f32, 0) == 0          # d % H != 0
    assert ws(0, 64, 64, 2, 256, f32, 0) == 0
    assert ws(2, 64, 64, 2, 256, 7, 0) == 0             # bad dtype
    # the blocked schedule keeps (m, l, o) per position; the naive one does not
    assert ws(8, 256, 512, 8, 1024, bf, 0) > ws(8, 256, 512, 8, 1024, bf, 1)
    # headline: q/k~/v~ (3 x 2.1 GB) + o (4.3 GB) + m, l dominate
    hb = ws(512, 2048, 1024, 16, 4096, bf, 0)
    assert 10.5e9 < hb < 11.5e9
    assert L.rt_layer_host_workspace_bytes(512, 2048, 1024, 16, 4096, bf, 0) > hb + 4 * 2.1e9


def _step_kernel_launches(N):
    # the persistent step kernel runs segments of steps ending at a position t
    # whose fold has >= 16 keys (that fold follows as its own launch) or t = N
    segments = sum(1 for t in range(1, N + 1) if t == N or (t & -t) >= 16)
    big_folds = sum(1 for t in range(1, N) if (t & -t) >= 16)
    return segments + big_folds


def test_launch_count_matches_schedule(L):
    G, S, P = R.RT_DRIVER_GRAPH, R.RT_DRIVER_STREAM, R.RT_DRIVER_PERSISTENT
    for N in (1, 2, 7, 16, 17, 64, 2048):
        folds = sum(1 for t in range(1, N + 1) if min(t & -t, N - t) > 0)
        # per-kernel drivers: inv_rms + projection + finalise(position 1) + 4
        # GEMMs per step + one fold per step that has one
        assert L.rt_layer_launch_count(4, N, 512, 8, 1024, R.RT_BF16, 0, G) == 3 + 4 * N + folds
        assert L.rt_layer_launch_count(4, N, 512, 8, 1024, R.RT_BF16, 0, S) == 3 + 4 * N + folds
        # persistent: the step kernel's segments + the folds of >= 16 keys between them
        assert L.rt_layer_launch_count(4, N, 512, 8, 1024, R.RT_BF16, 0, P) == 3 + _step_kernel_launches(N)
        assert L.rt_layer_launch_count(4, N, 512, 8, 1024, R.RT_BF16, 1, G) == 2 + 5 * N
        assert L.rt_layer_launch_count(4, N, 512, 8, 1024, R.RT_BF16, 1, P) == -1   # blocked only
    # the headline: 2047 folds; persistent: 128 segments and 127 large folds
    assert L.rt_layer_launch_count(512, 2048, 1024, 16, 4096, R.RT_BF16, 0, G) == 3 + 4 * 2048 + 2047
    assert L.rt_layer_launch_count(512, 2048, 1024, 16, 4096, R.RT_BF16, 0, P) == 3 + 128 + 127
    assert L.rt_layer_launch_count(4, 8, 64, 2, 256, R.RT_F32, 0, G) == 2 + 8 * 8 + 7
    assert L.rt_layer_launch_count(4, 8, 64, 2, 256, R.RT_F32, 0, P) == -1
    assert L.rt_layer_launch_count(4, 8, 64, 2, 256, R.RT_F32, 0, 3) == -1
    assert L.rt_layer_launch_count(4, 8, 64, 2, 256, R.RT_BF16, 0, R.RT_DRIVER_GRAPH) == -1


def _fwd(L, ptr, B=2, N=8, d=64, H=2, d_ff=256, dtype=R.RT_F32, sched=0, driver=0, ws_bytes=1 << 30,
         ws=None):
    p = [ctypes.c_void_p(ptr)] * 7
    out = [ctypes.c_void_p(ptr)] * 3
    return L.rt_layer_forward(*p, B, N, d, H, d_ff, dtype, sched, driver, *out,
                              ctypes.c_void_p(ptr if ws is None else ws), ctypes.c_size_t(ws_bytes), None)


def test_forward_argument_validation_happens_before_any_launch(L):
    fake = 1 << 40                                       # never dereferenced
    assert _fwd(L, 0) == R.RT_ERR_INVALID_ARG           # null pointers
    assert _fwd(L, fake + 4) == R.RT_ERR_INVALID_ARG    # misaligned tensors
    assert _fwd(L, fake, dtype=5) == R.RT_ERR_INVALID_ARG
    assert _fwd(L, fake, driver=9) == R.RT_ERR_INVALID_ARG
    assert _fwd(L, fake, H=3) == R.RT_ERR_INVALID_ARG
    assert _fwd(L, fake, dtype=R.RT_BF16) == R.RT_ERR_UNSUPPORTED   # d_h = 32 in bf16
    assert _fwd(L, fake, ws_bytes=100) == R.RT_ERR_WORKSPACE
    assert _fwd(L, fake, ws=fake + 128) == R.RT_ERR_WORKSPACE        # workspace not 256-aligned


def test_no_device_is_reported_not_faked(L):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments: the library must refuse to run rather than compute on the CPU
    assert _fwd(L, 1 << 40) == R.RT_ERR_DEVICE
    assert L.rt_gemm_bf16(ctypes.c_void_p(1 << 40), ctypes.c_void_p(1 << 40),
                          ctypes.cast(ctypes.c_void_p(1 << 40), ctypes.POINTER(ctypes.c_float)),
                          128, 128, 64, ctypes.c_void_p(1 << 40), None) == R.RT_ERR_DEVICE
    # the allocation-free projection sets up the device first, too
    assert L.rt_project_qkv_noalloc(ctypes.c_void_p(1 << 40), ctypes.c_void_p(1 << 40), 2, 8, 64,
                                    ctypes.c_void_p(1 << 40), None) == R.RT_ERR_DEVICE
    assert L.rt_project_qkv_noalloc_status(None) == R.RT_ERR_DEVICE


def test_component_entry_points_require_an_error_word(L):
    # the tensor-core kernels behind these calls record bounded-wait timeouts
    # in err_dev; a call without one (or with a misaligned one) is refused
    # before anything is enqueued
    p = ctypes.c_void_p(1 << 40)
    fp = ctypes.cast(p, ctypes.POINTER(ctypes.c_float))
    for err, want in ((None, R.RT_ERR_INVALID_ARG), (ctypes.c_void_p((1 << 40) + 2), R.RT_ERR_INVALID_ARG)):
        assert L.rt_gemm_bf16(p, p, fp, 128, 128, 64, err, None) == want
        assert L.rt_project_qkv(p, p, 2, 8, 64, R.RT_BF16, p, p, err, None) == want
        assert L.rt_block_fold(p, 192, p, p, 64, fp, fp, fp, 2, 1, 64, 4, 4, 0, 4, R.RT_BF16, err, None) == want


def test_noalloc_validation_happens_before_any_launch(L):
    p = ctypes.c_void_p(1 << 40)
    call = L.rt_project_qkv_noalloc
    assert call(None, p, 2, 8, 64, p, None) == R.RT_ERR_INVALID_ARG
    assert call(p, p, 0, 8, 64, p, None) == R.RT_ERR_INVALID_ARG
    assert call(p, p, 2, 8, 96, p, None) == R.RT_ERR_UNSUPPORTED       # d % 64 != 0
    # B*N = 2^20 + 1 rows: beyond the fixed scratch array
    assert call(p, p, 1025, 1024, 64, p, None) == R.RT_ERR_WORKSPACE


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(R, "_lib", None)
    monkeypatch.setattr(R, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        R.lib()


def _param_counts():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(rt_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_header(L):
    counts = _param_counts()
    assert len(counts) == len(R.EXPORTS)
    for name, n in counts.items():
        fn = getattr(L, name)
        got = len(fn.argtypes) if fn.argtypes is not None else 0
        assert got == n, f"{name}: binding declares {got} arguments, header {n}"


def test_recompute_validation_happens_before_any_launch(L):
    assert L.rt_layer_recompute_workspace_bytes(4, 16, 128) >= 256 + 4 * 16 * 4 + 2 * 128 * 128 * 2
    assert L.rt_layer_recompute_workspace_bytes(4, 16, 96) == 0          # d % 64 != 0
    assert L.rt_layer_recompute_workspace_bytes(0, 16, 128) == 0
    p = ctypes.c_void_p(1 << 40)
    big = ctypes.c_size_t(1 << 30)
    call = L.rt_layer_recompute_kv
    assert call(None, p, p, 4, 16, 128, p, p, p, big, None) == R.RT_ERR_INVALID_ARG
    assert call(p, p, p, 4, 16, 96, p, p, p, big, None) == R.RT_ERR_UNSUPPORTED
    assert call(ctypes.c_void_p((1 << 40) + 8), p, p, 4, 16, 128, p, p, p, big, None) == R.RT_ERR_INVALID_ARG
    assert call(p, p, p, 4, 16, 128, p, p, p, ctypes.c_size_t(64), None) == R.RT_ERR_WORKSPACE


def test_pages_entry_point_validation_happens_before_any_launch(L):
    p = ctypes.c_void_p(1 << 40)

    def call(Lv=1, d=128, H=2, ws_bytes=1 << 34, driver=R.RT_DRIVER_GRAPH):
        return L.rt_layer_forward_pages(*([p] * 7), 2, 16, d, H, 256, Lv, p, p, p, p, ctypes.c_size_t(ws_bytes),
                                        None, driver)
    assert call(Lv=0) == R.RT_ERR_INVALID_ARG          # the stack depth L >= 1
    assert call(d=96, H=2) == R.RT_ERR_UNSUPPORTED       # bf16 needs d_h = 64
    assert call(ws_bytes=16) == R.RT_ERR_WORKSPACE
    assert call(driver=7) == R.RT_ERR_INVALID_ARG
    assert L.rt_layer_forward_pages(None, *([p] * 6), 2, 16, 128, 2, 256, 1, p, p, p, p,
                                    ctypes.c_size_t(1 << 34), None, R.RT_DRIVER_GRAPH) == R.RT_ERR_INVALID_ARG


def test_chunked_entry_point_validation_happens_before_any_launch(L):
    assert L.rt_layer_chunked_workspace_bytes(4, 64, 128, 2, 256, 16) > L.rt_layer_chunked_workspace_bytes(
        4, 64, 128, 2, 256, 1)                                        # per-step buffers hold B x C rows
    assert L.rt_layer_chunked_workspace_bytes(4, 64, 128, 2, 256, 0) == 0
    assert L.rt_layer_chunked_workspace_bytes(4, 64, 96, 2, 256, 4) == 0   # bf16 needs d_h = 64
    p = ctypes.c_void_p(1 << 40)

    def call(C=4, ws_bytes=1 << 34):
        return L.rt_layer_forward_chunked(*([p] * 7), 4, 64, 128, 2, 256, C, p, p, p, p,
                                          ctypes.c_size_t(ws_bytes), None)
    assert call(C=0) == R.RT_ERR_INVALID_ARG
    assert call(ws_bytes=16) == R.RT_ERR_WORKSPACE
